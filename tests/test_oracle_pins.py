"""Pins of the CPU oracle against facts other than itself.

Each test ties an oracle function to something its own code cannot fake: a
value the pages print, a closed form, a textbook/library routine on a
special case, an invariant of the definition, or brute force on tiny inputs.
Citations name the page title and section.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp as scipy_logsumexp

import oracle
from gen import counter_hash as ch
from gen import recipes

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16(x):
    return ch.f32_to_bf16_bits(np.asarray(x, dtype=np.float64))


# --------------------------------------------------------------- accounting

def test_kv_cache_size_worked_example():
    """Page "长上下文：稀疏注意力 / DSA / IndexShare", "动手：算清两堵墙": the
    printed output 0.2 / 7.0 / 53.4 GiB."""
    rows = []
    with open(os.path.join(GOLDEN, "kv_cache_size.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if not line:
                continue
            if line[0] == "per_token_kib":
                per_tok = int(line[1])
                continue
            rows.append([int(v) for v in line[:5]] + [line[5]])
    assert len(rows) == 3
    for n_layers, kv_heads, head_dim, bytes_per, n_tok, expect in rows:
        got = oracle.kv_cache_gib(n_layers, kv_heads, head_dim, n_tok, bytes_per)
        assert f"{got:.1f}" == expect
    one_tok = oracle.kv_cache_gib(28, 4, 128, 1, 2) * 1024 ** 3
    assert one_tok == per_tok * 1024


def test_pair_counts_at_1m():
    """Same page and section: 1e12 full pairs, 82 亿 with a 8192 window
    (1/122), 20.5 亿 with top-k 2048 (1/488), each as rounded on the page."""
    vals = {}
    with open(os.path.join(GOLDEN, "pair_counts.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if line:
                vals[line[0]] = line[1:]
    n = int(vals["n"][0])
    pc = oracle.pair_counts(n, 8192, 2048)
    for key, name in (("full", "full"), ("window", "window8192"), ("topk", "topk2048")):
        printed, unit, sig, ratio = vals[name]
        # the page rounds to the significant digits it prints
        assert float(f"{pc[key] / float(unit):.{int(sig)}g}") == float(printed)
        assert round(pc["full"] / pc[key]) == int(ratio)


# ------------------------------------------------------------------ scores

def test_index_scores_one_hot_query_reads_a_key_column():
    """A one-hot indexer query e_c scores each key by its c-th entry; a
    transposed operand or wrong axis fails this."""
    rng = _rng(1)
    k = rng.integers(-4, 5, size=(37, 16))
    for c in (0, 5, 15):
        q = np.zeros((1, 16))
        q[0, c] = 1.0
        s = oracle.index_scores(_bf16(q), _bf16(k))
        np.testing.assert_array_equal(s[0], k[:, c])
    q2 = np.zeros((2, 16))
    q2[0, 3] = 2.0
    q2[1, 7] = -1.0
    s = oracle.index_scores(_bf16(q2), _bf16(k))
    np.testing.assert_array_equal(s[0], 2 * k[:, 3])
    np.testing.assert_array_equal(s[1], -k[:, 7])


def test_index_scores_integer_inputs_are_exact():
    rng = _rng(2)
    q = rng.integers(-4, 5, size=(5, 128))
    k = rng.integers(-4, 5, size=(50, 128))
    s = oracle.index_scores(_bf16(q), _bf16(k))
    exact = np.array([[sum(int(a) * int(b) for a, b in zip(qr, kr)) for kr in k] for qr in q])
    np.testing.assert_array_equal(s, exact)
    assert np.abs(s).max() <= 16 * 128


# --------------------------------------------------------------- selection

def _brute_topk(scores, k):
    """Brute force over all k-subsets: largest total score, then the
    lexicographically smallest sorted position tuple (the lower-position
    tie-break).  Independent of any sort of the scores."""
    n = len(scores)
    kk = min(k, n)
    best = None
    for sub in itertools.combinations(range(n), kk):
        key = (sum(scores[i] for i in sub), tuple(-i for i in sub))
        if best is None or key > best[0]:
            best = (key, sub)
    return np.array(best[1], dtype=np.int64)


def test_topk_matches_brute_force_on_tiny_rows():
    rng = _rng(3)
    for trial in range(300):
        n = int(rng.integers(1, 10))
        k = int(rng.integers(1, 11))
        scores = [int(v) for v in rng.integers(-3, 4, size=n)]  # many ties
        got = oracle.topk_select(np.array(scores, dtype=np.float64), k)
        np.testing.assert_array_equal(got, _brute_topk(scores, k))


def test_topk_set_dominates_its_complement():
    """Every chosen element beats every unchosen one under (score desc,
    position asc); the result is ascending and of size min(k, n)."""
    rng = _rng(4)
    for trial in range(50):
        n = int(rng.integers(1, 3000))
        k = int(rng.integers(1, 600))
        s = rng.integers(-40, 41, size=n).astype(np.float64)
        sel = oracle.topk_select(s, k)
        assert sel.size == min(k, n)
        assert np.all(np.diff(sel) > 0)
        mask = np.zeros(n, bool)
        mask[sel] = True
        if mask.all():
            continue
        worst_in = min(zip(-s[mask], np.nonzero(mask)[0]), key=lambda t: (-t[0], -t[1]))
        rest = np.nonzero(~mask)[0]
        for u in rest[:200]:
            # chosen (worst) must rank before u
            assert (-worst_in[0] > s[u]) or (-worst_in[0] == s[u] and worst_in[1] < u)


def test_topk_special_cases():
    # all-equal scores -> the first k positions
    np.testing.assert_array_equal(oracle.topk_select(np.zeros(100), 7), np.arange(7))
    # fewer candidates than k -> all of them
    np.testing.assert_array_equal(oracle.topk_select(np.array([3.0, -1.0, 2.0]), 10), [0, 1, 2])
    # -0.0 and +0.0 compare equal (position decides)
    np.testing.assert_array_equal(oracle.topk_select(np.array([-0.0, 0.0, -1.0]), 1), [0])
    np.testing.assert_array_equal(oracle.topk_select(np.array([-1.0, -0.0, 0.0]), 1), [1])
    with pytest.raises(ValueError):
        oracle.topk_select(np.array([1.0, np.nan]), 1)


def test_index_topk_causal_rows_take_everything_below_k():
    """Config-1 shape on a small scale: query t has t+1 causal candidates,
    so rows with t+1 <= k keep every earlier position."""
    rng = _rng(5)
    L, d, k = 300, 16, 64
    q = _bf16(rng.integers(-4, 5, size=(1, L, d)))
    kk = _bf16(rng.integers(-4, 5, size=(1, L, d)))
    idx, count = oracle.index_topk(q, kk, L, 0, k)
    for t in range(L):
        assert count[0, t] == min(k, t + 1)
        if t + 1 <= k:
            np.testing.assert_array_equal(idx[0, t, : t + 1], np.arange(t + 1))
            assert np.all(idx[0, t, t + 1:] == -1)
        assert idx[0, t, : count[0, t]].max() <= t


def test_index_topk_decode_lengths_per_sequence():
    rng = _rng(6)
    B, T, d, k = 3, 50, 8, 10
    q = _bf16(rng.integers(-4, 5, size=(B, 1, d)))
    kk = _bf16(rng.integers(-4, 5, size=(B, T, d)))
    lens = np.array([50, 7, 0])
    idx, count = oracle.index_topk(q, kk, lens, 10 ** 9, k)
    assert list(count[:, 0]) == [10, 7, 0]
    assert np.all(idx[2, 0] == -1)
    np.testing.assert_array_equal(idx[1, 0, :7], np.arange(7))


def test_planted_needles_are_retrieved():
    """Planted needle (p, t): k_idx[p] = 8 q_idx[t].  For integer q != 0 with
    entries in [-4, 4], 8|q|^2 >= 8|q|_1 > 4|q|_1 >= any unplanted score, so
    only the other planted rows can outrank p, and p is in the top-k."""
    cfg = recipes.Prefill("needle_small", seed=11, B=1, L=4096, d=64, Hq=4, Hkv=1, D=128,
                          k=64, n_layers=1, share_every=1, n_needles=32)
    inp = recipes.prefill_host_inputs(cfg, with_attention=False)
    q, kk = inp["q_idx"][0], inp["k_idx"][0]
    pairs = recipes.needle_pairs(cfg)
    for p, t in pairs:
        qv = oracle.bf16_bits_to_f64(q[0, t])
        s = oracle.index_scores(q[0, t:t + 1], kk[0, : t + 1])[0]
        assert s[p] == 8 * float(qv @ qv)
        sel = oracle.topk_select(s, cfg.k)
        assert p in set(sel.tolist())


# --------------------------------------------------------------- attention

def _sdpa_dense_causal(q, K, V):
    """torch's scaled_dot_product_attention (float64, causal) with each kv
    head repeated for its query heads: the textbook dense attention."""
    Tq, Hq, D = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(np.repeat(K, G, axis=1)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(np.repeat(V, G, axis=1)).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return o[0].permute(1, 0, 2).numpy()


def test_sparse_attention_with_k_at_least_context_is_dense_causal():
    """[YOIO] §1.1: with every causal key selected, sparse attention is
    softmax(QK^T/sqrt(d))V with a causal mask."""
    rng = _rng(7)
    L, Hq, Hkv, D, d = 40, 4, 2, 32, 8
    qi = _bf16(rng.integers(-4, 5, size=(1, L, d)))
    ki = _bf16(rng.integers(-4, 5, size=(1, L, d)))
    idx, count = oracle.index_topk(qi, ki, L, 0, L)
    q = rng.standard_normal((1, L, Hq, D))
    K = rng.standard_normal((1, L, Hkv, D))
    V = rng.standard_normal((1, L, Hkv, D))
    out, _ = oracle.sparse_attention(q, K, V, idx, count)
    ref = _sdpa_dense_causal(q[0], K[0], V[0])
    np.testing.assert_allclose(out[0], ref, rtol=1e-12, atol=1e-12)


def _sdpa_over_rows(q, K_rows, V_rows):
    """torch's scaled_dot_product_attention (float64, no mask) of one query
    token's heads over its own selected rows, each kv head repeated for its
    query heads."""
    Hq, D = q.shape
    Hkv = K_rows.shape[1]
    G = Hq // Hkv
    qt = torch.from_numpy(np.ascontiguousarray(q))[:, None, :]                          # [Hq, 1, D]
    kt = torch.from_numpy(np.repeat(K_rows, G, axis=1)).permute(1, 0, 2)               # [Hq, n, D]
    vt = torch.from_numpy(np.repeat(V_rows, G, axis=1)).permute(1, 0, 2)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[:, 0].numpy()  # [Hq, D]


def test_sparse_attention_decode_each_sequence_attends_over_its_own_rows():
    """[YOIO] §1.1 and §2.3 per decode sequence: sequence b's query heads
    attend over sequence b's selected rows only.  Four sequences with
    different row counts (one empty, between two full ones) against torch's
    SDPA on each sequence alone; an output computed from another sequence's
    query or rows, or a batch broadcast, differs."""
    rng = _rng(21)
    Hq, Hkv, D = 8, 2, 16
    counts = [5, 0, 37, 12]
    B = len(counts)
    q = rng.standard_normal((B, Hq, D)) * 2
    Kr = [rng.standard_normal((n, Hkv, D)) for n in counts]
    Vr = [rng.standard_normal((n, Hkv, D)) for n in counts]
    out, lse = oracle.sparse_attention_decode(q, Kr, Vr)
    assert out.shape == (B, Hq, D) and lse.shape == (B, Hq)
    scale = 1.0 / math.sqrt(D)
    for b, n in enumerate(counts):
        if n == 0:
            assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        np.testing.assert_allclose(out[b], _sdpa_over_rows(q[b], Kr[b], Vr[b]), rtol=1e-12, atol=1e-12)
        G = Hq // Hkv
        for h in range(Hq):
            z = Kr[b][:, h // G] @ q[b, h] * scale
            assert abs(lse[b, h] - scipy_logsumexp(z)) < 1e-12
    # each sequence alone gives the same result as inside the batch
    for b in (0, 2, 3):
        o1, l1 = oracle.sparse_attention_decode(q[b:b + 1], Kr[b:b + 1], Vr[b:b + 1])
        np.testing.assert_array_equal(o1[0], out[b])
        np.testing.assert_array_equal(l1[0], lse[b])


def test_sparse_attention_batched_with_per_sequence_indices():
    """Prefill sparse attention at B = 2 with different indices per sequence
    and row: each (b, t) against torch's SDPA with a boolean mask holding
    exactly row t's selected positions of sequence b's cache."""
    rng = _rng(22)
    B, T, Hq, Hkv, D, k = 2, 12, 4, 2, 16, 5
    q = rng.standard_normal((B, T, Hq, D))
    K = rng.standard_normal((B, T, Hkv, D))
    V = rng.standard_normal((B, T, Hkv, D))
    idx = np.full((B, T, k), -1, np.int32)
    count = np.zeros((B, T), np.int32)
    for b in range(B):
        for t in range(T):
            n = min(k, t + 1) - (b * t) % 2      # sequences differ in counts as well as positions
            sel = np.sort(rng.choice(t + 1, size=max(n, 1), replace=False))
            idx[b, t, : sel.size] = sel
            count[b, t] = sel.size
    out, _ = oracle.sparse_attention(q, K, V, idx, count)
    G = Hq // Hkv
    for b in range(B):
        mask = np.zeros((T, T), dtype=bool)
        for t in range(T):
            mask[t, idx[b, t, : count[b, t]]] = True
        qt = torch.from_numpy(q[b]).permute(1, 0, 2)
        kt = torch.from_numpy(np.repeat(K[b], G, axis=1)).permute(1, 0, 2)
        vt = torch.from_numpy(np.repeat(V[b], G, axis=1)).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask))
        np.testing.assert_allclose(out[b], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_attention_output_is_convex_combination_of_selected_rows():
    rng = _rng(8)
    Hq, Hkv, D, n = 8, 2, 16, 33
    q = rng.standard_normal((Hq, D)) * 3
    K = rng.standard_normal((n, Hkv, D))
    V = rng.standard_normal((n, Hkv, D))
    o, lse = oracle.attention_over_rows(q, K, V)
    G = Hq // Hkv
    for h in range(Hq):
        g = h // G
        assert np.all(o[h] <= V[:, g].max(axis=0) + 1e-12)
        assert np.all(o[h] >= V[:, g].min(axis=0) - 1e-12)
    # weights sum to one: V = 1 everywhere gives 1
    o1, _ = oracle.attention_over_rows(q, K, np.ones_like(V))
    np.testing.assert_allclose(o1, 1.0, rtol=0, atol=1e-12)
    # one constant V row repeated gives that row
    row = rng.standard_normal((Hkv, D))
    oc, _ = oracle.attention_over_rows(q, K, np.broadcast_to(row, V.shape).copy())
    for h in range(Hq):
        np.testing.assert_allclose(oc[h], row[h // G], atol=1e-12)


def test_attention_special_cases():
    rng = _rng(9)
    D = 8
    K = rng.standard_normal((5, 1, D))
    V = rng.standard_normal((5, 1, D))
    # q = 0: uniform weights -> mean of the selected V rows; lse = log n
    o, lse = oracle.attention_over_rows(np.zeros((2, D)), K, V)
    np.testing.assert_allclose(o, np.broadcast_to(V[:, 0].mean(axis=0), (2, D)), atol=1e-12)
    np.testing.assert_allclose(lse, math.log(5), atol=1e-12)
    # two rows whose scaled scores differ by delta: weight = logistic(delta)
    q = np.zeros((1, D))
    q[0, 0] = 1.0
    K2 = np.zeros((2, 1, D))
    K2[0, 0, 0] = 2.0
    V2 = np.zeros((2, 1, D))
    V2[0, 0, :] = 1.0
    o2, _ = oracle.attention_over_rows(q, K2, V2, scale=1.5)
    w = 1.0 / (1.0 + math.exp(-3.0))
    np.testing.assert_allclose(o2[0], w, atol=1e-12)
    # empty selection
    o3, l3 = oracle.attention_over_rows(np.ones((3, D)), np.zeros((0, 1, D)), np.zeros((0, 1, D)))
    assert np.all(o3 == 0) and np.all(np.isneginf(l3))


def test_attention_is_invariant_to_the_order_of_selected_rows():
    rng = _rng(10)
    q = rng.standard_normal((4, 16))
    K = rng.standard_normal((20, 2, 16))
    V = rng.standard_normal((20, 2, 16))
    perm = rng.permutation(20)
    o1, l1 = oracle.attention_over_rows(q, K, V)
    o2, l2 = oracle.attention_over_rows(q, K[perm], V[perm])
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_lse_is_log_sum_exp_of_scaled_scores():
    from scipy.special import logsumexp
    rng = _rng(12)
    q = rng.standard_normal((2, 32))
    K = rng.standard_normal((9, 1, 32))
    V = rng.standard_normal((9, 1, 32))
    _, lse = oracle.attention_over_rows(q, K, V, scale=0.3)
    for h in range(2):
        np.testing.assert_allclose(lse[h], logsumexp(0.3 * K[:, 0] @ q[h]), atol=1e-12)


# -------------------------------------------------------------------- gist

def test_gist_equal_scores_take_the_first_chunks():
    n_chunks, cl, kc = 50, 16, 8
    gk = np.zeros((n_chunks, 4))
    for p in (0, 5, 16):
        rows, chunks = oracle.gist_route_unfold(np.ones(4), gk, cl, kc, p)
        np.testing.assert_array_equal(chunks, np.arange(kc))
        assert rows.size == kc * (cl + 1) + p
        np.testing.assert_array_equal(rows[: kc * 17], np.arange(kc * 17))
        np.testing.assert_array_equal(rows[kc * 17:], n_chunks * 17 + np.arange(p))


def test_gist_hand_worked_example():
    """4 chunks of 2 raw tokens + 1 gist (stride 3); gist scores
    [1, 5, -2, 5] with k = 2 keep chunks 1 and 3; rows are written out by
    hand from the interleaved layout, then the 2-token partial chunk."""
    gk = np.array([[1.0], [5.0], [-2.0], [5.0]])
    rows, chunks = oracle.gist_route_unfold(np.array([1.0]), gk, chunk_len=2, k_chunks=2, partial_len=2)
    assert chunks.tolist() == [1, 3]
    assert rows.tolist() == [3, 4, 5, 9, 10, 11, 12, 13]
    # more chunks requested than exist -> all chunks
    rows, chunks = oracle.gist_route_unfold(np.array([1.0]), gk, chunk_len=2, k_chunks=9, partial_len=0)
    assert chunks.tolist() == [0, 1, 2, 3]
    assert rows.tolist() == list(range(12))


# ----------------------------------------------------------------- sharing

def test_layer_owners_every_four_layers():
    """[LC] "DSA 与 IndexShare": every 4 layers share one indexer result;
    [IC] §五: 75% of indexer computation removed -> 1 full layer in 4."""
    owners = oracle.layer_owners(28, share_every=4)
    assert owners == [4 * (l // 4) for l in range(28)]
    full = sum(1 for l, o in enumerate(owners) if o == l)
    assert full == 7 and 1 - full / 28 == 0.75


def test_layer_owners_pattern():
    """[IC] §二: a shared layer reuses the nearest full layer before it."""
    assert oracle.layer_owners(6, pattern="FSSFSF") == [0, 0, 0, 3, 3, 5]
    assert oracle.layer_owners(1, pattern="F") == [0]
    for bad in ("SFF", "FX", "FF"):
        with pytest.raises(ValueError):
            oracle.layer_owners(3, pattern=bad)


# ------------------------------------------------------- the pins catch slips
#
# Plausible slips planted in the oracle (on the CPU, through monkeypatch)
# must make the batch pins above fail.

def _mutant_decode_swapped(q, Kr, Vr, scale=None):
    B = len(Kr)
    return _ORIG_DECODE(q, [Kr[(b + 1) % B] for b in range(B)], [Vr[(b + 1) % B] for b in range(B)], scale)


def _mutant_decode_first_query(q, Kr, Vr, scale=None):
    q = np.asarray(q)
    return _ORIG_DECODE(np.broadcast_to(q[:1], q.shape).copy(), Kr, Vr, scale)


def _mutant_prefill_first_cache(q, K, V, idx, count, scale=None):
    K = np.asarray(K)
    V = np.asarray(V)
    return _ORIG_PREFILL(q, np.broadcast_to(K[:1], K.shape).copy(), np.broadcast_to(V[:1], V.shape).copy(),
                         idx, count, scale)


_ORIG_DECODE = oracle.sparse_attention_decode
_ORIG_PREFILL = oracle.sparse_attention


@pytest.mark.parametrize("mutant", [_mutant_decode_swapped, _mutant_decode_first_query])
def test_decode_pin_catches_batch_slips(monkeypatch, mutant):
    monkeypatch.setattr(oracle, "sparse_attention_decode", mutant)
    with pytest.raises(AssertionError):
        test_sparse_attention_decode_each_sequence_attends_over_its_own_rows()


def test_prefill_batch_pin_catches_a_shared_cache(monkeypatch):
    monkeypatch.setattr(oracle, "sparse_attention", _mutant_prefill_first_cache)
    with pytest.raises(AssertionError):
        test_sparse_attention_batched_with_per_sequence_indices()


# ------------------------------------------------------- multi-head indexer

def _mh_brute(q, w, k):
    """sum_h w[t,h] * max(0, q[t,h] . k[j]) in Python integers."""
    Tq, H, d = q.shape
    out = [[0] * k.shape[0] for _ in range(Tq)]
    for t in range(Tq):
        for j in range(k.shape[0]):
            tot = 0
            for h in range(H):
                dot = sum(int(q[t, h, c]) * int(k[j, c]) for c in range(d))
                tot += int(w[t, h]) * max(0, dot)
            out[t][j] = tot
    return np.array(out, dtype=np.float64)


def test_multihead_scores_match_python_integers():
    """The multi-head indexer (an extension of the pages' light indexer,
    [LC] "DSA 与 IndexShare") on integer inputs equals the sum over heads
    of weight x ReLU(dot) evaluated in Python integers."""
    rng = _rng(31)
    Tq, H, d, Tk = 3, 5, 7, 11
    q = rng.integers(-4, 5, size=(Tq, H, d))
    w = rng.integers(-3, 4, size=(Tq, H))
    k = rng.integers(-4, 5, size=(Tk, d))
    got = oracle.index_scores_multihead(_bf16(q), w.astype(np.float32), _bf16(k))
    np.testing.assert_array_equal(got, _mh_brute(q, w, k))


def test_multihead_special_cases():
    rng = _rng(32)
    Tq, d, Tk = 4, 16, 30
    q1 = rng.integers(-4, 5, size=(Tq, 1, d))
    k = rng.integers(-4, 5, size=(Tk, d))
    plain = oracle.index_scores(_bf16(q1[:, 0]), _bf16(k))
    # one head with weight 1 is the plain dot product clipped at zero
    one = oracle.index_scores_multihead(_bf16(q1), np.ones((Tq, 1)), _bf16(k))
    np.testing.assert_array_equal(one, np.maximum(plain, 0))
    # linear in the weights; invariant to the order of the heads
    H = 6
    q = rng.integers(-4, 5, size=(Tq, H, d))
    w1 = rng.integers(-3, 4, size=(Tq, H)).astype(np.float64)
    w2 = rng.integers(-3, 4, size=(Tq, H)).astype(np.float64)
    s = lambda ww, qq=q: oracle.index_scores_multihead(_bf16(qq), ww, _bf16(k))
    np.testing.assert_array_equal(s(w1 + w2), s(w1) + s(w2))
    perm = rng.permutation(H)
    np.testing.assert_array_equal(s(w1[:, perm], q[:, perm]), s(w1))
    # heads whose dot is negative everywhere contribute nothing
    qn = q.copy()
    qn[:, 0] = -1                             # head 0: q = -1 everywhere ...
    kp = np.abs(k) + 1                        # ... against all-positive keys
    a = oracle.index_scores_multihead(_bf16(qn), w1, _bf16(kp))
    b = oracle.index_scores_multihead(_bf16(qn[:, 1:]), w1[:, 1:], _bf16(kp))
    np.testing.assert_array_equal(a, b)


def test_multihead_topk_uses_the_weighted_scores():
    """index_topk with weights selects by the multi-head score, with the
    same tie rule, and one head of weight 1 over non-negative dots selects
    as the single-head indexer does."""
    rng = _rng(33)
    B, Tq, H, d, Tk, kk = 2, 5, 4, 8, 40, 7
    q = rng.integers(-4, 5, size=(B, Tq, H, d))
    w = rng.integers(0, 4, size=(B, Tq, H)).astype(np.float32)
    k = rng.integers(-4, 5, size=(B, Tk, d))
    idx, cnt = oracle.index_topk(_bf16(q), _bf16(k), Tk, Tk - Tq, kk, w=w)
    for b in range(B):
        sc = _mh_brute(q[b], w[b], k[b])
        for t in range(Tq):
            n = Tk - Tq + t + 1
            order = sorted(range(n), key=lambda j: (-sc[t, j], j))[:kk]
            np.testing.assert_array_equal(idx[b, t, :cnt[b, t]], sorted(order))
    qa = np.abs(rng.integers(0, 5, size=(1, Tq, 1, d)))
    ka = np.abs(rng.integers(0, 5, size=(1, Tk, d)))
    i1, _ = oracle.index_topk(_bf16(qa), _bf16(ka), Tk, Tk - Tq, kk, w=np.ones((1, Tq, 1)))
    i2, _ = oracle.index_topk(_bf16(qa[:, :, 0]), _bf16(ka), Tk, Tk - Tq, kk)
    np.testing.assert_array_equal(i1, i2)


def _mutant_mh_no_relu(q_idx, w, k_idx):
    q = oracle.bf16_bits_to_f64(q_idx)
    k = oracle.bf16_bits_to_f64(k_idx)
    return np.einsum("th,thj->tj", np.asarray(w, np.float64), np.einsum("thd,jd->thj", q, k))


def _mutant_mh_relu_after_sum(q_idx, w, k_idx):
    q = oracle.bf16_bits_to_f64(q_idx)
    k = oracle.bf16_bits_to_f64(k_idx)
    return np.maximum(np.einsum("th,thj->tj", np.asarray(w, np.float64), np.einsum("thd,jd->thj", q, k)), 0)


@pytest.mark.parametrize("mutant", [_mutant_mh_no_relu, _mutant_mh_relu_after_sum])
def test_multihead_pin_catches_slips(monkeypatch, mutant):
    monkeypatch.setattr(oracle, "index_scores_multihead", mutant)
    with pytest.raises(AssertionError):
        test_multihead_scores_match_python_integers()


# ------------------------------------------------------ two-level gist routing

def test_hier_gist_with_every_group_kept_is_single_level_routing():
    """[SSA] §五 / [GSA] 2.4: when the coarse stage keeps every group, the
    two-level routing is the single-level selective unfolding ([SSA] §三)."""
    rng = _rng(41)
    n_chunks, M, d = 50, 8, 16
    q = _bf16(rng.integers(-4, 5, size=d))
    gk = _bf16(rng.integers(-4, 5, size=(n_chunks, d)))
    mk = _bf16(rng.integers(-4, 5, size=(n_chunks // M, d)))
    for kc in (1, 5, 40, 60):
        rows, chunks, groups = oracle.hier_gist_route_unfold(q, mk, gk, M, 4, n_chunks // M, kc, 3)
        r1, c1 = oracle.gist_route_unfold(q, gk, 4, kc, 3)
        np.testing.assert_array_equal(chunks, c1)
        np.testing.assert_array_equal(rows, r1)
        np.testing.assert_array_equal(groups, np.arange(n_chunks // M))


def test_hier_gist_hand_worked_example():
    """Four groups of two chunks plus one trailing chunk (9 chunks, group
    size 2), d = 2, query (1, 0): the meta scores are the meta keys' first
    entries (3, 1, 4, 1): k_groups = 2 keeps groups 0 and 2 (chunks 0, 1, 4,
    5) and chunk 8 (no meta-gist yet) is a candidate too.  Gist scores of
    chunks 0..8 are (0, 2, 9, 9, 5, 1, 7, 7, 3): among the candidates the top
    3 are chunks 4 (5), 8 (3), 1 (2) -- chunks 2, 3, 6, 7 score higher but
    sit in groups the coarse stage dropped."""
    q = _bf16([1, 0])
    gk = _bf16([[0, 1], [2, 0], [9, 0], [9, 0], [5, 0], [1, 0], [7, 0], [7, 0], [3, 0]])
    mk = _bf16([[3, 0], [1, 0], [4, 0], [1, 0]])
    rows, chunks, groups = oracle.hier_gist_route_unfold(q, mk, gk, 2, 1, 2, 3, 1)
    np.testing.assert_array_equal(groups, [0, 2])
    np.testing.assert_array_equal(chunks, [1, 4, 8])
    # chunk_len 1: chunk c occupies rows 2c (raw) and 2c + 1 (gist); the partial chunk starts at 18
    np.testing.assert_array_equal(rows, [2, 3, 8, 9, 16, 17, 18])


def test_hier_gist_ties_take_lower_groups_and_chunks():
    q = _bf16([0, 0])
    gk = _bf16(np.ones((12, 2)))
    mk = _bf16(np.ones((3, 2)))
    _, chunks, groups = oracle.hier_gist_route_unfold(q, mk, gk, 4, 2, 2, 5, 0)
    np.testing.assert_array_equal(groups, [0, 1])
    np.testing.assert_array_equal(chunks, [0, 1, 2, 3, 4])


# ------------------------------------------------- index overlap, layer roles

def test_index_overlap_counts_shared_positions():
    """[IC] §一: the overlap of two selections, against Python sets."""
    rng = _rng(51)
    rows, k = 20, 30
    a = np.full((rows, k), -1, np.int32)
    b = np.full((rows, k), -1, np.int32)
    ca, cb = rng.integers(0, k + 1, rows), rng.integers(0, k + 1, rows)
    for r in range(rows):
        a[r, : ca[r]] = np.sort(rng.choice(60, ca[r], replace=False))
        b[r, : cb[r]] = np.sort(rng.choice(60, cb[r], replace=False))
    got = oracle.index_overlap(a, ca, b, cb)
    for r in range(rows):
        assert got[r] == len(set(a[r, : ca[r]].tolist()) & set(b[r, : cb[r]].tolist()))
    np.testing.assert_array_equal(oracle.index_overlap(a, ca, a, ca), ca)   # a selection overlaps itself fully


def test_greedy_pattern_hand_worked():
    """[IC] §三: greedy removal of the indexer whose loss is smallest.  Six
    layers in two blocks {0, 1, 2} and {3, 4, 5}: within a block the overlap
    is 0.9, across blocks 0.2.  Keeping two indexers, the search keeps the
    first layer of each block: "FSSFSS"."""
    L = 6
    ov = np.full((L, L), 0.2)
    for blk in ((0, 1, 2), (3, 4, 5)):
        for i in blk:
            for j in blk:
                ov[i, j] = 0.9
    np.fill_diagonal(ov, 1.0)
    assert oracle.greedy_pattern(ov, 2) == "FSSFSS"
    assert oracle.greedy_pattern(ov, 6) == "FFFFFF"
    assert oracle.greedy_pattern(ov, 1) == "FSSSSS"
    # equal losses everywhere: the lower layers go first
    assert oracle.greedy_pattern(np.ones((5, 5)), 3) == "FSSFF"


def test_greedy_pattern_is_exhaustive_optimum_when_one_indexer_is_removed():
    """Removing one indexer, the greedy step is the exhaustive best single
    removal (checked against every choice)."""
    rng = _rng(52)
    L = 7
    ov = rng.uniform(0.3, 1.0, (L, L))
    np.fill_diagonal(ov, 1.0)
    pat = oracle.greedy_pattern(ov, L - 1)
    owners = oracle.layer_owners(L, pat)
    got = sum(ov[l, owners[l]] for l in range(L))
    best = max(sum(ov[l, oracle.layer_owners(L, "".join("S" if i == r else "F" for i in range(L)))[l]]
                   for l in range(L)) for r in range(1, L))
    assert abs(got - best) < 1e-12


# ------------------------------------------------------------ fp8 (E4M3) inputs

def test_e4m3_decoder_format_values():
    """The E4M3 decoder (reading 10) against values the OCP FP8 format fixes:
    1.0 is exponent field 7 with a zero mantissa, the largest finite value is
    448 (field 15, mantissa 6), the smallest normal 2^-6, the smallest
    subnormal 2^-9, S.1111.111 is NaN, and there are no infinities."""
    dec = lambda c: float(oracle.e4m3_bits_to_f64(np.array([c], dtype=np.uint8))[0])
    assert dec(0x00) == 0.0 and dec(0x80) == 0.0 and math.copysign(1.0, dec(0x80)) == -1.0
    for code, value in [(0x38, 1.0), (0xB8, -1.0), (0x40, 2.0), (0x44, 3.0), (0x48, 4.0), (0xC8, -4.0),
                        (0x3C, 1.5), (0x7E, 448.0), (0xFE, -448.0), (0x08, 2.0 ** -6), (0x01, 2.0 ** -9),
                        (0x07, 7 * 2.0 ** -9), (0x0F, 1.875 * 2.0 ** -6), (0x77, 240.0), (0x78, 256.0)]:
        assert dec(code) == value, hex(code)
    assert math.isnan(dec(0x7F)) and math.isnan(dec(0xFF))
    vals = oracle.e4m3_bits_to_f64(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(vals) > 0), "positive codes must decode in increasing order"
    assert not np.isinf(oracle.e4m3_bits_to_f64(np.arange(256, dtype=np.uint8))).any()
    neg = oracle.e4m3_bits_to_f64(np.arange(0x80, 0xFF, dtype=np.uint8))
    np.testing.assert_array_equal(neg, -vals)


def test_e4m3_pin_catches_slips(monkeypatch):
    """A decoder with the exponent bias off by one, or subnormals scaled as
    normals, fails the format pin."""
    real = oracle.e4m3_bits_to_f64

    def bias8(codes):
        return real(codes) / 2.0

    def no_subnormal(codes):
        c = np.asarray(codes, dtype=np.uint8)
        v = real(c)
        sub = ((c >> 3) & 0xF) == 0
        return np.where(sub, np.where(c & 0x80, -1.0, 1.0) * (1 + (c & 7) / 8.0) * 2.0 ** -6 * (c & 7 > 0), v)

    for mutant in (bias8, no_subnormal):
        monkeypatch.setattr(oracle, "e4m3_bits_to_f64", mutant)
        with pytest.raises(AssertionError):
            test_e4m3_decoder_format_values()
    monkeypatch.setattr(oracle, "e4m3_bits_to_f64", real)


def test_fp8_inputs_select_as_the_same_integers_in_bf16():
    """Integer values in [-4, 4] are exact in E4M3, so the top-k of their
    E4M3 codes equals the top-k of their bf16 bits, one head and several."""
    rng = _rng(41)
    B, Tk, d, k = 3, 70, 64, 9
    q = rng.integers(-4, 5, size=(B, 1, d))
    kk = rng.integers(-4, 5, size=(B, Tk, d))
    lens = np.array([70, 33, 5])
    a = oracle.index_topk(ch.e4m3_codes(q), ch.e4m3_codes(kk), lens, Tk - 1, k)
    b = oracle.index_topk(_bf16(q), _bf16(kk), lens, Tk - 1, k)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    H = 6
    qh = rng.integers(-4, 5, size=(B, 1, H, d))
    w = rng.integers(-3, 4, size=(B, 1, H)).astype(np.float32)
    a = oracle.index_topk(ch.e4m3_codes(qh), ch.e4m3_codes(kk), Tk, Tk - 1, k, w=w)
    b = oracle.index_topk(_bf16(qh), _bf16(kk), Tk, Tk - 1, k, w=w)
    np.testing.assert_array_equal(a[0], b[0])
