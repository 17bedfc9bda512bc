"""GPU parity against the CPU oracle at sizes the oracle finishes in seconds.

Indices and counts must match bit for bit (integer-valued indexer inputs make
every fp32 score exact); attention outputs must be within max-abs 2e-2 and
mean-abs 2e-3 of the fp64 oracle.  Sizes span several tiles and ragged
tails; edge cases cover empty rows, k >= candidates, all-equal and signed-zero
scores, heavy ties and the candidate-overflow fallback."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import shared_top_routing_b200 as sa
from gen import counter_hash as ch
from tests.gpu_util import assert_close_attn, assert_lse_close, bits_of, dev, i32, to_dev

pytestmark = pytest.mark.gpu


def _ints(seed, tid, shape, lo=-4, hi=4):
    return ch.int_bf16(seed, tid, count=int(np.prod(shape)), lo=lo, hi=hi).reshape(shape)


def _normals(seed, tid, shape):
    return ch.normal_bf16(seed, tid, count=int(np.prod(shape))).reshape(shape)


# ---------------------------------------------------------------- decode top-k

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("k,lens,Tk_max", [
    (256, [3000, 1, 0, 257], 3000),            # direct mode, ragged, empty row, n = k + 1
    (7, [9999, 5000, 7, 6], 10007),            # n <= k rows
    (2048, [16385, 30000, 2047, 40000], 40000),  # candidate mode, several collect CTAs
    (4096, [50000, 4096, 4097, 100], 50000),   # largest k
    (1, [12345, 1, 20000], 20000),
])
def test_decode_topk_matches_oracle(d, k, lens, Tk_max):
    B = len(lens)
    seed = 1000 + d + k
    q = _ints(seed, 1, (B, d))
    kk = _ints(seed, 2, (B, Tk_max, d))
    idx, cnt, sc = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k, Tk=max(lens), q_pos0=10 ** 9,
                                          kv_len=i32(lens), with_scores=True)
    ridx, rcnt = oracle.index_topk(q[:, None, :], kk, np.array(lens), 10 ** 9, k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt[:, 0])
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx[:, 0])
    # scores of the chosen positions
    sc = sc.cpu().numpy()
    for b in range(B):
        n = rcnt[b, 0]
        if n:
            full = oracle.index_scores(q[b:b + 1], kk[b, ridx[b, 0, :n]])[0]
            np.testing.assert_array_equal(sc[b, :n], full)
        assert np.all(np.isneginf(sc[b, n:]))


@pytest.mark.parametrize("n", [5000, 60000])
def test_decode_topk_all_equal_and_signed_zero_scores(n):
    """q = 0 makes every score +0 or -0 (the sign of each key's entries):
    all compare equal, so the first k positions win.  n = 60000 overflows the
    candidate list and takes the full-row path."""
    d, k = 128, 2048
    q = np.zeros((1, d), np.uint16)
    kk = _ints(77, 3, (1, n, d), lo=-4, hi=0)      # many all-negative rows -> -0 scores
    kk[0, ::3] = ch.f32_to_bf16_bits(-np.ones(d))  # certainly -0
    idx, cnt = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k)
    torch.cuda.synchronize()
    assert cnt.item() == k
    np.testing.assert_array_equal(idx.cpu().numpy()[0], np.arange(k))


def test_decode_topk_heavy_ties():
    """A one-hot query gives only 9 distinct scores: huge tie groups at the
    threshold, decided by position."""
    d, n, k = 64, 40000, 3000
    q = np.zeros((2, d))
    q[0, 5] = 1.0
    q[1, 0] = -2.0
    qb = ch.f32_to_bf16_bits(q)
    kk = _ints(78, 4, (2, n, d))
    idx, cnt = sa.sa_index_score_topk(to_dev(qb), to_dev(kk), k)
    ridx, rcnt = oracle.index_topk(qb[:, None, :], kk, n, n - 1, k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx[:, 0])
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt[:, 0])


def test_decode_topk_q_pos0_limits_candidates():
    d, n, k = 64, 1000, 100
    q = _ints(79, 1, (1, d))
    kk = _ints(79, 2, (1, n, d))
    idx, cnt = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k, Tk=n, q_pos0=49)
    torch.cuda.synchronize()
    assert cnt.item() == 50
    np.testing.assert_array_equal(idx.cpu().numpy()[0, :50], np.arange(50))
    assert np.all(idx.cpu().numpy()[0, 50:] == -1)


# --------------------------------------------------------------- prefill top-k

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,L,k,Tk,q_pos0", [
    (1, 1, 16, 1, 0),
    (2, 77, 16, 77, 0),
    (1, 300, 64, 300, 0),
    (1, 1000, 256, 1000, 0),
    (2, 130, 40, 530, 400),     # chunked prefill: queries are the last 130 of 530 tokens
    (1, 64, 2048, 20000, 19936),  # rows longer than the in-smem limit: streamed row scan, 2 chunks
    (1, 16, 300, 40000, 39984),   # 4 chunks, small k
])
def test_prefill_topk_matches_oracle(d, B, L, k, Tk, q_pos0):
    seed = 2000 + L + d
    q = _ints(seed, 1, (B, L, d))
    kk = _ints(seed, 2, (B, Tk, d))
    idx, cnt = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k, Tk=Tk, q_pos0=q_pos0)
    ridx, rcnt = oracle.index_topk(q, kk, Tk, q_pos0, k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


# Rows of more than 8192 candidates take two scoring passes: the first keeps
# each group's maximum (groups of g = 1..128 positions, chosen per row), the
# k-th largest group maximum bounds the k-th key from below, the second keeps
# only the keys at or above the bound.

@pytest.mark.parametrize("k", [4096, 2048, 1024, 512, 256, 128, 64, 32, 7])
def test_prefill_topk_bounded_every_group_size(k):
    """~9000-candidate rows: k from 4096 down to 7 gives groups of 1 to 128
    positions; 200 rows span two row blocks with a ragged tail."""
    B, L, d = 1, 200, 64
    q_pos0 = 9000
    Tk = q_pos0 + L
    seed = 3100 + k
    q = _ints(seed, 1, (B, L, d))
    kk = _ints(seed, 2, (B, Tk, d))
    idx, cnt, score = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k, Tk=Tk, q_pos0=q_pos0, with_scores=True)
    ridx, rcnt = oracle.index_topk(q, kk, Tk, q_pos0, k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    s = oracle.index_scores(q[0], kk[0])
    got = score.cpu().numpy()[0]
    for t in (0, 77, L - 1):
        np.testing.assert_array_equal(got[t, :k], s[t, ridx[0, t]].astype(np.float32))


def test_prefill_topk_bounded_mixed_row_lengths():
    """One launch whose rows hold 3601..8200 candidates with k = 4096: rows
    of at most k candidates take every one, the rest are bounded."""
    B, L, d, k = 1, 4600, 64, 4096
    q_pos0 = 3600
    Tk = q_pos0 + L
    q = _ints(3201, 1, (B, L, d))
    kk = _ints(3201, 2, (B, Tk, d))
    idx, cnt = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k, Tk=Tk, q_pos0=q_pos0)
    ridx, rcnt = oracle.index_topk(q, kk, Tk, q_pos0, k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


@pytest.mark.parametrize("lo,hi", [(0, 0), (-1, 1)])
def test_prefill_topk_bounded_ties(lo, hi):
    """All-equal scores make every key a candidate (lists longer than shared
    memory, read in place); scores in [-64, 64] tie heavily at the bound."""
    B, L, d, k = 1, 130, 64, 2048
    q_pos0 = 12000
    Tk = q_pos0 + L
    q = _ints(3301 + hi, 1, (B, L, d), lo, hi)
    kk = _ints(3301 + hi, 2, (B, Tk, d), lo, hi)
    idx, cnt = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k, Tk=Tk, q_pos0=q_pos0)
    ridx, rcnt = oracle.index_topk(q, kk, Tk, q_pos0, k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


def test_prefill_topk_bounded_per_sequence_lengths():
    """Two sequences with cache lengths 20000 and 11000 in a 20480-row cache:
    the second sequence's rows are capped by its length."""
    B, L, d, k = 2, 150, 128, 1000
    Tk_max, Tk, q_pos0 = 20480, 20000, 19850
    q = _ints(3401, 1, (B, L, d))
    kk = _ints(3401, 2, (B, Tk_max, d))
    lens = np.array([20000, 11000], np.int32)
    idx, cnt = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k, Tk=Tk, q_pos0=q_pos0,
                                      kv_len=torch.from_numpy(lens).to(dev()))
    ridx, rcnt = oracle.index_topk(q, kk, lens, q_pos0, k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


def test_prefill_topk_bounded_several_batches():
    """A 2^20-row key buffer makes a batch 128 rows, so 300 queries over
    ~10000 live keys take three bounded batches (the later ones start past
    row 0 of the queries)."""
    B, L, d, k = 1, 300, 64, 512
    Tk_max, Tk = 1 << 20, 10000
    q_pos0 = Tk - L
    q = _ints(3501, 1, (B, L, d))
    kk = np.zeros((B, Tk_max, d), dtype=np.uint16)
    kk[:, :Tk] = _ints(3501, 2, (B, Tk, d))
    idx, cnt = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k, Tk=Tk, q_pos0=q_pos0)
    ridx, rcnt = oracle.index_topk(q, kk[:, :Tk], Tk, q_pos0, k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


def test_prefill_topk_real_valued_scores():
    """Non-integer bf16 inputs: the GPU's fp32 tile sums may differ from the
    fp64 oracle in the last bits, so compare sets via the oracle's scores:
    every chosen position must be valid and the chosen score sum must equal
    the oracle's within fp32 rounding."""
    B, L, d, k = 1, 400, 64, 50
    q = _normals(81, 1, (B, L, d))
    kk = _normals(81, 2, (B, L, d))
    idx, cnt = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k)
    ridx, rcnt = oracle.index_topk(q, kk, L, 0, k)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    s = oracle.index_scores(q[0], kk[0])
    for t in range(L):
        n = rcnt[0, t]
        got = idx[0, t, :n]
        assert np.all(np.diff(got) > 0) and got.max() <= t
        np.testing.assert_allclose(s[t, got].sum(), s[t, ridx[0, t, :n]].sum(), rtol=1e-5, atol=1e-3)


# ----------------------------------------------------------------- attention

# ------------------------------------------------------ multi-head indexer

def _weights(seed, shape, lo=-3, hi=3):
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=shape).astype(np.float32)


@pytest.mark.parametrize("d,H", [(64, 1), (64, 4), (64, 16), (64, 33), (64, 64), (128, 8), (128, 32)])
@pytest.mark.parametrize("lens,Tk_max,k", [([3000, 1700], 3000, 256), ([40000, 9000, 20000], 40000, 2048)])
def test_decode_multihead_topk_matches_oracle(d, H, lens, Tk_max, k):
    """Multi-head weighted indexer (sum over heads of weight x ReLU(q_h . k)),
    one query per sequence: indices and counts bit-exact against the oracle
    (integer inputs and weights keep every fp32 partial sum exact), with
    per-sequence lengths, head counts that fill one to four 16-head groups
    and negative weights."""
    B = len(lens)
    seed = 700 + d + H
    q = _ints(seed, 1, (B, H, d))
    w = _weights(seed, (B, H))
    kk = _ints(seed, 2, (B, Tk_max, d))
    idx, cnt, sc = sa.sa_index_score_topk_mh(to_dev(q), torch.from_numpy(w).to(dev()), to_dev(kk), k, Tk=Tk_max,
                                             q_pos0=Tk_max - 1, kv_len=i32(lens), with_scores=True)
    ridx, rcnt = oracle.index_topk(q[:, None], kk, np.array(lens), Tk_max - 1, k, w=w[:, None])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt[:, 0])
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx[:, 0])
    # the reported scores are the oracle's scores of the chosen positions
    sc = sc.cpu().numpy()
    for b, n in enumerate(lens):
        ref = oracle.index_scores_multihead(q[b][None], w[b][None], kk[b, :n])[0]
        c = rcnt[b, 0]
        np.testing.assert_array_equal(sc[b, :c], ref[ridx[b, 0, :c]])


@pytest.mark.parametrize("d,H,B,L,k", [(64, 16, 2, 300, 64), (128, 8, 1, 2500, 256), (64, 3, 1, 5000, 512)])
def test_prefill_multihead_topk_matches_oracle(d, H, B, L, k):
    """Causal prefill rows with the multi-head indexer: short rows (one CTA
    per row) and rows over 4096 candidates (slices over many CTAs)."""
    seed = 800 + d + H + L
    q = _ints(seed, 1, (B, L, H, d))
    w = _weights(seed, (B, L, H))
    kk = _ints(seed, 2, (B, L, d))
    idx, cnt = sa.sa_index_score_topk_mh(to_dev(q), torch.from_numpy(w).to(dev()), to_dev(kk), k)
    ridx, rcnt = oracle.index_topk(q, kk, L, 0, k, w=w)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)


def test_multihead_topk_ties_and_bad_arguments():
    """Zero weights make every score 0: the lowest positions win.  Head
    counts beyond the supported maximum and a missing weight pointer are
    refused on the host."""
    B, H, d, T, k = 2, 5, 64, 9000, 1000
    q = _ints(77, 1, (B, H, d))
    kk = _ints(77, 2, (B, T, d))
    w = torch.zeros((B, H), dtype=torch.float32, device=dev())
    idx, cnt = sa.sa_index_score_topk_mh(to_dev(q), w, to_dev(kk), k, Tk=T, q_pos0=T - 1)
    torch.cuda.synchronize()
    assert (cnt.cpu().numpy() == k).all()
    np.testing.assert_array_equal(idx.cpu().numpy(), np.tile(np.arange(k, dtype=np.int32), (B, 1)))
    L = sa.lib()
    fake = ctypes.c_void_p(0x100000)
    assert L.sa_index_score_topk_mh(fake, fake, fake, 1, 1, 65, 10, 10, 64, 4, 9, None, fake, fake, None,
                                    fake, 1 << 30, None) == sa.SA_ERR_UNSUPPORTED
    assert L.sa_index_score_topk_mh(fake, fake, fake, 1, 1, 33, 10, 10, 128, 4, 9, None, fake, fake, None,
                                    fake, 1 << 30, None) == sa.SA_ERR_UNSUPPORTED
    assert L.sa_index_score_topk_mh(fake, None, fake, 1, 1, 4, 10, 10, 64, 4, 9, None, fake, fake, None,
                                    fake, 1 << 30, None) == sa.SA_ERR_INVALID_ARG


# ------------------------------------------------------------- fp8 indexer

def _e4m3(seed, tid, shape, lo=-4, hi=4):
    return ch.int_e4m3(seed, tid, count=int(np.prod(shape)), lo=lo, hi=hi).reshape(shape)


def _u8(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).to(dev())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,k,lens,Tk_max", [
    (1, 256, [3000, 1, 0, 257], 3000),          # direct selection, ragged, empty row
    (1, 2048, [16385, 30000, 2047, 40000], 40000),   # split selection
    (1, 7, [9999, 5000, 7, 6], 10007),          # n <= k rows
    (4, 512, [9000, 4096, 4097, 1], 9000),      # multi-head, both sides of the split threshold
    (16, 2048, [33000, 20000], 33000),          # the 16-head workload's shape
    (32, 100, [5000, 3000, 4100], 5000),        # two head groups
])
def test_fp8_decode_topk_matches_oracle(d, H, k, lens, Tk_max):
    """fp8 (E4M3) queries and keys: indices, counts and scores bit-exact
    against the oracle on the same codes, and equal to the bf16 path's
    selection of the same integers."""
    B = len(lens)
    seed = 5000 + d + 7 * H + k
    q8 = _e4m3(seed, 1, (B, H, d))
    k8 = _e4m3(seed, 2, (B, Tk_max, d))
    w = _ints(seed, 3, (B, H), lo=-3, hi=3) if H > 1 else None
    wf = oracle.bf16_bits_to_f64(w).astype(np.float32) if w is not None else None
    wt = torch.from_numpy(wf).to(dev()) if w is not None else None
    idx, cnt, sc = sa.sa_index_score_topk_fp8(_u8(q8), _u8(k8), k, w=wt, Tk=max(lens), q_pos0=10 ** 9,
                                              kv_len=i32(lens), with_scores=True)
    if H == 1:
        ridx, rcnt = oracle.index_topk(q8[:, :, :].reshape(B, 1, d), k8, np.array(lens), 10 ** 9, k)
    else:
        ridx, rcnt = oracle.index_topk(q8[:, None], k8, np.array(lens), 10 ** 9, k, w=wf[:, None])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt[:, 0])
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx[:, 0])
    sc = sc.cpu().numpy()
    for b in range(B):
        n = rcnt[b, 0]
        if n:
            rows = k8[b, ridx[b, 0, :n]]
            if H == 1:
                full = oracle.index_scores(q8[b, :1], rows)[0]
            else:
                full = oracle.index_scores_multihead(q8[b][None], wf[b][None], rows)[0]
            np.testing.assert_array_equal(sc[b, :n], full)
        assert np.all(np.isneginf(sc[b, n:]))
    # the same integers through the bf16 indexer choose the same positions
    qb = oracle.e4m3_bits_to_f64(q8)
    kb = ch.f32_to_bf16_bits(oracle.e4m3_bits_to_f64(k8))
    if H == 1:
        bidx, bcnt = sa.sa_index_score_topk(to_dev(ch.f32_to_bf16_bits(qb[:, 0])), to_dev(kb), k, Tk=max(lens),
                                            q_pos0=10 ** 9, kv_len=i32(lens))
    else:
        bidx, bcnt = sa.sa_index_score_topk_mh(to_dev(ch.f32_to_bf16_bits(qb)), wt, to_dev(kb), k, Tk=max(lens),
                                               q_pos0=10 ** 9, kv_len=i32(lens))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bidx.cpu().numpy(), idx.cpu().numpy())
    np.testing.assert_array_equal(bcnt.cpu().numpy(), cnt.cpu().numpy())


def test_fp8_decode_topk_heavy_ties_and_float8_tensors():
    """A one-hot query gives 9 distinct scores, so the boundary is a huge tie
    group decided by position; torch.float8_e4m3fn tensors are accepted as
    they are."""
    d, n, k = 128, 40000, 3000
    q = np.zeros((2, d))
    q[0, 5] = 1.0
    q[1, 100] = -2.0
    k8 = _e4m3(91, 2, (2, n, d))
    q8 = ch.e4m3_codes(q)
    idx, cnt = sa.sa_index_score_topk_fp8(_u8(q8).view(torch.float8_e4m3fn), _u8(k8).view(torch.float8_e4m3fn), k)
    ridx, rcnt = oracle.index_topk(q8[:, None, :], k8, n, n - 1, k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt[:, 0])
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx[:, 0])


def test_fp8_device_codes_match_the_host_generator():
    """The device inputs of the fp8 workload (the bf16 integer tensors
    converted on the device) are the host generator's E4M3 codes."""
    from gen import torch_inputs as TI
    t = TI.dev_int((4, 1000, 64), 13, 7, dev())
    got = TI.to_e4m3(t).cpu().numpy()
    np.testing.assert_array_equal(got, _e4m3(13, 7, (4, 1000, 64)))


def _random_index(rng, B, Tk_max, k, counts):
    idx = np.full((B, k), -1, np.int32)
    for b, c in enumerate(counts):
        idx[b, :c] = np.sort(rng.choice(Tk_max, size=c, replace=False))
    return idx


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (28, 4), (8, 1), (16, 16), (24, 12), (15, 3)])
@pytest.mark.parametrize("k,counts", [(2048, [2048, 1000, 0, 1]), (100, [100, 33, 64, 7]),
                                      (1104, [1104, 1090, 1, 1089])])
def test_decode_attention_matches_oracle(Hq, Hkv, k, counts):
    rng = np.random.default_rng(Hq * 1000 + k)
    B, Tk_max, D = len(counts), 3000, 128
    q = _normals(3000 + Hq, 1, (B, Hq, D))
    K = _normals(3000 + Hq, 2, (B, Tk_max, Hkv, D))
    V = _normals(3000 + Hq, 3, (B, Tk_max, Hkv, D))
    idx = _random_index(rng, B, Tk_max, k, counts)
    out, lse = sa.sa_sparse_attn_decode(to_dev(q), to_dev(K), to_dev(V), i32(idx), i32(counts),
                                        with_lse=True)
    Kr = [K[b, idx[b, :c]] for b, c in enumerate(counts)]
    Vr = [V[b, idx[b, :c]] for b, c in enumerate(counts)]
    ref, rlse = oracle.sparse_attention_decode(q, Kr, Vr)
    torch.cuda.synchronize()
    assert_close_attn(out.float().cpu().numpy(), ref, "decode attention")
    assert_lse_close(lse.cpu().numpy(), rlse, "decode lse")


def test_decode_attention_scale_and_repeat_calls():
    """Explicit scale; two calls in a row reuse one workspace."""
    B, Hq, Hkv, D, Tk_max, k = 2, 8, 2, 128, 500, 300
    q = _normals(31, 1, (B, Hq, D))
    K = _normals(31, 2, (B, Tk_max, Hkv, D))
    V = _normals(31, 3, (B, Tk_max, Hkv, D))
    idx = _random_index(np.random.default_rng(5), B, Tk_max, k, [300, 250])
    ref, _ = oracle.sparse_attention_decode(q, [K[0, idx[0]], K[1, idx[1, :250]]],
                                            [V[0, idx[0]], V[1, idx[1, :250]]], scale=0.05)
    L = sa.lib()
    ws = torch.zeros(L.sa_sparse_attn_decode_workspace(B, Hq, Hkv, D, k), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        out = sa.sa_sparse_attn_decode(to_dev(q), to_dev(K), to_dev(V), i32(idx), i32([300, 250]),
                                       scale=0.05, ws=ws)
        torch.cuda.synchronize()
        assert_close_attn(out.float().cpu().numpy(), ref, "decode attention, scale 0.05")
        # the kernel error word is zero after a good call
        assert not ws[:4].cpu().numpy().any(), "decode workspace error word set"


@pytest.mark.parametrize("Hq,Hkv,k", [(32, 8, 2048), (28, 4, 2048), (16, 4, 100)])
def test_decode_attention_chained_after_an_index_run(Hq, Hkv, k):
    """A full layer's index run, then three layers attending over its index,
    launched back to back (each kernel may start while the one before it
    drains).  The newest key is forced into some sequences' selection.
    Every layer matches the oracle, and the index is unchanged."""
    B, T, d, D = 3, 9000, 128, 128
    qi = _ints(51, 1, (B, d))
    ki = _ints(51, 2, (B, T, d))
    for b in (0, 1):   # the newest key of sequences 0 and 1 is 8 x their query: selected
        ki[b, T - 1] = ch.f32_to_bf16_bits(8.0 * ch.bf16_bits_to_f64(qi[b]))
    ridx, rcnt = oracle.index_topk(qi[:, None, :], ki, T, T - 1, k)
    assert T - 1 in set(ridx[0, 0].tolist()) and T - 1 in set(ridx[1, 0].tolist())
    dev_in = [(_normals(52 + layer, 1, (B, Hq, D)), _normals(52 + layer, 2, (B, T, Hkv, D)),
               _normals(52 + layer, 3, (B, T, Hkv, D))) for layer in range(3)]
    dev_t = [tuple(to_dev(x) for x in trio) for trio in dev_in]
    idx_d, cnt_d = sa.sa_index_score_topk(to_dev(qi), to_dev(ki), k, Tk=T, q_pos0=T - 1)
    outs = [sa.sa_sparse_attn_decode(q, K, V, idx_d, cnt_d) for q, K, V in dev_t]
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx_d.cpu().numpy(), ridx[:, 0])
    for layer, ((q, K, V), out) in enumerate(zip(dev_in, outs)):
        ref, _ = oracle.sparse_attention_decode(q, [K[b, ridx[b, 0, : rcnt[b, 0]]] for b in range(B)],
                                                [V[b, ridx[b, 0, : rcnt[b, 0]]] for b in range(B)])
        assert_close_attn(out.float().cpu().numpy(), ref, f"layer {layer}")


# ------------------------------------------------- gather once, attend many

@pytest.mark.parametrize("Hkv,k,counts", [(8, 2048, [2048, 1000, 0]), (4, 100, [100, 37, 64]),
                                          (2, 1104, [1104, 1090, 5]), (1, 300, [1, 299, 300])])
def test_gather_rows_copies_the_selected_rows(Hkv, k, counts):
    """[YOIO] §2.1-§2.2: the selected rows of the shared cache, once, in
    selection order; zeros past each count."""
    rng = np.random.default_rng(k + Hkv)
    B, Tk_max = len(counts), 3000
    K = _normals(61, 2, (B, Tk_max, Hkv, 128))
    V = _normals(61, 3, (B, Tk_max, Hkv, 128))
    idx = _random_index(rng, B, Tk_max, k, counts)
    kr, vr = sa.sa_gather_rows(to_dev(K), to_dev(V), i32(idx), i32(counts))
    torch.cuda.synchronize()
    kr, vr = bits_of(kr), bits_of(vr)
    assert kr.shape == (B, k, Hkv * 128 + 8)
    assert not kr[:, :, Hkv * 128:].any() and not vr[:, :, Hkv * 128:].any()   # the row pads
    kr = kr[:, :, : Hkv * 128].reshape(B, k, Hkv, 128)
    vr = vr[:, :, : Hkv * 128].reshape(B, k, Hkv, 128)
    for b, c in enumerate(counts):
        np.testing.assert_array_equal(kr[b, :c], K[b, idx[b, :c]])
        np.testing.assert_array_equal(vr[b, :c], V[b, idx[b, :c]])
        assert not kr[b, c:].any() and not vr[b, c:].any()


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (28, 4), (8, 2), (8, 1), (15, 3)])
@pytest.mark.parametrize("k,counts", [(2048, [2048, 1000, 0, 1]), (100, [100, 33, 64, 7]), (1104, [1104, 1090, 1, 17])])
def test_decode_attention_over_compact_rows_matches_oracle(Hq, Hkv, k, counts):
    rng = np.random.default_rng(Hq * 100 + k)
    B, Tk_max, D = len(counts), 3000, 128
    q = _normals(4000 + Hq, 1, (B, Hq, D))
    K = _normals(4000 + Hq, 2, (B, Tk_max, Hkv, D))
    V = _normals(4000 + Hq, 3, (B, Tk_max, Hkv, D))
    idx = _random_index(rng, B, Tk_max, k, counts)
    kr, vr = sa.sa_gather_rows(to_dev(K), to_dev(V), i32(idx), i32(counts))
    out, lse = sa.sa_sparse_attn_decode_rows(to_dev(q), kr, vr, i32(counts), with_lse=True)
    ref, rlse = oracle.sparse_attention_decode(q, [K[b, idx[b, :c]] for b, c in enumerate(counts)],
                                               [V[b, idx[b, :c]] for b, c in enumerate(counts)])
    torch.cuda.synchronize()
    assert_close_attn(out.float().cpu().numpy(), ref, "attention over compact rows")
    assert_lse_close(lse.cpu().numpy(), rlse, "lse over compact rows")


def test_one_cache_one_index_gather_once_attend_many():
    """YOCO + CLSA ([YOIO] §2.1-§2.2): four layers share one KV cache and one
    index; the rows are gathered once and each layer attends over them with
    its own queries.  Every layer matches the oracle and the per-layer
    gathered path."""
    B, T, d, k, Hq, Hkv = 3, 9000, 128, 2048, 32, 8
    qi = _ints(62, 1, (B, d))
    ki = _ints(62, 2, (B, T, d))
    K = _normals(62, 3, (B, T, Hkv, 128))
    V = _normals(62, 4, (B, T, Hkv, 128))
    Kd, Vd = to_dev(K), to_dev(V)
    idx, cnt = sa.sa_index_score_topk(to_dev(qi), to_dev(ki), k, Tk=T, q_pos0=T - 1)
    kr, vr = sa.sa_gather_rows(Kd, Vd, idx, cnt)
    ridx, rcnt = oracle.index_topk(qi[:, None, :], ki, T, T - 1, k)
    Kr = [K[b, ridx[b, 0, : rcnt[b, 0]]] for b in range(B)]
    Vr = [V[b, ridx[b, 0, : rcnt[b, 0]]] for b in range(B)]
    for layer in range(4):
        q = _normals(63 + layer, 1, (B, Hq, 128))
        qd = to_dev(q)
        once = sa.sa_sparse_attn_decode_rows(qd, kr, vr, cnt)
        each = sa.sa_sparse_attn_decode(qd, Kd, Vd, idx, cnt)
        torch.cuda.synchronize()
        ref, _ = oracle.sparse_attention_decode(q, Kr, Vr)
        assert_close_attn(once.float().cpu().numpy(), ref, f"layer {layer}, gathered once")
        assert_close_attn(each.float().cpu().numpy(), ref, f"layer {layer}, gathered per layer")
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx[:, 0])


def test_decode_attention_many_sequences():
    """More (sequence, head block) pairs than CTAs: every CTA's range spans
    several pairs, some pairs are empty, and each pair has one contributor."""
    rng = np.random.default_rng(77)
    B, Hq, Hkv, D, Tk_max, k = 300, 8, 2, 128, 200, 64
    counts = [int(c) for c in rng.integers(0, k + 1, size=B)]
    counts[0], counts[1], counts[-1] = 0, k, 1
    q = _normals(41, 1, (B, Hq, D))
    K = _normals(41, 2, (B, Tk_max, Hkv, D))
    V = _normals(41, 3, (B, Tk_max, Hkv, D))
    idx = _random_index(rng, B, Tk_max, k, counts)
    out, lse = sa.sa_sparse_attn_decode(to_dev(q), to_dev(K), to_dev(V), i32(idx), i32(counts),
                                        with_lse=True)
    ref, rlse = oracle.sparse_attention_decode(q, [K[b, idx[b, :c]] for b, c in enumerate(counts)],
                                               [V[b, idx[b, :c]] for b, c in enumerate(counts)])
    torch.cuda.synchronize()
    assert_close_attn(out.float().cpu().numpy(), ref, "decode attention, 300 sequences")
    assert_lse_close(lse.cpu().numpy(), rlse, "decode lse, 300 sequences")


@pytest.mark.parametrize("Hq,Hkv,k", [(8, 1, 256), (16, 4, 64), (12, 4, 100)])
def test_prefill_attention_matches_oracle(Hq, Hkv, k):
    B, L, d, D = 2, 300, 64, 128
    seed = 4000 + Hq + k
    qi = _ints(seed, 1, (B, L, d))
    ki = _ints(seed, 2, (B, L, d))
    q = _normals(seed, 3, (B, L, Hq, D))
    K = _normals(seed, 4, (B, L, Hkv, D))
    V = _normals(seed, 5, (B, L, Hkv, D))
    idx, cnt = sa.sa_index_score_topk(to_dev(qi), to_dev(ki), k)
    out, lse = sa.sa_sparse_attn_prefill(to_dev(q), to_dev(K), to_dev(V), idx, cnt, with_lse=True)
    ridx, rcnt = oracle.index_topk(qi, ki, L, 0, k)
    ref, rlse = oracle.sparse_attention(q, K, V, ridx, rcnt)
    torch.cuda.synchronize()
    assert_close_attn(out.float().cpu().numpy(), ref, "prefill attention")
    assert_lse_close(lse.cpu().numpy(), rlse, "prefill lse")


def test_prefill_attention_with_k_at_least_context_is_dense_causal():
    """k >= L selects every causal key: the output is dense causal attention
    (checked against torch's SDPA on the CPU in fp64)."""
    B, L, Hq, Hkv, D, d = 1, 200, 8, 2, 128, 64
    qi = _ints(55, 1, (B, L, d))
    ki = _ints(55, 2, (B, L, d))
    q = _normals(55, 3, (B, L, Hq, D))
    K = _normals(55, 4, (B, L, Hkv, D))
    V = _normals(55, 5, (B, L, Hkv, D))
    idx, cnt = sa.sa_index_score_topk(to_dev(qi), to_dev(ki), 256)
    out = sa.sa_sparse_attn_prefill(to_dev(q), to_dev(K), to_dev(V), idx, cnt)
    f = lambda x: torch.from_numpy(oracle.bf16_bits_to_f64(x))
    G = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(
        f(q)[0].permute(1, 0, 2), f(K)[0].repeat_interleave(G, 1).permute(1, 0, 2),
        f(V)[0].repeat_interleave(G, 1).permute(1, 0, 2), is_causal=True).permute(1, 0, 2)
    torch.cuda.synchronize()
    assert_close_attn(out[0].float().cpu().numpy(), ref.numpy(), "dense-equivalent prefill")


def test_attention_constant_values_and_clamped_indices():
    """V rows all equal to one row -> output equals that row for any weights;
    out-of-range indices inside count read a clamped row, never fault."""
    B, Hq, Hkv, D, Tk_max, k = 1, 4, 1, 128, 64, 16
    q = _normals(9, 1, (B, Hq, D))
    K = _normals(9, 2, (B, Tk_max, Hkv, D))
    row = _normals(9, 3, (1, 1, 1, D))
    V = np.broadcast_to(row, (B, Tk_max, Hkv, D)).copy()
    idx = np.arange(k, dtype=np.int32)[None] * 4
    idx[0, 3] = 10 ** 6
    idx[0, 4] = -5
    out = sa.sa_sparse_attn_decode(to_dev(q), to_dev(K), to_dev(V), i32(idx), i32([k]))
    torch.cuda.synchronize()
    expect = np.broadcast_to(oracle.bf16_bits_to_f64(row[0, 0, 0]), (Hq, D))
    assert_close_attn(out[0].float().cpu().numpy(), expect, "constant V")


# ---------------------------------------------------------------------- gist

@pytest.mark.parametrize("n_chunks,k_chunks,chunk_len,partial", [
    (500, 64, 16, [1, 7, 16]),
    (40, 64, 16, [0, 3, 16]),          # fewer chunks than k
    (20000, 64, 16, [16, 5, 1]),       # candidate mode
    (3000, 100, 4, [2, 0, 4]),
])
def test_gist_route_unfold_matches_oracle(n_chunks, k_chunks, chunk_len, partial):
    B, d = len(partial), 128
    qr = _ints(5000 + n_chunks, 1, (B, d))
    gk = _ints(5000 + n_chunks, 2, (B, n_chunks, d))
    rows, cnt, chunks = sa.sa_gist_route_unfold(to_dev(qr), to_dev(gk), chunk_len, k_chunks,
                                                i32(partial), with_chunks=True)
    torch.cuda.synchronize()
    rows, cnt, chunks = rows.cpu().numpy(), cnt.cpu().numpy(), chunks.cpu().numpy()
    stride = k_chunks * (chunk_len + 1) + chunk_len
    for b in range(B):
        rr, rc = oracle.gist_route_unfold(qr[b], gk[b], chunk_len, k_chunks, partial[b])
        assert cnt[b] == rr.size
        np.testing.assert_array_equal(rows[b, : rr.size], rr)
        assert np.all(rows[b, rr.size:stride] == -1)
        np.testing.assert_array_equal(chunks[b, : rc.size], rc)
        assert np.all(chunks[b, rc.size:] == -1)


@pytest.mark.parametrize("n_chunks,M,k_groups,k_chunks,chunk_len,partial,d", [
    (8192, 16, 8, 64, 16, 5, 128), (8192, 16, 8, 128, 16, 16, 128), (1000, 7, 12, 40, 4, 0, 64),
    (40, 8, 10, 20, 16, 3, 128), (300, 32, 2, 100, 8, 8, 64), (5, 8, 3, 4, 16, 2, 128)])
def test_hier_gist_route_unfold_matches_oracle(n_chunks, M, k_groups, k_chunks, chunk_len, partial, d):
    """[SSA] §五 / [GSA] 2.4: coarse meta-gist selection, fine gist selection
    among the kept groups' chunks plus the trailing chunks, unfolding.  Cases:
    the bench's shape, every candidate kept, a ragged trailing group, every
    group kept, fewer candidates than k, and no complete group at all."""
    B = 3
    seed = n_chunks + M
    qr = _ints(seed, 1, (B, d))
    gk = _ints(seed, 2, (B, n_chunks, d))
    mk = _ints(seed, 3, (B, n_chunks // M, d))
    part = i32([partial, 0, chunk_len][:B])
    rows, cnt, chunks, groups = sa.sa_hier_gist_route_unfold(to_dev(qr), to_dev(mk), to_dev(gk), chunk_len, M,
                                                             k_groups, k_chunks, part, with_chunks=True,
                                                             with_groups=True)
    torch.cuda.synchronize()
    rows, cnt, chunks, groups = (x.cpu().numpy() for x in (rows, cnt, chunks, groups))
    for b, p in enumerate([partial, 0, chunk_len][:B]):
        rr, rc, rg = oracle.hier_gist_route_unfold(qr[b], mk[b], gk[b], M, chunk_len, k_groups, k_chunks, p)
        np.testing.assert_array_equal(groups[b, : rg.size], rg)
        assert (groups[b, rg.size:] == -1).all()
        np.testing.assert_array_equal(chunks[b, : rc.size], rc)
        assert (chunks[b, rc.size:] == -1).all()
        assert cnt[b] == rr.size
        np.testing.assert_array_equal(rows[b, : rr.size], rr)
        assert (rows[b, rr.size:] == -1).all()


def test_hier_gist_ties_and_limits():
    B, n_chunks, M, d = 2, 4096, 16, 64
    qr = np.zeros((B, d), np.uint16)                 # every score 0: lowest groups and chunks win
    gk = _ints(5, 2, (B, n_chunks, d))
    mk = _ints(5, 3, (B, n_chunks // M, d))
    rows, cnt, chunks, groups = sa.sa_hier_gist_route_unfold(to_dev(qr), to_dev(mk), to_dev(gk), 16, M, 4, 10,
                                                             None, with_chunks=True, with_groups=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(groups.cpu().numpy(), np.tile(np.arange(4), (B, 1)))
    np.testing.assert_array_equal(chunks.cpu().numpy(), np.tile(np.arange(10), (B, 1)))
    assert (cnt.cpu().numpy() == 10 * 17).all()
    fake = ctypes.c_void_p(0x100000)
    L = sa.lib()
    # too many meta keys / candidates for one CTA's shared memory: refused on the host
    assert L.sa_hier_gist_route_unfold(fake, fake, fake, 1, 8193 * 2, 16, 1, 64, 4, 4, None, fake, fake, None, None,
                                       None) == sa.SA_ERR_UNSUPPORTED
    assert L.sa_hier_gist_route_unfold(fake, fake, fake, 1, 100000, 16, 16, 64, 600, 4, None, fake, fake, None,
                                       None, None) == sa.SA_ERR_UNSUPPORTED


def test_gist_equal_scores_take_first_chunks():
    B, n_chunks, d = 2, 300, 64
    qr = np.zeros((B, d), np.uint16)
    gk = _ints(6, 1, (B, n_chunks, d))
    rows, cnt = sa.sa_gist_route_unfold(to_dev(qr), to_dev(gk), 16, 64, i32([3, 0]))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(rows.cpu().numpy()[0, : 64 * 17], np.arange(64 * 17))
    assert list(cnt.cpu().numpy()) == [64 * 17 + 3, 64 * 17]


# --------------------------------------------------------------- index cache

def test_index_cache_layers_share_one_index():
    """[IC] §二/§六 and [LC] "DSA 与 IndexShare": the group's full layer runs
    the indexer once; each layer of the group attends over exactly that index."""
    B, T, d, k, Hq, Hkv, D, n_layers = 2, 5000, 128, 512, 16, 4, 128, 4
    q_idx = _ints(7, 1, (B, d))
    k_idx = _ints(7, 2, (B, T, d))
    cache = sa.IndexCache(n_layers, B, 1, k, share_every=4, device=dev())
    cache.begin_step()
    with pytest.raises(sa.SAError):
        cache.get(2)
    cache.update(0, to_dev(q_idx), to_dev(k_idx), Tk=T, q_pos0=T - 1)
    ridx, rcnt = oracle.index_topk(q_idx[:, None, :], k_idx, T, T - 1, k)
    versions = set()
    for layer in range(n_layers):
        idx, cnt, ver = cache.get_tensors(layer)
        versions.add(ver)
        q = _normals(70 + layer, 1, (B, Hq, D))
        K = _normals(70 + layer, 2, (B, T, Hkv, D))
        V = _normals(70 + layer, 3, (B, T, Hkv, D))
        out = sa.sa_sparse_attn_decode(to_dev(q), to_dev(K), to_dev(V), idx.view(B, k), cnt.view(B))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
        ref, _ = oracle.sparse_attention_decode(q, [K[b, ridx[b, 0]] for b in range(B)],
                                                [V[b, ridx[b, 0]] for b in range(B)])
        assert_close_attn(out.float().cpu().numpy(), ref, f"layer {layer}")
    assert len(versions) == 1
    cache.close()


def test_index_cache_non_uniform_pattern_fssfsf():
    """[IC] §三: the full/shared pattern need not be uniform (a searched
    pattern keeps some indexers and drops others).  Pattern "FSSFSF" over 6
    layers with 3 indexers (layers 0, 3, 5, each with its own indexer query
    and keys): every layer attends over exactly its owner's index, and each
    owner's index matches the oracle."""
    B, T, d, k, Hq, Hkv, D = 2, 4000, 64, 256, 8, 2, 128
    pattern = "FSSFSF"
    owners = oracle.layer_owners(len(pattern), pattern)
    cache = sa.IndexCache(len(pattern), B, 1, k, pattern=pattern, device=dev())
    q_idx = {f: _ints(80 + f, 1, (B, d)) for f in set(owners)}
    k_idx = {f: _ints(80 + f, 2, (B, T, d)) for f in set(owners)}
    ref = {f: oracle.index_topk(q_idx[f][:, None, :], k_idx[f], T, T - 1, k) for f in set(owners)}
    cache.begin_step()
    versions = {}
    for layer, c in enumerate(pattern):
        assert cache.is_full(layer) == (1 if c == "F" else 0)
        assert cache.owner(layer) == owners[layer]
        if c == "F":
            cache.update(layer, to_dev(q_idx[layer]), to_dev(k_idx[layer]), Tk=T, q_pos0=T - 1)
        idx, cnt, ver = cache.get_tensors(layer)
        versions.setdefault(owners[layer], set()).add(ver)
        q = _normals(90 + layer, 1, (B, Hq, D))
        K = _normals(90 + layer, 2, (B, T, Hkv, D))
        V = _normals(90 + layer, 3, (B, T, Hkv, D))
        out = sa.sa_sparse_attn_decode(to_dev(q), to_dev(K), to_dev(V), idx.view(B, k), cnt.view(B))
        torch.cuda.synchronize()
        ridx, rcnt = ref[owners[layer]]
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
        np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt)
        want, _ = oracle.sparse_attention_decode(q, [K[b, ridx[b, 0, : rcnt[b, 0]]] for b in range(B)],
                                                 [V[b, ridx[b, 0, : rcnt[b, 0]]] for b in range(B)])
        assert_close_attn(out.float().cpu().numpy(), want, f"pattern {pattern} layer {layer}")
    # one version per full layer, a new one at each full layer
    assert all(len(v) == 1 for v in versions.values())
    assert len({next(iter(v)) for v in versions.values()}) == 3
    cache.close()


def test_index_overlap_and_a_searched_pattern_end_to_end():
    """[IC] §一-§三 on synthetic layers: six layers in two blocks whose
    indexer queries differ little inside a block; each layer's own top-k,
    the adjacent-layer overlaps (kernel against the oracle), the greedy
    search keeping two indexers (library against the oracle), then a decode
    step through an index cache with the searched pattern, every layer's
    attention against the oracle."""
    rng = np.random.default_rng(91)
    B, T, d, k, Hq, Hkv, L = 2, 6000, 64, 512, 8, 2, 6
    ki = _ints(92, 2, (B, T, d))
    base = [rng.integers(-4, 5, size=(B, d)) for _ in range(2)]
    qs = []
    for l in range(L):
        q = base[l // 3].copy()
        q[:, rng.choice(d, 3, replace=False)] = rng.integers(-4, 5, size=(B, 3))   # a small per-layer change
        qs.append(ch.f32_to_bf16_bits(q.astype(np.float64)))
    own = [sa.sa_index_score_topk(to_dev(qs[l]), to_dev(ki), k, Tk=T, q_pos0=T - 1) for l in range(L)]
    ref = [oracle.index_topk(qs[l][:, None, :], ki, T, T - 1, k) for l in range(L)]
    ov = np.zeros((L, L))
    for a in range(L):
        for b in range(L):
            got = sa.sa_index_overlap(own[a][0], own[a][1], own[b][0], own[b][1])
            want = oracle.index_overlap(ref[a][0][:, 0], ref[a][1][:, 0], ref[b][0][:, 0], ref[b][1][:, 0])
            torch.cuda.synchronize()
            np.testing.assert_array_equal(got.cpu().numpy(), want)
            ov[a, b] = (want / ref[a][1][:, 0]).mean()
    assert ov[1, 0] > 0.5 and ov[3, 2] < 0.5          # similar inside a block, not across
    pattern = sa.sa_index_pattern_greedy(ov, 2)
    assert pattern == oracle.greedy_pattern(ov, 2)
    owners = oracle.layer_owners(L, pattern)
    cache = sa.IndexCache(L, B, 1, k, pattern=pattern, device=dev())
    cache.begin_step()
    for layer in range(L):
        if cache.is_full(layer) == 1:
            cache.update(layer, to_dev(qs[layer]), to_dev(ki), Tk=T, q_pos0=T - 1)
        idx, cnt, _ = cache.get_tensors(layer)
        q = _normals(93 + layer, 1, (B, Hq, 128))
        K = _normals(93 + layer, 2, (B, T, Hkv, 128))
        V = _normals(93 + layer, 3, (B, T, Hkv, 128))
        out = sa.sa_sparse_attn_decode(to_dev(q), to_dev(K), to_dev(V), idx.view(B, k), cnt.view(B))
        torch.cuda.synchronize()
        ridx, rcnt = ref[owners[layer]]
        np.testing.assert_array_equal(idx.view(B, k).cpu().numpy(), ridx[:, 0])
        want, _ = oracle.sparse_attention_decode(q, [K[b, ridx[b, 0, : rcnt[b, 0]]] for b in range(B)],
                                                 [V[b, ridx[b, 0, : rcnt[b, 0]]] for b in range(B)])
        assert_close_attn(out.float().cpu().numpy(), want, f"pattern {pattern} layer {layer}")
    cache.close()


# ------------------------------------------------------------- device inputs

def test_device_generator_matches_host_generator():
    from gen import device as gd
    t = torch.empty(100003, dtype=torch.bfloat16, device=dev())
    gd.fill_normal(t, 12, 34, start=777)
    np.testing.assert_array_equal(t.view(torch.int16).cpu().numpy().view(np.uint16),
                                  ch.normal_bf16(12, 34, start=777, count=100003))
    gd.fill_int(t, 12, 35, start=5)
    np.testing.assert_array_equal(t.view(torch.int16).cpu().numpy().view(np.uint16),
                                  ch.int_bf16(12, 35, start=5, count=100003))


# ------------------------------------------------------- workspace reuse

def test_one_workspace_serves_calls_of_any_shape():
    """One caller-owned workspace reused by calls whose shapes grow and
    shrink: one-query rows in every selection path (one CTA per row, slices
    over many CTAs, 1/4-million-key rows, more rows than the fixed
    histogram region holds) with prefill calls between them, then decode
    attention calls of varying B*Hkv on one zero-filled workspace."""
    L = sa.lib()
    # (B, rows per sequence, key rows, d, k): one-query rows of every
    # selection path, with prefill calls (short and bounded rows) between
    # them on the same workspace
    cases = [(1, 1, 60000, 64, 100), (2, 1, 40000, 64, 3000), (1, 300, 300, 64, 64),
             (4, 1, 20000, 128, 2048), (1, 1, 300000, 64, 2048), (1, 200, 9000, 64, 512),
             (3, 1, 5000, 128, 7), (2, 1, 270000, 128, 4096), (65, 1, 6000, 64, 100)]
    need = max(L.sa_index_score_topk_workspace(B, Tq, n, d, k) for B, Tq, n, d, k in cases)
    ws = torch.zeros(need, dtype=torch.uint8, device=dev())
    for i, (B, Tq, n, d, k) in enumerate(cases):
        q = _ints(900 + i, 1, (B, Tq, d))
        kk = _ints(900 + i, 2, (B, n, d))
        idx, cnt = sa.sa_index_score_topk(to_dev(q), to_dev(kk), k, ws=ws)
        ridx, rcnt = oracle.index_topk(q, kk, n, n - Tq, k)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(cnt.cpu().numpy(), rcnt, err_msg=str((B, Tq, n, d, k)))
        np.testing.assert_array_equal(idx.cpu().numpy(), ridx, err_msg=str((B, Tq, n, d, k)))
    acases = [(4, 8, 32, 2048), (1, 4, 28, 2048), (8, 8, 32, 512), (2, 2, 8, 100)]
    aneed = max(L.sa_sparse_attn_decode_workspace(B, Hq, Hkv, 128, k) for B, Hkv, Hq, k in acases)
    wsa = torch.zeros(aneed, dtype=torch.uint8, device=dev())
    rng = np.random.default_rng(77)
    for i, (B, Hkv, Hq, k) in enumerate(acases):
        Tk_max = 3000
        counts = [k - (b % 3) * 5 for b in range(B)]
        qv = _normals(950 + i, 1, (B, Hq, 128))
        K = _normals(950 + i, 2, (B, Tk_max, Hkv, 128))
        V = _normals(950 + i, 3, (B, Tk_max, Hkv, 128))
        idx = _random_index(rng, B, Tk_max, k, counts)
        out = sa.sa_sparse_attn_decode(to_dev(qv), to_dev(K), to_dev(V), i32(idx), i32(counts), ws=wsa)
        ref, _ = oracle.sparse_attention_decode(qv, [K[b, idx[b, :c]] for b, c in enumerate(counts)],
                                                [V[b, idx[b, :c]] for b, c in enumerate(counts)])
        torch.cuda.synchronize()
        assert_close_attn(out.float().cpu().numpy(), ref, f"attention case {i}")
