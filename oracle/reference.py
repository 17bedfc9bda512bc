"""Oracle definitions (numpy, float64).  Test infrastructure only.

Sources, cited by page title and section:

* [YOIO] "你只索引一次：当AI学会'过目不忘'的遗忘艺术" -- a write-up of
  *You Only Index Once: Cross-Layer Sparse Attention with Shared Routing*.
* [LC]   "长上下文：稀疏注意力 / DSA / IndexShare".
* [SSA]  "斯坦福大学研究团队如何让AI'聪明地遗忘'" (Simplified Sparse Attention).
* [IC]   "清华提出IndexCache技术：让AI大模型处理长文本时速度提升80%".
* [GSA]  "Forget, Then Recall: Learnable Compression and Selective Unfolding
  via Gist Sparse Attention" (an AI-written summary page).

Readings where the pages are silent (each also stated where it is used):

1. The indexer score is one head, a plain dot product q_idx . k_idx, with
   no activation, weight or scale ([LC] "DSA 与 IndexShare" names only a
   light indexer that scores every history token).
2. Causality is inclusive: query t at absolute position q_pos0 + t may
   select every cached position j <= q_pos0 + t (itself included) with
   j < the cache length.
3. Selection keeps min(k, n) candidates with the largest score; equal
   scores are ordered by lower position first.  The result is a set,
   reported in ascending position order, padded with -1.
4. Attention over a selected set is softmax(q.K^T * scale) V with
   scale = 1/sqrt(head_dim) ([YOIO] §1.1), query head h reading kv head
   h // (Hq / Hkv).  An empty set gives a zero output and lse = -inf.
5. The index is per query token and is shared by all heads and all layers
   of a group; a group's first layer is its full layer ([LC] "DSA 与
   IndexShare": every 4 layers share one indexer result; [IC] §二: a shared
   layer reuses the nearest preceding full layer's index).
6. Gist routing scores the routing query against each complete chunk's gist
   key, keeps the top-k chunks (equal scores: lower chunk first) and
   unfolds each chosen chunk's raw tokens plus its own gist, then appends
   the current partial chunk; unchosen gists are left out ([SSA] §三 and §八,
   [GSA] 2.2 and the ablation in 4).
7. The multi-head indexer (an extension beyond the pages' light indexer,
   after DeepSeek's published lightning indexer): H indexer heads, each
   with its own query vector and a per-query weight, score one shared key
   per token as sum_h w_h * ReLU(q_h . k).  Selection is unchanged.
8. Two-level gist routing: meta-gist keys are routing keys only (their
   rows are not attended), one per complete group of chunks; the chunks
   after the last complete group have no meta-gist yet and are always
   second-stage candidates; the unfolded rows are those of single-level
   routing for the chunks chosen in the second stage.
9. The layer-role search of IndexCache needs a trained model and a
   calibration loss; here the loss of sharing is stood in for by the index
   overlap itself (1 - overlap of a layer's own selection with the one it
   would reuse), the greedy removal order being the page's.
10. fp8 indexer inputs (an extension: the pages do not give the indexer's
    number format) are OCP FP8 E4M3 codes: 1 sign bit, 4 exponent bits with
    bias 7, 3 mantissa bits, subnormals at exponent field 0, no infinities,
    S.1111.111 is NaN.  A score is the exact dot product of the decoded
    values, as for bf16 inputs.
"""
from __future__ import annotations

import math

import numpy as np


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64, exactly."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_bits_to_f64(codes) -> np.ndarray:
    """OCP FP8 E4M3 codes (uint8) -> float64, exactly (reading 10):
    exponent field e and mantissa field m give (-1)^s (1 + m/8) 2^(e-7) for
    e > 0, (-1)^s (m/8) 2^-6 for e = 0, and NaN for e = 15, m = 7."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    subnormal = (m / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, subnormal, normal)
    return np.where((e == 15) & ((c & 0x7) == 7), np.nan, v)


def _f64(x) -> np.ndarray:
    """Inputs as float64: uint16 arrays are bf16 bit patterns, uint8 arrays
    E4M3 codes, anything else is taken as values."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return bf16_bits_to_f64(x)
    if x.dtype == np.uint8:
        return e4m3_bits_to_f64(x)
    return x.astype(np.float64)


# ----------------------------------------------------------------- indexer

def n_candidates(t: int, q_pos0: int, kv_len: int) -> int:
    """Number of causal candidates of query t (reading 2): positions
    0 .. min(q_pos0 + t, kv_len - 1)."""
    return max(0, min(q_pos0 + t + 1, kv_len))


def index_scores(q_idx, k_idx) -> np.ndarray:
    """Indexer scores s[t, j] = q_idx[t] . k_idx[j] ([LC] "DSA 与 IndexShare":
    the indexer gives every history token a relevance score; reading 1).

    q_idx: [Tq, d], k_idx: [Tk, d] (bf16 bits or floats).  Returns [Tq, Tk]
    float64.  For integer-valued inputs every entry is an exact integer.
    """
    q = _f64(q_idx)
    k = _f64(k_idx)
    return q @ k.T


def index_scores_multihead(q_idx, w, k_idx) -> np.ndarray:
    """Multi-head weighted indexer scores (reading 7):
    s[t, j] = sum_h w[t, h] * max(0, q_idx[t, h] . k_idx[j]).

    q_idx: [Tq, H, d]; w: [Tq, H] (per query and indexer head); k_idx:
    [Tk, d], one key per cached token shared by every indexer head.  Returns
    [Tq, Tk] float64 (exact integers for integer-valued inputs).
    """
    q = _f64(q_idx)
    k = _f64(k_idx)
    wt = np.asarray(w, dtype=np.float64)
    dots = np.einsum("thd,jd->thj", q, k)
    return np.einsum("th,thj->tj", wt, np.maximum(dots, 0.0))


def topk_select(scores, k: int) -> np.ndarray:
    """Top-k of one query's candidate scores ([LC] "DSA 与 IndexShare": each
    query keeps only its top-k tokens; [YOIO] §1.3 token-level top-k).

    ``scores[j]`` is the score of position j (all positions are candidates).
    Returns the chosen positions in ascending order (reading 3): sort by
    (score descending, position ascending) with a full sort and keep the
    first min(k, n).
    """
    s = np.asarray(scores, dtype=np.float64)
    if np.isnan(s).any():
        raise ValueError("scores hold NaN; selection is undefined for NaN")
    n = s.shape[0]
    order = np.lexsort((np.arange(n), -s))  # primary: -score, secondary: position
    return np.sort(order[: min(k, n)])


def index_topk(q_idx, k_idx, kv_len, q_pos0: int, k: int, w=None):
    """Indexer scoring plus per-query top-k for a batch.

    q_idx: [B, Tq, d] (one indexer head), or [B, Tq, H, d] with weights w
    [B, Tq, H] (the multi-head indexer of index_scores_multihead); k_idx:
    [B, Tk_max, d]; kv_len: int or [B] cache lengths; query t of batch b has
    n_candidates(t, q_pos0, kv_len[b]) candidates.  Returns (idx int32
    [B, Tq, k] padded with -1, count int32 [B, Tq]).
    """
    q_idx = np.asarray(q_idx)
    k_idx = np.asarray(k_idx)
    B, Tq = q_idx.shape[:2]
    lens = np.broadcast_to(np.asarray(kv_len, dtype=np.int64), (B,))
    idx = np.full((B, Tq, k), -1, dtype=np.int32)
    count = np.zeros((B, Tq), dtype=np.int32)
    for b in range(B):
        n_max = n_candidates(Tq - 1, q_pos0, int(lens[b]))
        if n_max == 0:
            continue
        if w is None:
            s = index_scores(q_idx[b], k_idx[b, :n_max])
        else:
            s = index_scores_multihead(q_idx[b], np.asarray(w)[b], k_idx[b, :n_max])
        for t in range(Tq):
            n = n_candidates(t, q_pos0, int(lens[b]))
            sel = topk_select(s[t, :n], k)
            idx[b, t, : sel.size] = sel
            count[b, t] = sel.size
    return idx, count


# --------------------------------------------------------------- attention

def attention_over_rows(q, K_rows, V_rows, scale: float | None = None):
    """Exact attention of one query token over a selected row set.

    q: [Hq, D]; K_rows, V_rows: [n, Hkv, D].  For head h with kv head
    g = h // (Hq/Hkv): z = (K_rows[:, g] @ q[h]) * scale,
    o = softmax(z) @ V_rows[:, g] ([YOIO] §1.1, Attention(Q,K,V) =
    softmax(QK^T/sqrt(d_k))V, applied to the selected keys only as in [YOIO]
    §2.3's selector).  Returns (o [Hq, D] float64, lse [Hq] natural log).
    """
    q = _f64(q)
    Kr = _f64(K_rows)
    Vr = _f64(V_rows)
    Hq, D = q.shape
    n = Kr.shape[0]
    Hkv = Kr.shape[1] if n else max(1, Hq)
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    out = np.zeros((Hq, D), dtype=np.float64)
    lse = np.full((Hq,), -np.inf, dtype=np.float64)
    if n == 0:
        return out, lse
    G = Hq // Hkv
    for h in range(Hq):
        g = h // G
        z = (Kr[:, g, :] @ q[h]) * scale
        m = z.max()
        p = np.exp(z - m)
        l = p.sum()
        out[h] = (p @ Vr[:, g, :]) / l
        lse[h] = m + math.log(l)
    return out, lse


def sparse_attention(q, K, V, idx, count, scale: float | None = None):
    """Prefill sparse attention: every query token t attends to its selected
    rows idx[b, t, :count[b, t]] of the layer's own K/V cache.

    q: [B, T, Hq, D]; K, V: [B, Tk_max, Hkv, D]; idx: [B, T, k]; count: [B, T].
    Returns (out [B, T, Hq, D], lse [B, T, Hq]) float64.
    """
    q = np.asarray(q)
    B, T, Hq, D = q.shape
    out = np.zeros((B, T, Hq, D), dtype=np.float64)
    lse = np.full((B, T, Hq), -np.inf, dtype=np.float64)
    for b in range(B):
        for t in range(T):
            sel = np.asarray(idx[b, t, : int(count[b, t])], dtype=np.int64)
            o, l = attention_over_rows(q[b, t], np.asarray(K)[b, sel], np.asarray(V)[b, sel], scale)
            out[b, t] = o
            lse[b, t] = l
    return out, lse


def sparse_attention_decode(q, K_rows_per_batch, V_rows_per_batch, scale: float | None = None):
    """Decode sparse attention, one query token per sequence.

    q: [B, Hq, D]; K_rows_per_batch[b], V_rows_per_batch[b]: [n_b, Hkv, D],
    the rows selected for sequence b (already gathered by the caller, so
    large caches need not sit in host memory).
    """
    q = np.asarray(q)
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.full((B, Hq), -np.inf, dtype=np.float64)
    for b in range(B):
        out[b], lse[b] = attention_over_rows(q[b], K_rows_per_batch[b], V_rows_per_batch[b], scale)
    return out, lse


# -------------------------------------------------------------------- gist

def gist_route_unfold(q_route, gist_key, chunk_len: int, k_chunks: int, partial_len: int):
    """Gist routing with selective unfolding for one decode query.

    [SSA] §三 / [GSA] 2.2: the query is scored against every chunk's gist
    token by dot product, the top-k chunks are kept, and each kept chunk is
    unfolded into its raw tokens together with its own gist; per [SSA] §八
    and [GSA] 4 (ablation) unkept gists are left out (reading 6).  The
    cache is interleaved: chunk c holds rows (chunk_len+1)*c .. +chunk_len-1
    (raw) and (chunk_len+1)*c + chunk_len (gist); the partial chunk starts
    at (chunk_len+1)*n_chunks and holds partial_len rows.

    Returns (rows int64 ascending, chunks int64 ascending).
    """
    gk = _f64(gist_key)
    n_chunks = gk.shape[0]
    r = gk @ _f64(q_route)
    chunks = topk_select(r, k_chunks)
    stride = chunk_len + 1
    parts = [c * stride + np.arange(stride) for c in chunks]
    parts.append(n_chunks * stride + np.arange(partial_len))
    rows = np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)
    return rows.astype(np.int64), chunks.astype(np.int64)


def hier_gist_route_unfold(q_route, meta_key, gist_key, group_size: int, chunk_len: int, k_groups: int,
                           k_chunks: int, partial_len: int):
    """Two-level (coarse-to-fine) gist routing for one decode query ([SSA]
    §五 H-SSA, [GSA] 2.4 H-GSA; reading 8).

    Every complete group of group_size consecutive chunks has one meta-gist
    routing key.  The query is scored against every meta key and the top
    k_groups groups are kept (equal scores: lower group first).  The
    candidate chunks are those of the kept groups plus the chunks after the
    last complete group (no meta-gist yet); the query is scored against
    their gist keys and the top k_chunks candidates are kept (equal scores:
    lower chunk first).  They are unfolded exactly as gist_route_unfold does.

    meta_key: [n_chunks // group_size, d]; gist_key: [n_chunks, d].
    Returns (rows int64 ascending, chunks int64 ascending, groups int64
    ascending).
    """
    gk = _f64(gist_key)
    mk = _f64(meta_key)
    q = _f64(q_route)
    n_chunks = gk.shape[0]
    n_groups = n_chunks // group_size
    groups = topk_select(mk[:n_groups] @ q, k_groups) if n_groups else np.zeros(0, dtype=np.int64)
    parts = [g * group_size + np.arange(group_size) for g in groups]
    parts.append(np.arange(n_groups * group_size, n_chunks))
    cand = np.concatenate(parts).astype(np.int64)
    chunks = cand[topk_select(gk[cand] @ q, k_chunks)] if cand.size else cand
    stride = chunk_len + 1
    rparts = [c * stride + np.arange(stride) for c in chunks]
    rparts.append(n_chunks * stride + np.arange(partial_len))
    rows = np.concatenate(rparts)
    return rows.astype(np.int64), chunks.astype(np.int64), np.asarray(groups, dtype=np.int64)


# ----------------------------------------------------------------- sharing

def layer_owners(n_layers: int, pattern: str | None = None, share_every: int | None = None):
    """For each layer, the full layer whose index it uses.

    [IC] §二: layers are full (F, run their own indexer) or shared (S, reuse
    the index of the nearest full layer before them); [LC] "DSA 与
    IndexShare": every 4 layers share one indexer result (reading 5: the
    first layer of each group is full).
    """
    if pattern is None:
        if not share_every or share_every < 1:
            raise ValueError("need a pattern or share_every >= 1")
        pattern = "".join("F" if l % share_every == 0 else "S" for l in range(n_layers))
    if len(pattern) != n_layers or set(pattern) - {"F", "S"} or pattern[:1] != "F":
        raise ValueError(f"bad layer pattern {pattern!r}")
    owners = []
    cur = 0
    for l, c in enumerate(pattern):
        if c == "F":
            cur = l
        owners.append(cur)
    return owners


def index_overlap(idx_a, count_a, idx_b, count_b) -> np.ndarray:
    """Per row, how many positions two selections share ([IC] §一: adjacent
    layers' indexers pick 70-100% of the same tokens).  idx_*: [rows, k]
    (entries past count_* ignored).  Returns int64 [rows]."""
    ia = np.asarray(idx_a)
    ib = np.asarray(idx_b)
    ca = np.asarray(count_a).reshape(-1)
    cb = np.asarray(count_b).reshape(-1)
    ia = ia.reshape(ca.size, -1)
    ib = ib.reshape(cb.size, -1)
    return np.array([np.intersect1d(ia[r, : ca[r]], ib[r, : cb[r]]).size for r in range(ca.size)], dtype=np.int64)


def greedy_pattern(overlap, n_full: int) -> str:
    """Training-free layer-role search ([IC] §三, reading 9): start with every
    layer full; repeatedly make shared the one full layer (never layer 0)
    whose removal keeps the largest total retained overlap, until n_full
    full layers remain.  A shared layer reads its nearest preceding full
    layer's index, and retains overlap[l, owner] of its own selection
    (overlap[l, j]: mean fraction of layer l's own top-k that layer j's top-k
    contains).  Equal totals: the lower layer is made shared first."""
    ov = np.asarray(overlap, dtype=np.float64)
    L = ov.shape[0]
    full = [True] * L

    def total(fl):
        owner, t = 0, 0.0
        for l in range(L):
            if fl[l]:
                owner = l
            t += ov[l, owner]
        return t

    while sum(full) > max(1, n_full):
        best, best_t = None, None
        for l in range(1, L):
            if not full[l]:
                continue
            trial = list(full)
            trial[l] = False
            t = total(trial)
            if best_t is None or t > best_t:
                best, best_t = l, t
        full[best] = False
    return "".join("F" if f else "S" for f in full)


# -------------------------------------------------------------- accounting# -------------------------------------------------------------- accounting

def kv_cache_gib(n_layers: int, kv_heads: int, head_dim: int, n_tok: int, bytes_per: int = 2) -> float:
    """KV-cache size in GiB: layers x kv heads x head dim x 2 (K and V) x
    bytes per value x tokens ([LC] "键值显存墙（KV 显存墙）再细看一眼")."""
    return n_layers * kv_heads * head_dim * 2 * bytes_per * n_tok / 1024 ** 3


def pair_counts(n: int, window: int, k: int) -> dict:
    """Scored query-key pairs at context n ([LC] "动手：算清两堵墙"): full
    attention n^2, a sliding window n*window, token top-k n*k."""
    return {"full": n * n, "window": n * window, "topk": n * k}
