"""Workload recipes: shapes, seeds, tensor ids and value distributions.

Each workload names every input tensor by ``(seed, tid)`` of the counter
generator in ``gen.counter_hash`` and by a row-major shape.  Indexer inputs
(``q_idx``, ``k_idx``, gist routing query and keys) are integers uniform in
[-4, 4] stored as bfloat16, so every fp32 dot product of them is exact.
Attention inputs (``q``, ``K``, ``V``) are the Irwin-Hall(12) normal rounded
to bfloat16.

Decode workloads hold ``N + steps`` cache rows; decode step ``s`` sees the
first ``N + s + 1`` of them (the row at ``N + s`` is the token appended by
that step) and its query sits at position ``N + s``.

The gist workload's cache is interleaved: chunk ``c`` occupies rows
``17c .. 17c+15`` (raw tokens) and ``17c+16`` (its gist token); the current
partial chunk follows at ``17 * n_chunks``.  Step ``s`` has a partial chunk of
``s + 1`` tokens.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import counter_hash as ch

# tensor kinds; tid = (kind << 16) | index (layer or group)
KIND_Q_IDX = 1
KIND_K_IDX = 2
KIND_Q = 3
KIND_K = 4
KIND_V = 5
KIND_Q_ROUTE = 6
KIND_GIST_KEY = 7
KIND_NEEDLE_T = 8
KIND_NEEDLE_P = 9
KIND_W_IDX = 10
KIND_META_KEY = 11


def tid(kind: int, index: int = 0) -> int:
    return (kind << 16) | index


@dataclass(frozen=True)
class Prefill:
    name: str
    seed: int
    B: int
    L: int
    d: int
    Hq: int
    Hkv: int
    D: int
    k: int
    n_layers: int
    share_every: int
    n_needles: int = 0

    @property
    def n_groups(self) -> int:
        return (self.n_layers + self.share_every - 1) // self.share_every


@dataclass(frozen=True)
class Decode:
    name: str
    seed: int
    B: int
    N: int
    d: int
    Hq: int
    Hkv: int
    D: int
    k: int
    n_layers: int
    share_every: int
    steps: int
    H_idx: int = 1          # indexer heads (> 1: the multi-head weighted indexer)
    shared_kv: bool = False  # one K/V cache for every layer (YOCO); the rows are gathered once per step
    fp8_idx: bool = False   # indexer queries and keys stored as E4M3 codes (the same integer values)

    @property
    def Tk_max(self) -> int:
        return self.N + self.steps

    @property
    def n_groups(self) -> int:
        return (self.n_layers + self.share_every - 1) // self.share_every


@dataclass(frozen=True)
class Gist:
    name: str
    seed: int
    B: int
    n_chunks: int
    chunk_len: int
    d: int
    k_chunks: int
    Hq: int
    Hkv: int
    D: int
    steps: int
    group_size: int = 0     # > 0: two-level routing, one meta-gist per group of chunks
    k_groups: int = 0

    @property
    def Tk_max(self) -> int:
        return self.n_chunks * (self.chunk_len + 1) + self.chunk_len

    @property
    def rows_cap(self) -> int:
        return self.k_chunks * (self.chunk_len + 1) + self.chunk_len


# The five benchmark workloads.
PREFILL_2K = Prefill("prefill_2k_1layer", seed=1, B=1, L=2048, d=64, Hq=8, Hkv=1, D=128,
                     k=256, n_layers=1, share_every=1)
DECODE_32K = Decode("decode_b8_32k_4layers", seed=2, B=8, N=32768, d=128, Hq=32, Hkv=8,
                    D=128, k=2048, n_layers=4, share_every=4, steps=64)
PREFILL_64K = Prefill("prefill_64k_4layers_needles", seed=3, B=1, L=65536, d=64, Hq=16,
                      Hkv=4, D=128, k=2048, n_layers=4, share_every=4, n_needles=32)
GIST_128K = Gist("gist_decode_b4_128k", seed=4, B=4, n_chunks=8192, chunk_len=16, d=128,
                 k_chunks=64, Hq=32, Hkv=8, D=128, steps=16)
DECODE_1M = Decode("decode_1m_28layers", seed=5, B=1, N=1 << 20, d=64, Hq=28, Hkv=4, D=128,
                   k=2048, n_layers=28, share_every=4, steps=16)

# The batch-8 decode step with a 16-head weighted indexer (sum over heads of
# weight x ReLU(q_h . k), integer weights in [-3, 3]) in place of the one-head
# dot product.
DECODE_32K_MH16 = Decode("decode_b8_32k_4layers_idx16heads", seed=6, B=8, N=32768, d=128, Hq=32, Hkv=8,
                         D=128, k=2048, n_layers=4, share_every=4, steps=64, H_idx=16)

# The batch-8 decode step with one K/V cache shared by all 4 layers (YOCO) and
# one index (CLSA): the selected rows are gathered once per step and every
# layer attends over the compact rows with its own queries.
YOCO_32K = Decode("yoco_decode_b8_32k_4layers_one_cache", seed=7, B=8, N=32768, d=128, Hq=32, Hkv=8, D=128,
                  k=2048, n_layers=4, share_every=4, steps=64, shared_kv=True)

# The gist decode step with two-level routing: one meta-gist per 16 chunks
# (512 meta keys), the top 8 groups' 128 chunks compete for the 64 unfolded.
HGIST_128K = Gist("hgist_decode_b4_128k_meta16", seed=8, B=4, n_chunks=8192, chunk_len=16, d=128, k_chunks=64,
                  Hq=32, Hkv=8, D=128, steps=16, group_size=16, k_groups=8)

# The 16-head decode step with the indexer's queries and keys stored as fp8
# (E4M3): the integer values of the bf16 workload in half the bytes.
DECODE_32K_MH16_FP8 = Decode("decode_b8_32k_4layers_idx16heads_fp8", seed=9, B=8, N=32768, d=128, Hq=32, Hkv=8,
                             D=128, k=2048, n_layers=4, share_every=4, steps=64, H_idx=16, fp8_idx=True)

ALL = [PREFILL_2K, DECODE_32K, PREFILL_64K, GIST_128K, DECODE_1M]


# ---------------------------------------------------------------- host fills

def _ints(seed, t, n, start=0, index=None):
    return ch.int_bf16(seed, t, start=start, count=None if index is not None else n, index=index)


def _normals(seed, t, n, start=0, index=None):
    return ch.normal_bf16(seed, t, start=start, count=None if index is not None else n, index=index)


def host_int_tensor(seed: int, t: int, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return _ints(seed, t, n).reshape(shape)


def host_normal_tensor(seed: int, t: int, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return _normals(seed, t, n).reshape(shape)


def host_rows(seed: int, t: int, row_shape, rows: np.ndarray, normal: bool,
              prefix_index: int = 0, rows_total: int | None = None) -> np.ndarray:
    """Regenerate selected rows of a tensor laid out as [prefix, rows_total, *row_shape].

    ``rows`` are indices along the row axis; ``prefix_index`` selects the
    leading (batch) index.  Returns bf16 bits shaped [len(rows), *row_shape].
    """
    row_elems = int(np.prod(row_shape))
    rows = np.asarray(rows, dtype=np.int64)
    base = (prefix_index * rows_total + rows) * row_elems
    flat = (base[:, None] + np.arange(row_elems, dtype=np.int64)[None, :]).reshape(-1)
    fill = _normals if normal else _ints
    vals = fill(seed, t, None, index=flat.astype(np.uint64))
    return vals.reshape((len(rows),) + tuple(row_shape))


# ------------------------------------------------------------------- needles

def needle_pairs(cfg: Prefill) -> list[tuple[int, int]]:
    """Planted needles ``(p, t)``: the indexer key at row ``p`` is set to
    8 * the indexer query of row ``t`` (``p < t``), so that row ``t`` must
    retrieve position ``p``.  Positions ``p`` are distinct.  Drawn from the
    counter generator; collisions are redrawn with the next counter."""
    pairs: list[tuple[int, int]] = []
    used: set[int] = set()
    c = 0
    lo_t = max(1, cfg.L // 32)
    while len(pairs) < cfg.n_needles:
        ut = int(ch.stream_outputs(cfg.seed, tid(KIND_NEEDLE_T), np.array([c]))[0])
        up = int(ch.stream_outputs(cfg.seed, tid(KIND_NEEDLE_P), np.array([c]))[0])
        c += 1
        t = lo_t + (((ut >> 32) * (cfg.L - lo_t)) >> 32)
        p = ((up >> 32) * t) >> 32
        if p in used or p >= t:
            continue
        used.add(p)
        pairs.append((p, t))
    return pairs


def plant_needles_host(cfg: Prefill, q_idx: np.ndarray, k_idx: np.ndarray) -> None:
    """In place on host bf16-bit arrays shaped [B, L, d] (batch 0 only)."""
    for p, t in needle_pairs(cfg):
        qv = ch.bf16_bits_to_f64(q_idx[0, t])
        k_idx[0, p] = ch.f32_to_bf16_bits(8.0 * qv)


# ------------------------------------------------------- per-config host sets

def prefill_host_inputs(cfg: Prefill, with_attention: bool = True) -> dict:
    """Full host inputs of a prefill workload (small workloads only)."""
    out = {"q_idx": [], "k_idx": [], "q": [], "K": [], "V": []}
    for g in range(cfg.n_groups):
        qi = host_int_tensor(cfg.seed, tid(KIND_Q_IDX, g), (cfg.B, cfg.L, cfg.d))
        ki = host_int_tensor(cfg.seed, tid(KIND_K_IDX, g), (cfg.B, cfg.L, cfg.d))
        if cfg.n_needles and g == 0:
            plant_needles_host(cfg, qi, ki)
        out["q_idx"].append(qi)
        out["k_idx"].append(ki)
    if with_attention:
        for layer in range(cfg.n_layers):
            out["q"].append(host_normal_tensor(cfg.seed, tid(KIND_Q, layer), (cfg.B, cfg.L, cfg.Hq, cfg.D)))
            out["K"].append(host_normal_tensor(cfg.seed, tid(KIND_K, layer), (cfg.B, cfg.L, cfg.Hkv, cfg.D)))
            out["V"].append(host_normal_tensor(cfg.seed, tid(KIND_V, layer), (cfg.B, cfg.L, cfg.Hkv, cfg.D)))
    return out


def decode_q_idx_host(cfg: Decode, g: int, step: int) -> np.ndarray:
    """[B, d], or [B, H_idx, d] for a multi-head indexer."""
    n = cfg.B * cfg.H_idx * cfg.d
    q = _ints(cfg.seed, tid(KIND_Q_IDX, g), n, start=step * n)
    return q.reshape(cfg.B, cfg.d) if cfg.H_idx == 1 else q.reshape(cfg.B, cfg.H_idx, cfg.d)


def decode_w_idx_host(cfg: Decode, g: int, step: int) -> np.ndarray:
    """Multi-head indexer weights [B, H_idx] (float32 integers in [-3, 3])."""
    n = cfg.B * cfg.H_idx
    bits = ch.int_bf16(cfg.seed, tid(KIND_W_IDX, g), start=step * n, count=n, lo=-3, hi=3)
    return ch.bf16_bits_to_f64(bits).astype(np.float32).reshape(cfg.B, cfg.H_idx)


def decode_q_host(cfg: Decode, layer: int, step: int) -> np.ndarray:
    n = cfg.B * cfg.Hq * cfg.D
    return _normals(cfg.seed, tid(KIND_Q, layer), n, start=step * n).reshape(cfg.B, cfg.Hq, cfg.D)


def gist_q_route_host(cfg: Gist, step: int) -> np.ndarray:
    n = cfg.B * cfg.d
    return _ints(cfg.seed, tid(KIND_Q_ROUTE), n, start=step * n).reshape(cfg.B, cfg.d)


def gist_q_host(cfg: Gist, step: int) -> np.ndarray:
    n = cfg.B * cfg.Hq * cfg.D
    return _normals(cfg.seed, tid(KIND_Q), n, start=step * n).reshape(cfg.B, cfg.Hq, cfg.D)
