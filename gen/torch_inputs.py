"""Device-resident workload inputs (torch tensors filled by gen/device.cu).

Input construction only: allocation, seeded fills and the planted needles.
Layouts and tensor ids follow gen/recipes.py, so gen/recipes.host_rows can
regenerate any row on the host bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

from . import device as gd
from . import recipes as R


def dev_int(shape, seed: int, tid: int, device, start: int = 0):
    t = torch.empty(shape, dtype=torch.bfloat16, device=device)
    return gd.fill_int(t, seed, tid, start)


def dev_normal(shape, seed: int, tid: int, device, start: int = 0):
    t = torch.empty(shape, dtype=torch.bfloat16, device=device)
    return gd.fill_normal(t, seed, tid, start)


def to_e4m3(t):
    """A bfloat16 tensor of values exact in E4M3 -> their E4M3 codes (uint8)."""
    return t.float().to(torch.float8_e4m3fn).view(torch.uint8)


def from_host_bits(bits: np.ndarray, device):
    """Host bf16 bit patterns -> device bfloat16 tensor."""
    a = np.ascontiguousarray(bits).view(np.int16)
    return torch.from_numpy(a).to(device).view(torch.bfloat16)


def decode_inputs(cfg: R.Decode, device, layers=None, groups=None):
    """Caches and all steps' queries of a decode workload.

    k_idx[g]: [B, Tk_max, d]; K[l], V[l]: [B, Tk_max, Hkv, D];
    q_idx[g]: [steps, B, d]; q[l]: [steps, B, Hq, D]."""
    layers = range(cfg.n_layers) if layers is None else layers
    groups = range(cfg.n_groups) if groups is None else groups
    s = cfg.seed
    out = {"k_idx": {}, "q_idx": {}, "K": {}, "V": {}, "q": {}}
    if cfg.H_idx > 1:
        out["w_idx"] = {}
    for g in groups:
        out["k_idx"][g] = dev_int((cfg.B, cfg.Tk_max, cfg.d), s, R.tid(R.KIND_K_IDX, g), device)
        if cfg.H_idx == 1:
            out["q_idx"][g] = dev_int((cfg.steps, cfg.B, cfg.d), s, R.tid(R.KIND_Q_IDX, g), device)
        else:
            out["q_idx"][g] = dev_int((cfg.steps, cfg.B, cfg.H_idx, cfg.d), s, R.tid(R.KIND_Q_IDX, g), device)
            wb = torch.empty((cfg.steps, cfg.B, cfg.H_idx), dtype=torch.bfloat16, device=device)
            gd.fill_int(wb, s, R.tid(R.KIND_W_IDX, g), 0, lo=-3, hi=3)
            out["w_idx"][g] = wb.float()
    if cfg.fp8_idx:
        # the same integer values as E4M3 codes (exact: |v| <= 4)
        for name in ("k_idx", "q_idx"):
            for g in out[name]:
                out[name][g] = to_e4m3(out[name][g])
    for l in layers:
        if cfg.shared_kv and l > 0 and 0 in out["K"]:   # one cache for every layer
            out["K"][l], out["V"][l] = out["K"][0], out["V"][0]
        else:
            lk = 0 if cfg.shared_kv else l
            out["K"][l] = dev_normal((cfg.B, cfg.Tk_max, cfg.Hkv, cfg.D), s, R.tid(R.KIND_K, lk), device)
            out["V"][l] = dev_normal((cfg.B, cfg.Tk_max, cfg.Hkv, cfg.D), s, R.tid(R.KIND_V, lk), device)
        out["q"][l] = dev_normal((cfg.steps, cfg.B, cfg.Hq, cfg.D), s, R.tid(R.KIND_Q, l), device)
    return out


def prefill_inputs(cfg: R.Prefill, device, layers=None):
    """q_idx[g], k_idx[g]: [B, L, d] (needles planted in group 0);
    q[l]: [B, L, Hq, D]; K[l], V[l]: [B, L, Hkv, D]."""
    layers = range(cfg.n_layers) if layers is None else layers
    s = cfg.seed
    out = {"k_idx": {}, "q_idx": {}, "K": {}, "V": {}, "q": {}}
    for g in range(cfg.n_groups):
        qi = dev_int((cfg.B, cfg.L, cfg.d), s, R.tid(R.KIND_Q_IDX, g), device)
        ki = dev_int((cfg.B, cfg.L, cfg.d), s, R.tid(R.KIND_K_IDX, g), device)
        if cfg.n_needles and g == 0:
            pairs = R.needle_pairs(cfg)
            p = torch.tensor([a for a, _ in pairs], device=device)
            t = torch.tensor([b for _, b in pairs], device=device)
            ki[0, p] = (qi[0, t].float() * 8.0).to(torch.bfloat16)  # exact: |8 q| <= 32
        out["q_idx"][g], out["k_idx"][g] = qi, ki
    for l in layers:
        out["q"][l] = dev_normal((cfg.B, cfg.L, cfg.Hq, cfg.D), s, R.tid(R.KIND_Q, l), device)
        out["K"][l] = dev_normal((cfg.B, cfg.L, cfg.Hkv, cfg.D), s, R.tid(R.KIND_K, l), device)
        out["V"][l] = dev_normal((cfg.B, cfg.L, cfg.Hkv, cfg.D), s, R.tid(R.KIND_V, l), device)
    return out


def gist_inputs(cfg: R.Gist, device):
    """gist_key [B, n_chunks, d]; K, V [B, Tk_max, Hkv, D] (interleaved cache);
    q_route [steps, B, d]; q [steps, B, Hq, D]; partial_len[s] = s + 1."""
    s = cfg.seed
    extra = {}
    if cfg.group_size:
        extra["meta_key"] = dev_int((cfg.B, cfg.n_chunks // cfg.group_size, cfg.d), s, R.tid(R.KIND_META_KEY), device)
    return {
        **extra,
        "gist_key": dev_int((cfg.B, cfg.n_chunks, cfg.d), s, R.tid(R.KIND_GIST_KEY), device),
        "K": dev_normal((cfg.B, cfg.Tk_max, cfg.Hkv, cfg.D), s, R.tid(R.KIND_K, 0), device),
        "V": dev_normal((cfg.B, cfg.Tk_max, cfg.Hkv, cfg.D), s, R.tid(R.KIND_V, 0), device),
        "q_route": dev_int((cfg.steps, cfg.B, cfg.d), s, R.tid(R.KIND_Q_ROUTE), device),
        "q": dev_normal((cfg.steps, cfg.B, cfg.Hq, cfg.D), s, R.tid(R.KIND_Q), device),
        "partial_len": [torch.full((cfg.B,), st + 1, dtype=torch.int32, device=device)
                        for st in range(cfg.steps)],
    }
