"""Benchmark of the sparse-attention hot path on B200.

Default workload (the headline): decode, batch 8 sequences of 32768 cached
tokens, 4 layers sharing one routing index (the group's first layer runs the
indexer once per step), indexer d = 128, attention 32 query heads over 8 kv
heads, head_dim 128, top-k 2048.  One step = the indexer top-k for the group
plus the gathered sparse attention of all 4 layers for one new token of every
sequence.  Metric: decode steps/s (whole job; weak scaling over GPUs, each
rank runs its own 8 sequences).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--config decode_32k|decode_1m|gist|prefill_2k|prefill_64k]

Prints one JSON line (rank 0).  Inputs are synthetic and seeded (gen/); they
are generated on the device before timing.  The per-step working set
(320 MiB) and the caches (4.3 GB) are larger than the 126 MB L2.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gen import recipes as R  # noqa: E402


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's inputs: every rank decodes its own sequences."""
    return seed + 1000 * rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of a per-rank value over the process group (a job's time
    is its slowest rank's); the value itself when world == 1."""
    if world <= 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_rank: float, ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time."""
    return world * units_per_rank / (ms / 1e3)

CONFIGS = {
    "decode_32k": R.DECODE_32K,
    "decode_1m": R.DECODE_1M,
    "gist": R.GIST_128K,
    "prefill_2k": R.PREFILL_2K,
    "prefill_64k": R.PREFILL_64K,
}
MIB = 1 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ------------------------------------------------------------ CUDA runtime

class Cudart:
    """The CUDA runtime that torch and libsa.so share, through ctypes: stream
    capture into CUDA graphs (torch's graph wrapper adds RNG-state fills to
    every replay) and plain async copies.  One copy per tensor; no batched
    copy APIs."""

    def __init__(self):
        import ctypes
        import torch  # noqa: F401  (loads the runtime first)
        self.ct = ctypes
        self.rt = ctypes.CDLL("libcudart.so.12")
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        self.rt.cudaStreamBeginCapture.argtypes = [P, I]
        self.rt.cudaStreamEndCapture.argtypes = [P, ctypes.POINTER(P)]
        self.rt.cudaGraphInstantiate.argtypes = [ctypes.POINTER(P), P, ctypes.c_ulonglong]
        self.rt.cudaGraphLaunch.argtypes = [P, P]
        self.rt.cudaGraphExecDestroy.argtypes = [P]
        self.rt.cudaGraphDestroy.argtypes = [P]
        self.rt.cudaMemcpyAsync.argtypes = [P, P, Z, I, P]
        self.rt.cudaMemcpy2DAsync.argtypes = [P, Z, P, Z, Z, Z, I, P]

    def check(self, rc, what):
        if rc != 0:
            raise RuntimeError(f"{what} failed with cudaError {rc}")

    def capture(self, stream, fn):
        """Records fn()'s work on `stream` into an instantiated graph."""
        ct = self.ct
        s = ct.c_void_p(stream.cuda_stream)
        self.check(self.rt.cudaStreamBeginCapture(s, 1), "cudaStreamBeginCapture")
        try:
            fn()
        finally:
            g = ct.c_void_p()
            rc = self.rt.cudaStreamEndCapture(s, ct.byref(g))
        self.check(rc, "cudaStreamEndCapture")
        ex = ct.c_void_p()
        self.check(self.rt.cudaGraphInstantiate(ct.byref(ex), g, 0), "cudaGraphInstantiate")
        self.rt.cudaGraphDestroy(g)
        return ex

    def launch(self, ex, stream):
        self.check(self.rt.cudaGraphLaunch(ex, self.ct.c_void_p(stream.cuda_stream)), "cudaGraphLaunch")

    def h2d(self, dst_ptr, src_ptr, nbytes, stream):
        self.check(self.rt.cudaMemcpyAsync(dst_ptr, src_ptr, nbytes, 1, self.ct.c_void_p(stream.cuda_stream)),
                   "cudaMemcpyAsync")

    def d2h(self, dst_ptr, src_ptr, nbytes, stream):
        self.check(self.rt.cudaMemcpyAsync(dst_ptr, src_ptr, nbytes, 2, self.ct.c_void_p(stream.cuda_stream)),
                   "cudaMemcpyAsync")

    def h2d_2d(self, dst_ptr, dpitch, src_ptr, spitch, width, height, stream):
        self.check(self.rt.cudaMemcpy2DAsync(dst_ptr, dpitch, src_ptr, spitch, width, height, 1,
                                             self.ct.c_void_p(stream.cuda_stream)), "cudaMemcpy2DAsync")


# --------------------------------------------------------------- clock sampler

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons (read-only)."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return None
        # samples under load: within 20% of the busiest clock seen, else all
        sm = [r[0] for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def gpu_uuid(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index or 0)


# ------------------------------------------------------------------ decode

class DecodeBench:
    """Decode step of a group-shared index: full layers run the indexer into
    the shared index buffer, every layer attends over it."""

    def __init__(self, cfg: R.Decode, device, rank: int):
        import torch
        import shared_top_routing_b200 as sa
        from gen import torch_inputs as TI
        self.torch, self.sa, self.cfg, self.dev = torch, sa, cfg, device
        seed_cfg = R.Decode(**{**cfg.__dict__, "seed": rank_seed(cfg.seed, rank)})
        self.inp = TI.decode_inputs(seed_cfg, device)
        c = cfg
        # all layers' K and V caches as slices of one [layers, 2, B, Tk_max, Hkv, D]
        # array, so a step's appended rows of every layer are one strided copy
        self.kv_all = torch.empty((c.n_layers, 2, c.B, c.Tk_max, c.Hkv, c.D), dtype=torch.bfloat16, device=device)
        for l in range(c.n_layers):
            self.kv_all[l, 0].copy_(self.inp["K"][l])
            self.kv_all[l, 1].copy_(self.inp["V"][l])
            self.inp["K"][l], self.inp["V"][l] = self.kv_all[l, 0], self.kv_all[l, 1]
        torch.cuda.empty_cache()
        self.cache = sa.IndexCache(c.n_layers, c.B, 1, c.k, share_every=c.share_every, device=device)
        L = sa.lib()
        self.ws_idx = torch.zeros(L.sa_index_score_topk_workspace(c.B, 1, c.Tk_max, c.d, c.k),
                                  dtype=torch.uint8, device=device)
        self.ws_attn = torch.zeros(max(256, L.sa_sparse_attn_decode_workspace(c.B, c.Hq, c.Hkv, c.D, c.k)),
                                   dtype=torch.uint8, device=device)
        self.out_all = torch.empty((c.n_layers, c.B, c.Hq, c.D), dtype=torch.bfloat16, device=device)
        self.out = [self.out_all[l] for l in range(c.n_layers)]
        self.graphs = {}
        self.events = {}
        # kernels per indexer run: score + finish, plus collect for rows longer
        # than one CTA scans; per attention call: split + merge
        self.launches_per_step = c.n_groups * (3 if c.Tk_max > (1 << 18) else 2) + 2 * c.n_layers

    def step(self, s: int, ev=None):
        c, sa = self.cfg, self.sa
        Tk = c.N + s + 1
        self.cache.begin_step()
        for layer in range(c.n_layers):
            if self.cache.is_full(layer) == 1:
                g = layer // c.share_every
                if ev is not None:
                    ev[("idx", layer, 0)].record()
                self.cache.update(layer, self.inp["q_idx"][g][s], self.inp["k_idx"][g], Tk=Tk,
                                  q_pos0=Tk - 1, ws=self.ws_idx)
                if ev is not None:
                    ev[("idx", layer, 1)].record()
            idx, cnt, _ = self.cache.get_tensors(layer)
            g = layer // c.share_every
            first = layer % c.share_every == 0
            last = layer % c.share_every == c.share_every - 1 or layer == c.n_layers - 1
            if ev is not None and first:
                ev[("attn", g, 0)].record()
            sa.sa_sparse_attn_decode(self.inp["q"][layer][s], self.inp["K"][layer], self.inp["V"][layer],
                                     idx.view(c.B, c.k), cnt.view(c.B), out=self.out[layer],
                                     ws=self.ws_attn)
            if ev is not None and last:
                ev[("attn", g, 1)].record()

    def _new_events(self):
        torch, c = self.torch, self.cfg
        ev = {}
        for layer in range(c.n_layers):
            for e in (0, 1):
                if layer % c.share_every == 0:
                    ev[("idx", layer, e)] = torch.cuda.Event(enable_timing=True, external=True)
                    ev[("attn", layer // c.share_every, e)] = torch.cuda.Event(enable_timing=True, external=True)
        return ev

    def capture(self, steps, rt):
        """Two graphs per step: the timed one holds only the step's kernels
        (event nodes between them would break the programmatic launch chain);
        the other brackets each indexer run, and each group's run of
        consecutive attention calls, with events."""
        torch = self.torch
        self.rt = rt
        self.stream = torch.cuda.Stream(device=self.dev)
        self.graphs_ev = {}
        for s in steps:
            ev = self._new_events()
            with torch.cuda.stream(self.stream):
                self.graphs[s] = rt.capture(self.stream, lambda: self.step(s))
                self.graphs_ev[s] = rt.capture(self.stream, lambda: self.step(s, ev))
            self.events[s] = ev

    def replay(self, s):
        self.rt.launch(self.graphs[s], self.stream)

    def replay_with_events(self, steps):
        for s in steps:
            self.rt.launch(self.graphs_ev[s], self.stream)
        self.torch.cuda.synchronize()

    def kernel_times(self, steps):
        """Average device time (ms) of one indexer run and of one attention
        call, from the events captured inside the graphs.  An attention call
        is timed as its group's run of consecutive calls (chained by
        programmatic launch, as in the timed graphs) divided by the calls in
        the run."""
        c = self.cfg
        idx_t, attn_t = [], []
        for s in set(steps):
            ev = self.events[s]
            for (kind, i, e), a in ev.items():
                if e != 0:
                    continue
                dt = a.elapsed_time(ev[(kind, i, 1)])
                if kind == "idx":
                    idx_t.append(dt)
                else:
                    calls = min(c.share_every, c.n_layers - i * c.share_every)
                    attn_t.append(dt / calls)
        return (statistics.mean(idx_t) if idx_t else None, statistics.mean(attn_t) if attn_t else None)

    def algorithmic_bytes(self):
        """Bytes the method must move per step (gathered K/V of the kept rows,
        the indexer-key stream, queries, indices and outputs)."""
        c = self.cfg
        Tk = c.N + 1
        score = c.n_groups * c.B * Tk * c.d * 2
        attn_one = c.B * c.k * c.Hkv * c.D * 2 * 2 + c.B * c.Hq * c.D * 2 * 2 + c.B * c.k * 4
        return score, attn_one


# DRAM bytes (read + write) per decode attention call, split + merge kernels,
# from an ncu capture of one call.  Must be re-measured (or removed) whenever
# either kernel changes.
MEASURED_TRAFFIC = {"decode_b8_32k_4layers": 67_303_680 + 1_033_984 + 2_554_880}


def run_native(args, cfg, rank, world):
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    if not isinstance(cfg, R.Decode):
        return run_native_other(args, cfg, rank, world, dev, peaks)
    b = DecodeBench(cfg, dev, rank)
    rt = Cudart()
    n_steps = cfg.steps
    torch.cuda.synchronize()
    # eager warm-up (kernel attributes, first-touch), then graph capture
    for i in range(max(1, args.warmup)):
        b.step(i % n_steps)
    torch.cuda.synchronize()
    b.capture(range(n_steps), rt)
    for i in range(args.warmup):
        b.replay(i % n_steps)
    torch.cuda.synchronize()

    sampler = ClockSampler(gpu_uuid(torch, dev)) if rank == 0 else None
    # keep the GPU busy ~1 s before the timed region so clocks are sampled under load
    t_end = time.time() + (args.soak_seconds if sampler else 0.0)
    i = 0
    while time.time() < t_end:
        b.replay(i % n_steps)
        i += 1
        if i % 64 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    order = [(args.warmup + i) % n_steps for i in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    start.record(b.stream)
    for s in order:
        b.replay(s)
    stop.record(b.stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(stop)
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(ms, world, dev)
    # per-call times from the event-bracketed graphs, replayed after the timed region
    b.replay_with_events(sorted(set(order)))
    idx_ms, attn_ms = b.kernel_times(order)
    ms_step = ms / args.steps
    value = job_rate(world, args.steps, ms)

    # end to end: per step H2D of the new token's rows and queries from pinned
    # host memory, the step, D2H of all layers' outputs; through the same API
    e2e = None if args.no_e2e else run_e2e(b, args, dev, world)

    score_bytes, attn_bytes = b.algorithmic_bytes()
    attn_gbs = attn_bytes / (attn_ms * 1e-3) / 1e9 if attn_ms else None
    roof = {"kernel": "attn_decode_split_kernel + attn_decode_merge_kernel (one decode attention call)",
            "bound": "hbm", "achieved": round(attn_gbs, 1) if attn_gbs else None,
            "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(attn_gbs / peaks["hbm_gbs"], 4) if attn_gbs else None,
            "traffic": args.traffic if args.traffic is not None else MEASURED_TRAFFIC.get(cfg.name),
            "peak_source": peaks["source"],
            "algorithmic_bytes_per_launch": attn_bytes}
    idx_gbs = score_bytes / cfg.n_groups / (idx_ms * 1e-3) / 1e9 if idx_ms else None
    step_bytes = score_bytes + cfg.n_layers * attn_bytes
    line = {
        "metric": "decode steps/s", "value": round(value, 2), "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter-hash generator; integer indexer inputs, Irwin-Hall normal K/V/q)",
        "config": {"workload": cfg.name, "batch": cfg.B, "context": cfg.N, "layers": cfg.n_layers,
                   "share_every": cfg.share_every, "d_idx": cfg.d, "q_heads": cfg.Hq,
                   "kv_heads": cfg.Hkv, "head_dim": cfg.D, "top_k": cfg.k,
                   "parallelism": f"replicas{world}",
                   "l2": "no flush; per-step working set 320 MiB and caches 4.3 GB exceed the 126 MB L2",
                   "timing": "CUDA graphs per step, CUDA events on the launch stream, max over ranks; "
                             "per-call kernel times from separate graphs whose events bracket each "
                             "indexer run and each group's run of attention calls (time / calls)"},
        "roofline": roof,
        "kernels": {"index_topk_ms": round(idx_ms, 5) if idx_ms else None,
                    "index_topk_scoring_GBps": round(idx_gbs, 1) if idx_gbs else None,
                    "attn_decode_ms": round(attn_ms, 5) if attn_ms else None,
                    "step_algorithmic_MiB": round(step_bytes / MIB, 2),
                    "step_hbm_frac": round(step_bytes / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
        "e2e": e2e,
        "gpu_launches": b.launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_decode(cfg, budget_s=args.cpu_seconds)
    return line


def run_e2e(b, args, dev, world):
    """Same steps through the public API with host buffers: every step copies
    its queries and the appended token's cache rows from pinned host memory
    and every layer's output back to pinned host memory.  The caches, queries
    and outputs of all layers are slices of one array each, so a step takes
    one copy for all layers' queries, one strided copy for all layers'
    appended K/V rows, one per indexer group for its query and key row, and
    one for all outputs."""
    import torch
    c = b.cfg
    rt = b.rt
    n_steps = c.steps
    st = b.stream
    pin = lambda t: t.contiguous().cpu().pin_memory()
    L, B = c.n_layers, c.B
    host = {}
    for s in range(n_steps):
        pos = c.N + s
        host[s] = {"q_idx": {g: pin(b.inp["q_idx"][g][s]) for g in b.inp["q_idx"]},
                   "k_row": {g: pin(b.inp["k_idx"][g][:, pos]) for g in b.inp["k_idx"]},
                   "q": pin(torch.stack([b.inp["q"][l][s] for l in range(L)])),
                   # rows (layer, K/V, sequence) in the order of b.kv_all
                   "kv_row": pin(b.kv_all[:, :, :, pos].reshape(L * 2 * B, -1))}
    out_h = torch.empty(b.out_all.shape, dtype=b.out_all.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host[0]["q_idx"].values()) + \
        sum(t.numel() * t.element_size() for t in host[0]["k_row"].values()) + \
        host[0]["q"].numel() * 2 + host[0]["kv_row"].numel() * 2
    d2h = out_h.numel() * out_h.element_size()
    qi_dev = {g: torch.empty_like(b.inp["q_idx"][g][0]) for g in b.inp["q_idx"]}
    q_all = torch.empty((L,) + tuple(b.inp["q"][0][0].shape), dtype=torch.bfloat16, device=dev)

    def row_copy(cache, src, pos, rows):
        # rows of one cache position, one per block of `pitch` bytes
        row_bytes = src[0].numel() * src.element_size()
        pitch = cache.shape[-3] * row_bytes if cache.dim() > 3 else cache[0].numel() * cache.element_size()
        rt.h2d_2d(cache.data_ptr() + pos * row_bytes, pitch, src.data_ptr(), row_bytes, row_bytes, rows, st)

    def e2e_step(s):
        h = host[s]
        pos = c.N + s
        for g in h["q_idx"]:
            rt.h2d(qi_dev[g].data_ptr(), h["q_idx"][g].data_ptr(), h["q_idx"][g].numel() * 2, st)
            row_copy(b.inp["k_idx"][g], h["k_row"][g], pos, B)
        rt.h2d(q_all.data_ptr(), h["q"].data_ptr(), h["q"].numel() * 2, st)
        row_copy(b.kv_all, h["kv_row"], pos, L * 2 * B)
        Tk = pos + 1
        b.cache.begin_step()
        for layer in range(c.n_layers):
            if b.cache.is_full(layer) == 1:
                g = layer // c.share_every
                b.cache.update(layer, qi_dev[g], b.inp["k_idx"][g], Tk=Tk, q_pos0=Tk - 1, ws=b.ws_idx)
            idx, cnt, _ = b.cache.get_tensors(layer)
            b.sa.sa_sparse_attn_decode(q_all[layer], b.inp["K"][layer], b.inp["V"][layer],
                                       idx.view(c.B, c.k), cnt.view(c.B), out=b.out[layer], ws=b.ws_attn)
        rt.d2h(out_h.data_ptr(), b.out_all.data_ptr(), out_h.numel() * out_h.element_size(), st)

    with torch.cuda.stream(st):
        for s in range(n_steps):
            e2e_step(s)
    torch.cuda.synchronize()
    graphs = {}
    with torch.cuda.stream(st):
        for s in range(n_steps):
            graphs[s] = rt.capture(st, lambda: e2e_step(s))
    for s in range(min(args.warmup, n_steps)):
        rt.launch(graphs[s], st)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    start.record(st)
    for i in range(args.steps):
        rt.launch(graphs[(args.warmup + i) % n_steps], st)
    stop.record(st)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(stop), world, dev)
    return {"value": round(job_rate(world, args.steps, ms), 2), "unit": "steps/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "how": "per-step CUDA graph: H2D of queries + appended cache rows from pinned memory "
                   "(all layers' queries in one copy, all layers' K/V rows in one strided copy), "
                   "index + attention calls, D2H of every layer's output (one copy)"}


# ------------------------------------------------------------ other configs

def run_native_other(args, cfg, rank, world, dev, peaks):
    """Prefill and gist workloads (reported beside the headline, not as it)."""
    import torch
    import shared_top_routing_b200 as sa
    from gen import torch_inputs as TI
    if isinstance(cfg, R.Gist):
        inp = TI.gist_inputs(dataclasses.replace(cfg, seed=rank_seed(cfg.seed, rank)), dev)
        rows_cap = cfg.rows_cap
        L = sa.lib()
        ws_g = torch.zeros(max(256, L.sa_gist_route_unfold_workspace(cfg.B, cfg.n_chunks, cfg.d, cfg.k_chunks)),
                           dtype=torch.uint8, device=dev)
        ws_a = torch.zeros(max(256, L.sa_sparse_attn_decode_workspace(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, rows_cap)),
                           dtype=torch.uint8, device=dev)
        out = torch.empty((cfg.B, cfg.Hq, cfg.D), dtype=torch.bfloat16, device=dev)

        def step(s):
            rows, cnt = sa.sa_gist_route_unfold(inp["q_route"][s], inp["gist_key"], cfg.chunk_len,
                                                cfg.k_chunks, inp["partial_len"][s], ws=ws_g)
            sa.sa_sparse_attn_decode(inp["q"][s], inp["K"], inp["V"], rows, cnt, out=out, ws=ws_a)
        n_steps, unit, per = cfg.steps, "steps/s", 1
        nbytes = cfg.B * cfg.n_chunks * cfg.d * 2 + cfg.B * rows_cap * cfg.Hkv * cfg.D * 4
        launches = 4   # gist score, finish, attention split, attention merge
    else:
        inp = TI.prefill_inputs(dataclasses.replace(cfg, seed=rank_seed(cfg.seed, rank)), dev)
        cache = sa.IndexCache(cfg.n_layers, cfg.B, cfg.L, cfg.k, share_every=cfg.share_every, device=dev)
        L = sa.lib()
        ws = torch.zeros(max(256, L.sa_index_score_topk_workspace(cfg.B, cfg.L, cfg.L, cfg.d, cfg.k)),
                         dtype=torch.uint8, device=dev)
        outs = [torch.empty_like(inp["q"][l]) for l in range(cfg.n_layers)]
        part_ev = []   # (kind, start, stop) of the last step, when recording

        def ev():
            e = torch.cuda.Event(enable_timing=True)
            e.record()
            return e

        def step(s, record=False):
            cache.begin_step()
            for layer in range(cfg.n_layers):
                if cache.is_full(layer) == 1:
                    g = layer // cfg.share_every
                    a = ev() if record else None
                    cache.update(layer, inp["q_idx"][g], inp["k_idx"][g], ws=ws)
                    if record:
                        part_ev.append(("index", a, ev()))
                idx, cnt, _ = cache.get_tensors(layer)
                a = ev() if record else None
                sa.sa_sparse_attn_prefill(inp["q"][layer], inp["K"][layer], inp["V"][layer], idx, cnt,
                                          out=outs[layer])
                if record:
                    part_ev.append(("attn", a, ev()))
        n_steps, unit, per = 1, "tokens/s", cfg.B * cfg.L
        nbytes = None
        launches = None
    for i in range(max(1, args.warmup)):
        step(i % n_steps)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(args.steps):
        step((args.warmup + i) % n_steps)
    stop.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = max_over_ranks(start.elapsed_time(stop), world, dev)
    value = job_rate(world, args.steps * per, ms)
    line = {"metric": "decode steps/s" if unit == "steps/s" else "prefill tokens/s",
            "value": round(value, 2), "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": cfg.name, "timing": "eager launches, CUDA events"}}
    if nbytes:
        line["kernels"] = {"step_algorithmic_MiB": round(nbytes / MIB, 2),
                           "step_hbm_frac": round(nbytes / (ms / args.steps * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    if launches:
        line["gpu_launches"] = launches * args.steps
    if isinstance(cfg, R.Prefill):
        # one more step with events around the indexer runs and the attention
        # calls (after the timed region)
        step(0, record=True)
        torch.cuda.synchronize()
        idx_ms = sum(a.elapsed_time(b) for kind, a, b in part_ev if kind == "index")
        attn_ms = [a.elapsed_time(b) for kind, a, b in part_ev if kind == "attn"]
        # causal (query, key) pairs per sequence, selected rows per sequence
        pairs = cfg.L * (cfg.L + 1) // 2
        sel = sum(min(cfg.k, t + 1) for t in range(cfg.L))
        idx_flops = cfg.n_groups * cfg.B * pairs * 2 * cfg.d            # one scoring of every causal pair
        attn_bytes = cfg.B * sel * cfg.Hkv * cfg.D * 2 * 2              # gathered K and V rows per layer
        attn_gbs = attn_bytes / (statistics.mean(attn_ms) * 1e-3) / 1e9
        idx_tf = idx_flops / (idx_ms * 1e-3) / 1e12
        line["roofline"] = {"kernel": "attn_prefill_kernel (one layer's attention)", "bound": "hbm",
                            "achieved": round(attn_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": round(attn_gbs / peaks["hbm_gbs"], 4), "traffic": None,
                            "peak_source": peaks["source"], "algorithmic_bytes_per_launch": attn_bytes,
                            "note": "gathered rows are mostly L2 hits (one layer's K/V is about the L2 size)"}
        line["indexer"] = {"ms_per_step": round(idx_ms, 4), "runs_per_step": cfg.n_groups,
                           "algorithmic_gflop_per_step": round(idx_flops / 1e9, 2),
                           "achieved_tflops": round(idx_tf, 1), "peak_tflops": peaks["bf16_tflops"],
                           "frac_of_tensor_peak": round(idx_tf * 1e12 / (peaks["bf16_tflops"] * 1e12), 4),
                           "what": "every causal pair scored once (2 d flops each) over the whole indexer "
                                   "run: scoring passes, bound, selection and emission"}
        line["attention_ms_per_layer"] = round(statistics.mean(attn_ms), 4)
    return line


# ------------------------------------------------------------- CPU oracle

def _decode_oracle_inputs(cfg: R.Decode, step: int, groups=None, layers=None, batches=None):
    """Host inputs the oracle needs for one decode step (generated untimed):
    full indexer caches of the groups, the step's queries, and -- after the
    oracle's own selection -- the selected K/V rows."""
    import oracle
    from gen import counter_hash as ch
    import numpy as np
    groups = range(cfg.n_groups) if groups is None else groups
    layers = range(cfg.n_layers) if layers is None else layers
    batches = range(cfg.B) if batches is None else batches
    Tk = cfg.N + step + 1
    inp = {"k_idx": {}, "q_idx": {}, "q": {}, "rows": {}}
    for g in groups:
        n = cfg.B * cfg.Tk_max * cfg.d
        inp["k_idx"][g] = ch.int_bf16(cfg.seed, R.tid(R.KIND_K_IDX, g), count=n).reshape(cfg.B, cfg.Tk_max, cfg.d)
        inp["q_idx"][g] = R.decode_q_idx_host(cfg, g, step)
    for l in layers:
        inp["q"][l] = R.decode_q_host(cfg, l, step)
    # rows each sequence selects (oracle's own top-k), regenerated per layer
    sel = {}
    for g in groups:
        idx, cnt = oracle.index_topk(inp["q_idx"][g][:, None, :], inp["k_idx"][g], Tk, Tk - 1, cfg.k)
        sel[g] = (idx[:, 0], cnt[:, 0])
    for l in layers:
        g = l // cfg.share_every
        idx, cnt = sel[g]
        Kr, Vr = [], []
        for b in batches:
            rows = idx[b, : cnt[b]]
            Kr.append(R.host_rows(cfg.seed, R.tid(R.KIND_K, l), (cfg.Hkv, cfg.D), rows, True, b, cfg.Tk_max))
            Vr.append(R.host_rows(cfg.seed, R.tid(R.KIND_V, l), (cfg.Hkv, cfg.D), rows, True, b, cfg.Tk_max))
        inp["rows"][l] = (Kr, Vr)
    return inp, Tk


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_decode_step(cfg: R.Decode, inp, Tk):
    """One oracle decode step on prepared host inputs: indexer top-k per
    group (full sort) and fp64 attention of every layer over its group's
    selected rows."""
    import oracle
    for g in inp["k_idx"]:
        oracle.index_topk(inp["q_idx"][g][:, None, :], inp["k_idx"][g], Tk, Tk - 1, cfg.k)
    for l, (Kr, Vr) in inp["rows"].items():
        oracle.sparse_attention_decode(inp["q"][l][: len(Kr)], Kr, Vr)


def cpu_baseline_decode(cfg: R.Decode, budget_s: float = 10.0):
    inp, Tk = _decode_oracle_inputs(cfg, 0)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_decode_step(cfg, inp, Tk)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 100:
            break
    return {"value": round(reps / el, 4), "unit": "steps/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"decode step 0 of {cfg.name} (all {cfg.B} sequences, {cfg.n_groups} indexer "
                      f"group(s), {cfg.n_layers} layers) repeated {reps} times in {el:.1f} s; numpy fp64; "
                      "host input generation and row regeneration untimed"}


def run_reference(args, cfg, rank, world):
    """The oracle as the reference arm: same metric, unit and config."""
    if rank != 0:
        return None
    if not isinstance(cfg, R.Decode):
        return {"impl": "reference", "unavailable": "reference arm implemented for decode workloads only"}
    # each step is one oracle decode step on a bounded sample: sequence 0 only
    batches = [0]
    inp, Tk = _decode_oracle_inputs(cfg, 0, batches=batches)
    sub = {**inp, "q_idx": {g: v[:1] for g, v in inp["q_idx"].items()},
           "k_idx": {g: v[:1] for g, v in inp["k_idx"].items()}}
    for _ in range(args.warmup):
        oracle_decode_step(cfg, sub, Tk)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_decode_step(cfg, sub, Tk)
    el = time.perf_counter() - t0
    # a full step covers all B sequences: scale the one-sequence sample
    value = args.steps / (el * cfg.B)
    cores = _blas_threads()
    return {"impl": "reference", "metric": "decode steps/s", "value": round(value, 5), "unit": "steps/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el * cfg.B / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "batch": cfg.B, "context": cfg.N, "layers": cfg.n_layers,
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 5), "unit": "steps/s", "cores": cores, "kind": "oracle",
                             "sample": f"sequence 0 of {cfg.B} per step (scaled by {cfg.B}); oracle in numpy fp64"},
            "e2e": {"value": round(value, 5), "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", choices=sorted(CONFIGS), default="decode_32k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="decode only: run fewer layers (small profiling cases; not the headline)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--soak-seconds", type=float, default=1.0,
                    help="busy time before the timed region so clocks are sampled under load")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the dominant kernel from an ncu capture")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    cfg = CONFIGS[args.config]
    if args.layers is not None and isinstance(cfg, R.Decode):
        cfg = R.Decode(**{**cfg.__dict__, "n_layers": args.layers,
                          "name": f"{cfg.name}_first{args.layers}layers"})
    if args.impl == "reference":
        line = run_reference(args, cfg, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = run_native(args, cfg, rank, world)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
