"""Benchmark of the sparse-attention hot path on B200.

Headline workload (the line's own metric): decode, batch 8 sequences of 32768
cached tokens, 4 layers sharing one routing index (the group's first layer
runs the indexer once per step), indexer d = 128, attention 32 query heads
over 8 kv heads, head_dim 128, top-k 2048.  One step = the indexer top-k for
the group plus the gathered sparse attention of all 4 layers for one new
token of every sequence.  Metric: decode steps/s (whole job; weak scaling
over GPUs, each rank runs its own 8 sequences).

The same JSON line carries, under "workloads", the other workloads of the
path, each timed as CUDA-graph steps with its own roofline, clocks,
CPU-oracle baseline and end-to-end figure:
  prefill_2k_1layer                      prefill tokens/s (L2 flushed between steps)
  prefill_64k_4layers_needles            prefill tokens/s
  gist_decode_b4_128k                    decode steps/s (L2 flushed between steps)
  hgist_decode_b4_128k_meta16            decode steps/s, two-level gist routing
  decode_1m_28layers                     decode steps/s
  decode_b8_32k_4layers_idx16heads       decode steps/s, 16-head weighted indexer
  decode_b8_32k_4layers_idx16heads_fp8   the same with E4M3 indexer queries and keys
  yoco_decode_b8_32k_4layers_one_cache   decode steps/s, one K/V cache gathered once

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--config decode_32k|decode_32k_mh|decode_32k_mh_fp8|yoco_32k|
                              decode_1m|gist|hgist|prefill_2k|prefill_64k]
                    [--no-workloads] [--layers L]

Prints one JSON line (rank 0).  Inputs are synthetic and seeded (gen/); they
are generated on the device before timing.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
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

L2_BYTES = 126 * (1 << 20)
MIB = 1 << 20


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's inputs: every rank runs its own sequences."""
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
    "decode_32k_mh": R.DECODE_32K_MH16,
    "decode_32k_mh_fp8": R.DECODE_32K_MH16_FP8,
    "yoco_32k": R.YOCO_32K,
    "hgist": R.HGIST_128K,
    "decode_1m": R.DECODE_1M,
    "gist": R.GIST_128K,
    "prefill_2k": R.PREFILL_2K,
    "prefill_64k": R.PREFILL_64K,
}
# workloads reported under "workloads" beside the headline, in run order
SUB_WORKLOADS = ("prefill_2k", "prefill_64k", "gist", "hgist", "decode_1m", "decode_32k_mh", "decode_32k_mh_fp8",
                 "yoco_32k")


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


# ------------------------------------------------------------ ncu traffic
#
# DRAM bytes (read + write) per launch of a workload's roofline kernel(s),
# from one `ncu --set full --clock-control none` capture on one B200: "attn"
# one decode attention call (split + merge) or one prefill attention layer,
# "index" one indexer run (scorer + split top-k), "route" one gist routing
# call.  The decode captures ran the workload with one layer (--layers 1:
# the per-call shapes are the workload's); prefill took the first attention
# launch.  NCU_SOURCES holds, per kind, the hash of the code (comments
# stripped) of the source files its kernels are built from, at the capture:
# once that code changes, the bench reports null.

CSRC = os.path.join(ROOT, "shared_top_routing_b200", "csrc")
KIND_SOURCES = {
    "attn": ("attn.cu", "sa_common.cuh", "tc_common.cuh"),
    "index": ("index_topk.cu", "sa_common.cuh", "tc_common.cuh"),
    "route": ("index_topk.cu", "sa_common.cuh", "tc_common.cuh"),
    "index_fp8": ("index_fp8.cu", "index_topk.cu", "sa_common.cuh", "tc_common.cuh"),
}


def _code_only(text: str) -> str:
    """Source text without comments and with whitespace collapsed: edits to
    comments leave the hash, and so the recorded traffic, in place."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def sources_sha16(files=None) -> str:
    """Hash of the code (comments stripped) of the named library source files
    (all of them by default)."""
    if files is None:
        files = [n for n in os.listdir(CSRC) if n.endswith((".cu", ".cuh", ".h"))]
    h = hashlib.sha256()
    for name in sorted(files):
        with open(os.path.join(CSRC, name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


NCU_SOURCES = {"attn": "d3a6d41ccafb13c6", "index": "70bb804a916a11f2", "route": "70bb804a916a11f2",
               "index_fp8": "c02a45fa0098b1c8"}
NCU_TRAFFIC: dict = {
    "decode_b8_32k_4layers": {"attn": 70906624, "index": 69190656},
    "decode_1m_28layers": {"attn": 6152704, "index": 144029952},
    "decode_b8_32k_4layers_idx16heads": {"attn": 70926592, "index": 68858880},
    "yoco_decode_b8_32k_4layers_one_cache": {"attn": 71278080},
    "gist_decode_b4_128k": {"attn": 20434944, "route": 8747264},
    "hgist_decode_b4_128k_meta16": {"attn": 20435200, "route": 727296},
    "prefill_64k_4layers_needles": {"attn": 2805648904},
    "prefill_2k_1layer": {"attn": 7254272},
    "decode_b8_32k_4layers_idx16heads_fp8": {"attn": 70881024, "index_fp8": 34980864},
}


def traffic_for(workload: str, kind: str):
    """DRAM bytes per launch of the workload's roofline kernel(s) of `kind`,
    or None when the library sources changed since the capture."""
    e = NCU_TRAFFIC.get(workload)
    if e is None or kind not in e or NCU_SOURCES[kind] != sources_sha16(KIND_SOURCES[kind]):
        return None
    return e[kind]


# ------------------------------------------------------------ CUDA runtime

class Cudart:
    """The CUDA runtime that torch and libsa.so share, through ctypes: stream
    capture into CUDA graphs (torch's graph wrapper adds RNG-state fills to
    every replay) and plain async copies.  One copy per tensor or strided
    block; no batched copy APIs."""

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
        self.rt.cudaGraphGetNodes.argtypes = [P, ctypes.POINTER(P), ctypes.POINTER(Z)]
        self.rt.cudaGraphNodeGetType.argtypes = [P, ctypes.POINTER(I)]
        self.rt.cudaMemcpyAsync.argtypes = [P, P, Z, I, P]
        self.rt.cudaMemcpy2DAsync.argtypes = [P, Z, P, Z, Z, Z, I, P]
        self.kernel_nodes = {}

    def check(self, rc, what):
        if rc != 0:
            raise RuntimeError(f"{what} failed with cudaError {rc}")

    def _count_kernel_nodes(self, g) -> int:
        ct = self.ct
        n = ct.c_size_t(0)
        self.check(self.rt.cudaGraphGetNodes(g, None, ct.byref(n)), "cudaGraphGetNodes")
        nodes = (ct.c_void_p * max(1, n.value))()
        self.check(self.rt.cudaGraphGetNodes(g, nodes, ct.byref(n)), "cudaGraphGetNodes")
        kernels = 0
        for i in range(n.value):
            t = ct.c_int(-1)
            self.check(self.rt.cudaGraphNodeGetType(ct.c_void_p(nodes[i]), ct.byref(t)), "cudaGraphNodeGetType")
            kernels += 1 if t.value == 0 else 0   # cudaGraphNodeTypeKernel
        return kernels

    def capture(self, stream, fn):
        """Records fn()'s work on `stream` into an instantiated graph; the
        number of kernel nodes it holds is kept in self.kernel_nodes."""
        ct = self.ct
        s = ct.c_void_p(stream.cuda_stream)
        self.check(self.rt.cudaStreamBeginCapture(s, 1), "cudaStreamBeginCapture")
        try:
            fn()
        finally:
            g = ct.c_void_p()
            rc = self.rt.cudaStreamEndCapture(s, ct.byref(g))
        self.check(rc, "cudaStreamEndCapture")
        kernels = self._count_kernel_nodes(g)
        ex = ct.c_void_p()
        self.check(self.rt.cudaGraphInstantiate(ct.byref(ex), g, 0), "cudaGraphInstantiate")
        self.rt.cudaGraphDestroy(g)
        self.kernel_nodes[ex.value] = kernels
        return ex

    def launch(self, ex, stream):
        self.check(self.rt.cudaGraphLaunch(ex, self.ct.c_void_p(stream.cuda_stream)), "cudaGraphLaunch")

    def destroy(self, ex):
        self.kernel_nodes.pop(ex.value, None)
        self.rt.cudaGraphExecDestroy(ex)

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


class Ctx:
    """What every measurement needs: device, peaks, rank, runtime."""

    def __init__(self, args, rank, world, dev, peaks):
        self.args, self.rank, self.world, self.dev, self.peaks = args, rank, world, dev, peaks
        self.rt = Cudart()
        self.flush_buf = None

    def flush_l2(self, stream):
        """Writes 256 MiB (twice the L2) on `stream`."""
        import torch
        if self.flush_buf is None:
            self.flush_buf = torch.empty(256 * MIB, dtype=torch.uint8, device=self.dev)
        with torch.cuda.stream(stream):
            self.flush_buf.fill_(7)

    def barrier(self):
        import torch
        torch.cuda.synchronize()
        if self.world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    def sampler(self):
        import torch
        return ClockSampler(gpu_uuid(torch, self.dev)) if self.rank == 0 else None

    def soak(self, replay, order, stream, seconds: float, flush: bool = False):
        """Replays steps for about `seconds` (untimed), so clock samples taken
        during the timed region that follows see the GPU under load."""
        import torch
        t_end = time.time() + seconds
        i = 0
        while time.time() < t_end:
            if flush:
                self.flush_l2(stream)
            replay(order[i % len(order)])
            i += 1
            if i % 16 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()

    def timed(self, replay, order, stream, flush: bool):
        """Device time (ms, max over ranks) of replay(s) for s in `order`.
        Without flush: one event pair around all steps.  With flush: an event
        pair around each step and an L2 flush between steps, outside the
        pairs; the step times are summed."""
        import torch
        self.barrier()
        if not flush:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for s in order:
                replay(s)
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b)
        else:
            pairs = []
            for s in order:
                self.flush_l2(stream)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                replay(s)
                b.record(stream)
                pairs.append((a, b))
            torch.cuda.synchronize()
            ms = sum(a.elapsed_time(b) for a, b in pairs)
        if self.world > 1:
            torch.distributed.barrier()
        return max_over_ranks(ms, self.world, self.dev)


def _frac(x, peak):
    return round(x / peak, 4) if x is not None and peak else None


def _r(x, nd=4):
    return round(x, nd) if x is not None else None


def _l2_note(step_bytes: int, resident_bytes: int, flush: bool) -> str:
    if flush:
        return (f"L2 flushed between timed steps (256 MiB written outside the timed pairs); per-step "
                f"working set {step_bytes / MIB:.1f} MiB, resident inputs {resident_bytes / 1e9:.2f} GB")
    return (f"no flush; per-step working set {step_bytes / MIB:.1f} MiB and resident inputs "
            f"{resident_bytes / 1e9:.2f} GB exceed the 126 MB L2")


# ------------------------------------------------------------------ decode

class DecodeBench:
    """Decode step of a group-shared index: full layers run the indexer into
    the shared index buffer, every layer attends over it."""

    def __init__(self, cfg: R.Decode, device, rank: int):
        import torch
        import shared_top_routing_b200 as sa
        from gen import device as gd
        from gen import torch_inputs as TI
        self.torch, self.sa, self.cfg, self.dev = torch, sa, cfg, device
        c = cfg
        seed = rank_seed(cfg.seed, rank)
        self.inp = TI.decode_inputs(R.Decode(**{**cfg.__dict__, "seed": seed}), device, layers=[])
        # all layers' K and V caches as slices of one [layers, 2, B, Tk_max, Hkv, D]
        # array, so a step's appended rows of every layer are one strided copy
        # (one cache for every layer when the layers share it)
        n_kv = 1 if c.shared_kv else c.n_layers
        self.kv_all = torch.empty((n_kv, 2, c.B, c.Tk_max, c.Hkv, c.D), dtype=torch.bfloat16, device=device)
        for l in range(n_kv):
            gd.fill_normal(self.kv_all[l, 0], seed, R.tid(R.KIND_K, l))
            gd.fill_normal(self.kv_all[l, 1], seed, R.tid(R.KIND_V, l))
        for l in range(c.n_layers):
            lk = 0 if c.shared_kv else l
            self.inp["K"][l], self.inp["V"][l] = self.kv_all[lk, 0], self.kv_all[lk, 1]
            self.inp["q"][l] = TI.dev_normal((c.steps, c.B, c.Hq, c.D), seed, R.tid(R.KIND_Q, l), device)
        self.gather_once = c.shared_kv
        if c.shared_kv:
            self.k_rows = torch.empty((c.B, c.k, c.Hkv * c.D + 8), dtype=torch.bfloat16, device=device)
            self.v_rows = torch.empty_like(self.k_rows)
        self.cache = sa.IndexCache(c.n_layers, c.B, 1, c.k, share_every=c.share_every, device=device)
        L = sa.lib()
        if c.fp8_idx:
            ws_idx = L.sa_index_score_topk_fp8_workspace(c.B, c.Tk_max, c.H_idx, c.d, c.k)
        elif c.H_idx == 1:
            ws_idx = L.sa_index_score_topk_workspace(c.B, 1, c.Tk_max, c.d, c.k)
        else:
            ws_idx = L.sa_index_score_topk_mh_workspace(c.B, 1, c.Tk_max, c.H_idx, c.d, c.k)
        self.ws_idx = torch.zeros(ws_idx, dtype=torch.uint8, device=device)
        self.ws_attn = torch.zeros(max(256, L.sa_sparse_attn_decode_workspace(c.B, c.Hq, c.Hkv, c.D, c.k)),
                                   dtype=torch.uint8, device=device)
        self.out_all = torch.empty((c.n_layers, c.B, c.Hq, c.D), dtype=torch.bfloat16, device=device)
        self.out = [self.out_all[l] for l in range(c.n_layers)]
        self.graphs = {}
        self.graphs_ev = {}
        self.events = {}

    def step(self, s: int, ev=None, q_all=None, q_idx=None, w_idx=None):
        c, sa = self.cfg, self.sa
        Tk = c.N + s + 1
        self.cache.begin_step()
        for layer in range(c.n_layers):
            g = layer // c.share_every
            if self.cache.is_full(layer) == 1:
                if ev is not None:
                    ev[("idx", layer, 0)].record()
                qi = q_idx[g] if q_idx is not None else self.inp["q_idx"][g][s]
                if c.fp8_idx:
                    # the fp8 indexer writes the group's buffers itself
                    wi = None
                    if c.H_idx > 1:
                        wi = w_idx[g] if w_idx is not None else self.inp["w_idx"][g][s]
                    sa.sa_index_score_topk_fp8(qi, self.inp["k_idx"][g], c.k, w=wi, Tk=Tk, q_pos0=Tk - 1,
                                               idx_out=self.cache.idx_buf.view(c.B, c.k),
                                               count_out=self.cache.count_buf.view(c.B), ws=self.ws_idx)
                    self.cache.mark_written(layer)
                elif c.H_idx == 1:
                    self.cache.update(layer, qi, self.inp["k_idx"][g], Tk=Tk, q_pos0=Tk - 1, ws=self.ws_idx)
                else:
                    # the multi-head indexer writes the group's buffers itself
                    wi = w_idx[g] if w_idx is not None else self.inp["w_idx"][g][s]
                    sa.sa_index_score_topk_mh(qi, wi, self.inp["k_idx"][g], c.k, Tk=Tk, q_pos0=Tk - 1,
                                              idx_out=self.cache.idx_buf, count_out=self.cache.count_buf,
                                              ws=self.ws_idx)
                    self.cache.mark_written(layer)
                if ev is not None:
                    ev[("idx", layer, 1)].record()
            idx, cnt, _ = self.cache.get_tensors(layer)
            first = layer % c.share_every == 0
            last = layer % c.share_every == c.share_every - 1 or layer == c.n_layers - 1
            if ev is not None and first:
                ev[("attn", g, 0)].record()
            q = q_all[layer] if q_all is not None else self.inp["q"][layer][s]
            if self.gather_once:
                # one cache and one index for the group: gather the rows at its
                # first layer, every layer attends over the compact rows
                if first:
                    sa.sa_gather_rows(self.inp["K"][layer], self.inp["V"][layer], idx.view(c.B, c.k),
                                      cnt.view(c.B), k_rows=self.k_rows, v_rows=self.v_rows)
                sa.sa_sparse_attn_decode_rows(q, self.k_rows, self.v_rows, cnt.view(c.B), out=self.out[layer],
                                              ws=self.ws_attn)
            else:
                sa.sa_sparse_attn_decode(q, self.inp["K"][layer], self.inp["V"][layer],
                                         idx.view(c.B, c.k), cnt.view(c.B), out=self.out[layer], ws=self.ws_attn)
            if ev is not None and last:
                ev[("attn", g, 1)].record()

    def _new_events(self):
        torch, c = self.torch, self.cfg
        ev = {}
        for layer in range(0, c.n_layers, c.share_every):
            for e in (0, 1):
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
        for s in steps:
            ev = self._new_events()
            with torch.cuda.stream(self.stream):
                self.graphs[s] = rt.capture(self.stream, lambda: self.step(s))
                self.graphs_ev[s] = rt.capture(self.stream, lambda: self.step(s, ev))
            self.events[s] = ev

    def replay(self, s):
        self.rt.launch(self.graphs[s], self.stream)

    def kernels_per_step(self, s) -> int:
        return self.rt.kernel_nodes[self.graphs[s].value]

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
        """Bytes the method must move: per indexer run (the indexer-key
        stream of every sequence) and per attention call (gathered K/V of the
        kept rows, queries, outputs and indices)."""
        c = self.cfg
        Tk = c.N + 1
        eb = 1 if c.fp8_idx else 2   # bytes per indexer element
        score_run = c.B * Tk * c.d * eb + c.B * c.H_idx * c.d * eb
        attn_one = c.B * c.k * c.Hkv * c.D * 2 * 2 + c.B * c.Hq * c.D * 2 * 2 + c.B * c.k * 4
        return score_run, attn_one

    def close(self):
        for g in list(self.graphs.values()) + list(self.graphs_ev.values()):
            self.rt.destroy(g)
        self.graphs.clear()
        self.graphs_ev.clear()
        self.cache.close()
        self.inp.clear()
        del self.kv_all, self.out_all, self.out, self.ws_idx, self.ws_attn


def decode_e2e(b: DecodeBench, ctx: Ctx, steps: int, warmup: int):
    """Same steps through the public API with host buffers: every step copies
    its queries and the appended token's cache rows from pinned host memory
    and every layer's output back to pinned host memory.  The caches, queries
    and outputs of all layers are slices of one array each, so a step takes
    one copy for all layers' queries, one strided copy for all layers'
    appended K/V rows, one per indexer group for its query and one strided
    copy for its key row, and one for all outputs."""
    import torch
    c = b.cfg
    rt = ctx.rt
    n_steps = c.steps
    st = b.stream
    pin = lambda t: t.contiguous().cpu().pin_memory()
    L, B = c.n_layers, c.B
    nkv = b.kv_all.shape[0]   # caches: one per layer, or one shared by every layer
    host = {}
    for s in range(n_steps):
        pos = c.N + s
        host[s] = {"q_idx": {g: pin(b.inp["q_idx"][g][s]) for g in b.inp["q_idx"]},
                   "w_idx": {g: pin(b.inp["w_idx"][g][s]) for g in b.inp.get("w_idx", {})},
                   "k_row": {g: pin(b.inp["k_idx"][g][:, pos]) for g in b.inp["k_idx"]},
                   "q": pin(torch.stack([b.inp["q"][l][s] for l in range(L)])),
                   # rows (layer, K/V, sequence) in the order of b.kv_all
                   "kv_row": pin(b.kv_all[:, :, :, pos].reshape(nkv * 2 * B, -1))}
    out_h = torch.empty(b.out_all.shape, dtype=b.out_all.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host[0]["q_idx"].values()) + \
        sum(t.numel() * t.element_size() for t in host[0]["w_idx"].values()) + \
        sum(t.numel() * t.element_size() for t in host[0]["k_row"].values()) + \
        host[0]["q"].numel() * 2 + host[0]["kv_row"].numel() * 2
    d2h = out_h.numel() * out_h.element_size()
    qi_dev = {g: torch.empty_like(b.inp["q_idx"][g][0]) for g in b.inp["q_idx"]}
    wi_dev = {g: torch.empty_like(b.inp["w_idx"][g][0]) for g in b.inp.get("w_idx", {})}
    q_all = torch.empty((L,) + tuple(b.inp["q"][0][0].shape), dtype=torch.bfloat16, device=ctx.dev)

    def row_copy(cache, src, pos, rows):
        # one row of `row_bytes` per block of `pitch` bytes (one cache position
        # of every sequence, and of every layer and K/V for b.kv_all)
        row_bytes = src[0].numel() * src.element_size()
        pitch = cache.shape[-3] * row_bytes if cache.dim() > 3 else cache[0].numel() * cache.element_size()
        rt.h2d_2d(cache.data_ptr() + pos * row_bytes, pitch, src.data_ptr(), row_bytes, row_bytes, rows, st)

    def e2e_step(s):
        h = host[s]
        pos = c.N + s
        for g in h["q_idx"]:
            rt.h2d(qi_dev[g].data_ptr(), h["q_idx"][g].data_ptr(),
                   h["q_idx"][g].numel() * h["q_idx"][g].element_size(), st)
            if g in wi_dev:
                rt.h2d(wi_dev[g].data_ptr(), h["w_idx"][g].data_ptr(), h["w_idx"][g].numel() * 4, st)
            row_copy(b.inp["k_idx"][g], h["k_row"][g], pos, B)
        rt.h2d(q_all.data_ptr(), h["q"].data_ptr(), h["q"].numel() * 2, st)
        row_copy(b.kv_all, h["kv_row"], pos, nkv * 2 * B)
        b.step(s, q_all=q_all, q_idx=qi_dev, w_idx=wi_dev if wi_dev else None)
        rt.d2h(out_h.data_ptr(), b.out_all.data_ptr(), d2h, st)

    with torch.cuda.stream(st):
        for s in range(n_steps):
            e2e_step(s)
    torch.cuda.synchronize()
    graphs = {}
    with torch.cuda.stream(st):
        for s in range(n_steps):
            graphs[s] = rt.capture(st, lambda: e2e_step(s))
    for i in range(warmup):
        rt.launch(graphs[i % n_steps], st)
    order = [(warmup + i) % n_steps for i in range(steps)]
    ms = ctx.timed(lambda s: rt.launch(graphs[s], st), order, st, flush=False)
    for g in graphs.values():
        rt.destroy(g)
    return {"value": round(job_rate(ctx.world, steps, ms), 2), "unit": "steps/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "how": "per-step CUDA graph: H2D of queries + appended cache rows from pinned memory "
                   "(all layers' queries in one copy, all layers' K/V rows in one strided copy), "
                   "index + attention calls, D2H of every layer's output (one copy)"}


def measure_decode(ctx: Ctx, cfg: R.Decode, steps: int, warmup: int, headline: bool):
    import torch
    args, peaks = ctx.args, ctx.peaks
    b = DecodeBench(cfg, ctx.dev, ctx.rank)
    rt = ctx.rt
    n_steps = cfg.steps
    torch.cuda.synchronize()
    # eager warm-up (kernel attributes, first touch), then graph capture
    for i in range(max(1, warmup)):
        b.step(i % n_steps)
    torch.cuda.synchronize()
    b.capture(range(n_steps), rt)
    for i in range(warmup):
        b.replay(i % n_steps)
    torch.cuda.synchronize()

    sampler = ctx.sampler()
    order = [(warmup + i) % n_steps for i in range(steps)]
    # keep the GPU busy before the timed region so clocks are sampled under load
    ctx.soak(b.replay, order, b.stream, args.soak_seconds if headline else args.soak_seconds / 2)
    ms = ctx.timed(b.replay, order, b.stream, flush=False)
    clocks = sampler.stop() if sampler else None
    launches = sum(b.kernels_per_step(s) for s in order)
    # per-call times from the event-bracketed graphs, replayed after the timed region
    b.replay_with_events(sorted(set(order)))
    idx_ms, attn_ms = b.kernel_times(order)
    ms_step = ms / steps
    value = job_rate(ctx.world, steps, ms)

    e2e = None if args.no_e2e else decode_e2e(b, ctx, steps, warmup)
    compare = None
    if cfg.shared_kv:
        # the same steps with the rows gathered again by every layer
        b.gather_once = False
        graphs = {}
        with torch.cuda.stream(b.stream):
            for s in range(n_steps):
                graphs[s] = rt.capture(b.stream, lambda: b.step(s))
        for i in range(warmup):
            rt.launch(graphs[i % n_steps], b.stream)
        ms2 = ctx.timed(lambda s: rt.launch(graphs[s], b.stream), order, b.stream, flush=False)
        for g in graphs.values():
            rt.destroy(g)
        b.gather_once = True
        compare = {"gather_per_layer_ms_per_step": round(ms2 / steps, 5),
                   "gather_once_ms_per_step": round(ms_step, 5),
                   "speedup": round(ms2 / ms, 4),
                   "what": "the same steps with every layer gathering its rows from the shared cache "
                           "(sa_sparse_attn_decode) instead of one gather per step and attention over the "
                           "compact rows (sa_gather_rows + sa_sparse_attn_decode_rows)"}

    score_run, attn_bytes = b.algorithmic_bytes()
    step_bytes = cfg.n_groups * score_run + cfg.n_layers * attn_bytes
    if cfg.shared_kv:   # the selected rows cross HBM once per step; each layer reads q/out/indices
        step_bytes = cfg.n_groups * score_run + attn_bytes + (cfg.n_layers - 1) * (attn_bytes - cfg.B * cfg.k *
                                                                                   cfg.Hkv * cfg.D * 4)
    attn_gbs = attn_bytes / (attn_ms * 1e-3) / 1e9 if attn_ms else None
    idx_gbs = score_run / (idx_ms * 1e-3) / 1e9 if idx_ms else None
    attn_total = cfg.n_layers * attn_ms if attn_ms else 0.0
    idx_total = cfg.n_groups * idx_ms if idx_ms else 0.0
    if attn_total >= idx_total:
        roof = {"kernel": "attn_decode_split_kernel + attn_decode_merge_kernel (one decode attention call)",
                "bound": "hbm", "achieved": _r(attn_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": _frac(attn_gbs, peaks["hbm_gbs"]), "algorithmic_bytes_per_launch": attn_bytes,
                "launch_ms": _r(attn_ms, 5)}
    else:
        roof = {"kernel": ("score_fp8_kernel" if cfg.fp8_idx else
                           "score_mh_kernel" if cfg.H_idx > 1 else "score_decode_kernel")
                          + " + split_topk_kernel (one indexer run)",
                "bound": "hbm", "achieved": _r(idx_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": _frac(idx_gbs, peaks["hbm_gbs"]), "algorithmic_bytes_per_launch": score_run,
                "launch_ms": _r(idx_ms, 5)}
    kind = "attn" if attn_total >= idx_total else ("index_fp8" if cfg.fp8_idx else "index")
    roof["traffic"] = args.traffic if (args.traffic is not None and headline) else traffic_for(cfg.name, kind)
    roof["peak_source"] = peaks["source"]
    resident = b.kv_all.numel() * 2 + sum(t.numel() * t.element_size() for t in b.inp["k_idx"].values())
    line = {
        "metric": "decode steps/s", "value": round(value, 2), "unit": "steps/s", "n_gpus": ctx.world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 (indexer e4m3)" if cfg.fp8_idx else "bf16",
        "data": "synthetic (seeded counter-hash generator; integer indexer inputs, Irwin-Hall normal K/V/q)",
        "config": {"workload": cfg.name, "batch": cfg.B, "context": cfg.N, "layers": cfg.n_layers,
                   "share_every": cfg.share_every, "d_idx": cfg.d, "indexer_heads": cfg.H_idx,
                   "indexer_dtype": "e4m3" if cfg.fp8_idx else "bf16", "q_heads": cfg.Hq,
                   "kv_heads": cfg.Hkv, "head_dim": cfg.D, "top_k": cfg.k,
                   "parallelism": f"replicas{ctx.world}",
                   "l2": _l2_note(step_bytes, resident, False),
                   "timing": "CUDA graphs per step, CUDA events on the launch stream, max over ranks; "
                             "per-call kernel times from separate graphs whose events bracket each "
                             "indexer run and each group's run of attention calls (time / calls), "
                             "replayed after the timed region (they carry event overhead the timed "
                             "graphs do not, so per-call times can sum to more than a step)"},
        "roofline": roof,
        "kernels": {"index_topk_ms": _r(idx_ms, 5), "index_topk_runs_per_step": cfg.n_groups,
                    "index_topk_scoring_GBps": _r(idx_gbs, 1),
                    "attn_decode_ms": _r(attn_ms, 5), "attn_decode_calls_per_step": cfg.n_layers,
                    "step_algorithmic_MiB": round(step_bytes / MIB, 2),
                    "step_hbm_frac": round(step_bytes / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if compare is not None:
        line["compare"] = compare
        line["config"]["shared_kv"] = True
        roof["note"] = ("attention over the compact rows, which one gather per step brought in; "
                        "the bytes are those of one gathered attention call")
    if ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_decode(cfg, args.cpu_seconds, b)
    b.close()
    return line


# ----------------------------------------------------------------- prefill

class PrefillBench:
    """One prefill step: every full layer runs the indexer over all causal
    pairs into the shared buffer, every layer attends over it."""

    def __init__(self, cfg: R.Prefill, device, rank: int):
        import torch
        import shared_top_routing_b200 as sa
        from gen import torch_inputs as TI
        self.torch, self.sa, self.cfg, self.dev = torch, sa, cfg, device
        self.inp = TI.prefill_inputs(dataclasses.replace(cfg, seed=rank_seed(cfg.seed, rank)), device)
        self.cache = sa.IndexCache(cfg.n_layers, cfg.B, cfg.L, cfg.k, share_every=cfg.share_every, device=device)
        self.ws = torch.zeros(max(256, sa.lib().sa_index_score_topk_workspace(cfg.B, cfg.L, cfg.L, cfg.d, cfg.k)),
                              dtype=torch.uint8, device=device)
        self.outs = [torch.empty_like(self.inp["q"][l]) for l in range(cfg.n_layers)]
        self.graph = self.graph_ev = None

    def step(self, ev=None):
        c, sa = self.cfg, self.sa
        self.cache.begin_step()
        for layer in range(c.n_layers):
            if self.cache.is_full(layer) == 1:
                g = layer // c.share_every
                if ev is not None:
                    ev[("idx", g, 0)].record()
                self.cache.update(layer, self.inp["q_idx"][g], self.inp["k_idx"][g], ws=self.ws)
                if ev is not None:
                    ev[("idx", g, 1)].record()
            idx, cnt, _ = self.cache.get_tensors(layer)
            if ev is not None:
                ev[("attn", layer, 0)].record()
            sa.sa_sparse_attn_prefill(self.inp["q"][layer], self.inp["K"][layer], self.inp["V"][layer], idx, cnt,
                                      out=self.outs[layer])
            if ev is not None:
                ev[("attn", layer, 1)].record()

    def capture(self, rt):
        torch, c = self.torch, self.cfg
        self.rt = rt
        self.stream = torch.cuda.Stream(device=self.dev)
        self.ev = {}
        for g in range(c.n_groups):
            for e in (0, 1):
                self.ev[("idx", g, e)] = torch.cuda.Event(enable_timing=True, external=True)
        for layer in range(c.n_layers):
            for e in (0, 1):
                self.ev[("attn", layer, e)] = torch.cuda.Event(enable_timing=True, external=True)
        with torch.cuda.stream(self.stream):
            self.graph = rt.capture(self.stream, lambda: self.step())
            self.graph_ev = rt.capture(self.stream, lambda: self.step(self.ev))

    def replay(self, _s=0):
        self.rt.launch(self.graph, self.stream)

    def part_times(self, reps: int, ctx: Ctx, flush: bool):
        """Mean device time (ms) of one indexer run and of one attention
        layer, from `reps` replays of the event-bracketed graph (each after
        an L2 flush when the timed steps had one)."""
        idx_t, attn_t = [], []
        for _ in range(reps):
            if flush:
                ctx.flush_l2(self.stream)
            self.rt.launch(self.graph_ev, self.stream)
            self.torch.cuda.synchronize()
            for (kind, i, e), a in self.ev.items():
                if e == 0:
                    (idx_t if kind == "idx" else attn_t).append(a.elapsed_time(self.ev[(kind, i, 1)]))
        return statistics.mean(idx_t), statistics.mean(attn_t)

    def close(self):
        for g in (self.graph, self.graph_ev):
            if g is not None:
                self.rt.destroy(g)
        self.cache.close()
        self.inp.clear()
        self.outs.clear()
        del self.ws


def prefill_e2e(pb: PrefillBench, ctx: Ctx, steps: int, warmup: int, flush: bool):
    """The prefill through the public API from host buffers: every step
    copies all its inputs (indexer queries and keys of each group, q/K/V of
    each layer) from pinned host memory, one copy per tensor, runs the index
    and attention calls and copies every layer's output back."""
    import torch
    rt, st = ctx.rt, pb.stream
    srcs = [pb.inp["q_idx"][g] for g in pb.inp["q_idx"]] + [pb.inp["k_idx"][g] for g in pb.inp["k_idx"]]
    for l in range(pb.cfg.n_layers):
        srcs += [pb.inp["q"][l], pb.inp["K"][l], pb.inp["V"][l]]
    host_in = [t.cpu().pin_memory() for t in srcs]
    host_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in pb.outs]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    def e2e_step():
        for d, h in zip(srcs, host_in):
            rt.h2d(d.data_ptr(), h.data_ptr(), h.numel() * h.element_size(), st)
        pb.step()
        for h, o in zip(host_out, pb.outs):
            rt.d2h(h.data_ptr(), o.data_ptr(), h.numel() * h.element_size(), st)

    with torch.cuda.stream(st):
        g = rt.capture(st, e2e_step)
    for _ in range(warmup):
        rt.launch(g, st)
    ms = ctx.timed(lambda s: rt.launch(g, st), range(steps), st, flush=flush)
    rt.destroy(g)
    units = pb.cfg.B * pb.cfg.L
    return {"value": round(job_rate(ctx.world, steps * units, ms), 2), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "how": "CUDA graph per step: H2D of every input tensor from pinned memory (one copy each), "
                   "index + attention calls, D2H of every layer's output (one copy each)"}


def measure_prefill(ctx: Ctx, cfg: R.Prefill, steps: int, warmup: int):
    import torch
    args, peaks = ctx.args, ctx.peaks
    pb = PrefillBench(cfg, ctx.dev, ctx.rank)
    flush = cfg.L <= 8192       # a small prefill's inputs would stay in L2 between steps
    for _ in range(max(1, warmup)):
        pb.step()
    torch.cuda.synchronize()
    pb.capture(ctx.rt)
    for _ in range(warmup):
        pb.replay()
    sampler = ctx.sampler()
    ctx.soak(pb.replay, [0], pb.stream, args.soak_seconds / 2, flush)
    ms = ctx.timed(pb.replay, range(steps), pb.stream, flush=flush)
    clocks = sampler.stop() if sampler else None
    idx_ms, attn_ms = pb.part_times(max(1, min(3, steps)), ctx, flush)
    units = cfg.B * cfg.L
    value = job_rate(ctx.world, steps * units, ms)
    # algorithmic work: every causal pair scored once (2 d flops); per layer
    # the selected rows' K and V of each kv head gathered once per token
    pairs = cfg.L * (cfg.L + 1) // 2
    sel = sum(min(cfg.k, t + 1) for t in range(cfg.L))
    idx_flops = cfg.B * pairs * 2 * cfg.d                                   # one indexer run
    gathered = cfg.B * sel * cfg.Hkv * cfg.D * 2 * 2                        # one layer
    attn_flops = cfg.B * sel * cfg.Hq * cfg.D * 2 * 2                       # QK and PV, one layer
    unique = (2 * cfg.B * cfg.L * cfg.Hq * cfg.D * 2 + 2 * cfg.B * cfg.L * cfg.Hkv * cfg.D * 2
              + cfg.B * cfg.L * cfg.k * 4 + cfg.B * cfg.L * 4)              # q, out, K, V, idx, count
    idx_tf = idx_flops / (idx_ms * 1e-3) / 1e12
    gath_gbs = gathered / (attn_ms * 1e-3) / 1e9
    uniq_gbs = unique / (attn_ms * 1e-3) / 1e9
    attn_tf = attn_flops / (attn_ms * 1e-3) / 1e12
    step_bytes = cfg.n_layers * unique
    resident = sum(t.numel() * 2 for d in ("q", "K", "V") for t in pb.inp[d].values())
    line = {
        "metric": "prefill tokens/s", "value": round(value, 2), "unit": "tokens/s", "n_gpus": ctx.world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(ms / steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter-hash generator; integer indexer inputs"
                + (", planted needles" if cfg.n_needles else "") + ", Irwin-Hall normal K/V/q)",
        "config": {"workload": cfg.name, "batch": cfg.B, "seq_len": cfg.L, "layers": cfg.n_layers,
                   "share_every": cfg.share_every, "d_idx": cfg.d, "q_heads": cfg.Hq, "kv_heads": cfg.Hkv,
                   "head_dim": cfg.D, "top_k": cfg.k, "needles": cfg.n_needles,
                   "parallelism": f"replicas{ctx.world}", "l2": _l2_note(step_bytes, resident, flush),
                   "timing": "one CUDA graph per step (indexer run + every layer's attention), CUDA events "
                             "on the launch stream, max over ranks; part times from a second graph "
                             "with events around the indexer run and each attention layer"},
        "roofline": {"kernel": "attn_prefill_kernel (one layer's attention)", "bound": "l2_gather",
                     "achieved": round(gath_gbs, 1), "unit": "GB/s gathered (K/V rows, mostly L2 hits)",
                     "peak": None, "frac": None,
                     "hbm_unique": {"achieved_GBps": round(uniq_gbs, 1), "peak": peaks["hbm_gbs"],
                                    "frac": _frac(uniq_gbs, peaks["hbm_gbs"]),
                                    "bytes_per_launch": unique,
                                    "what": "bytes every layer must read or write once: q, out, the "
                                            "layer's K/V, the index"},
                     "tensor": {"achieved_TFLOPs": round(attn_tf, 2), "peak": peaks["bf16_tflops"],
                                "frac": _frac(attn_tf, peaks["bf16_tflops"]), "flops_per_launch": attn_flops},
                     "algorithmic_bytes_per_launch": gathered, "launch_ms": round(attn_ms, 4),
                     "traffic": traffic_for(cfg.name, "attn"), "peak_source": peaks["source"]},
        "indexer": {"kernel": "score_prefill_tc_kernel passes + prefill_threshold_kernel + finish_kernel "
                              "(one indexer run)",
                    "bound": "tensor", "ms_per_run": round(idx_ms, 4), "runs_per_step": cfg.n_groups,
                    "algorithmic_gflop_per_run": round(idx_flops / 1e9, 3),
                    "achieved": round(idx_tf, 2), "unit": "TFLOP/s", "peak": peaks["bf16_tflops"],
                    "frac": _frac(idx_tf, peaks["bf16_tflops"]),
                    "frac_of_sustained": _frac(idx_tf, peaks["bf16_tflops_sustained"]),
                    "what": "every causal pair scored once (2 d flops each) over the whole indexer run: "
                            "scoring passes, bound, selection and emission"},
        "gpu_launches": steps * ctx.rt.kernel_nodes[pb.graph.value],
        "clocks": clocks,
    }
    line["e2e"] = None if args.no_e2e else prefill_e2e(pb, ctx, steps, warmup, flush)
    if ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prefill(cfg, args.cpu_seconds, pb)
    pb.close()
    return line


# -------------------------------------------------------------------- gist

class GistBench:
    """One gist decode step: route the query over the gists, unfold the kept
    chunks plus the partial chunk, attend over those rows."""

    def __init__(self, cfg: R.Gist, device, rank: int):
        import torch
        import shared_top_routing_b200 as sa
        from gen import torch_inputs as TI
        self.torch, self.sa, self.cfg, self.dev = torch, sa, cfg, device
        self.inp = TI.gist_inputs(dataclasses.replace(cfg, seed=rank_seed(cfg.seed, rank)), device)
        L = sa.lib()
        self.ws_g = torch.zeros(max(256, L.sa_gist_route_unfold_workspace(cfg.B, cfg.n_chunks, cfg.d, cfg.k_chunks)),
                                dtype=torch.uint8, device=device)
        self.ws_a = torch.zeros(max(256, L.sa_sparse_attn_decode_workspace(cfg.B, cfg.Hq, cfg.Hkv, cfg.D,
                                                                           cfg.rows_cap)),
                                dtype=torch.uint8, device=device)
        self.rows = torch.empty((cfg.B, cfg.rows_cap), dtype=torch.int32, device=device)
        self.cnt = torch.empty((cfg.B,), dtype=torch.int32, device=device)
        self.out = torch.empty((cfg.B, cfg.Hq, cfg.D), dtype=torch.bfloat16, device=device)
        self.graphs, self.graphs_ev, self.ev = {}, {}, {}

    def step(self, s, ev=None, q_route=None, q=None, partial=None, single_level=False):
        c, sa = self.cfg, self.sa
        if ev is not None:
            ev[0].record()
        qr = q_route if q_route is not None else self.inp["q_route"][s]
        pl = partial if partial is not None else self.inp["partial_len"][s]
        if c.group_size and not single_level:
            sa.sa_hier_gist_route_unfold(qr, self.inp["meta_key"], self.inp["gist_key"], c.chunk_len, c.group_size,
                                         c.k_groups, c.k_chunks, pl, rows_out=self.rows, count_out=self.cnt)
        else:
            sa.sa_gist_route_unfold(qr, self.inp["gist_key"], c.chunk_len, c.k_chunks, pl, rows_out=self.rows,
                                    count_out=self.cnt, ws=self.ws_g)
        if ev is not None:
            ev[1].record()
        sa.sa_sparse_attn_decode(q if q is not None else self.inp["q"][s], self.inp["K"], self.inp["V"],
                                 self.rows, self.cnt, out=self.out, ws=self.ws_a)
        if ev is not None:
            ev[2].record()

    def capture(self, rt):
        torch = self.torch
        self.rt = rt
        self.stream = torch.cuda.Stream(device=self.dev)
        for s in range(self.cfg.steps):
            ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
            with torch.cuda.stream(self.stream):
                self.graphs[s] = rt.capture(self.stream, lambda: self.step(s))
                self.graphs_ev[s] = rt.capture(self.stream, lambda: self.step(s, ev))
            self.ev[s] = ev

    def replay(self, s):
        self.rt.launch(self.graphs[s], self.stream)

    def part_times(self, ctx: Ctx):
        """Mean device time (ms) of the routing call and of the attention call,
        each step's event graph replayed once after an L2 flush."""
        r, a = [], []
        for s in range(self.cfg.steps):
            ctx.flush_l2(self.stream)
            self.rt.launch(self.graphs_ev[s], self.stream)
            self.torch.cuda.synchronize()
            ev = self.ev[s]
            r.append(ev[0].elapsed_time(ev[1]))
            a.append(ev[1].elapsed_time(ev[2]))
        return statistics.mean(r), statistics.mean(a)

    def close(self):
        for g in list(self.graphs.values()) + list(self.graphs_ev.values()):
            self.rt.destroy(g)
        self.inp.clear()


def gist_e2e(gb: GistBench, ctx: Ctx, steps: int, warmup: int):
    """Gist decode through the public API from host buffers: every step copies
    its routing query, attention query, partial-chunk lengths and the
    appended token's K and V rows (one strided copy each) from pinned host
    memory, and the output back."""
    import torch
    c, rt, st = gb.cfg, ctx.rt, gb.stream
    pin = lambda t: t.contiguous().cpu().pin_memory()
    base = c.n_chunks * (c.chunk_len + 1)
    host = {s: {"q_route": pin(gb.inp["q_route"][s]), "q": pin(gb.inp["q"][s]), "part": pin(gb.inp["partial_len"][s]),
                "k_row": pin(gb.inp["K"][:, base + s]), "v_row": pin(gb.inp["V"][:, base + s])}
            for s in range(c.steps)}
    qr_d = torch.empty_like(gb.inp["q_route"][0])
    q_d = torch.empty_like(gb.inp["q"][0])
    part_d = torch.empty_like(gb.inp["partial_len"][0])
    out_h = torch.empty(gb.out.shape, dtype=gb.out.dtype).pin_memory()
    row_bytes = c.Hkv * c.D * 2
    pitch = c.Tk_max * row_bytes
    h0 = host[0]
    h2d = sum(h0[x].numel() * h0[x].element_size() for x in h0)
    d2h = out_h.numel() * 2

    def e2e_step(s):
        h = host[s]
        rt.h2d(qr_d.data_ptr(), h["q_route"].data_ptr(), h["q_route"].numel() * 2, st)
        rt.h2d(q_d.data_ptr(), h["q"].data_ptr(), h["q"].numel() * 2, st)
        rt.h2d(part_d.data_ptr(), h["part"].data_ptr(), h["part"].numel() * 4, st)
        for cache, src in ((gb.inp["K"], h["k_row"]), (gb.inp["V"], h["v_row"])):
            rt.h2d_2d(cache.data_ptr() + (base + s) * row_bytes, pitch, src.data_ptr(), row_bytes, row_bytes,
                      c.B, st)
        gb.step(s, q_route=qr_d, q=q_d, partial=part_d)
        rt.d2h(out_h.data_ptr(), gb.out.data_ptr(), d2h, st)

    graphs = {}
    with torch.cuda.stream(st):
        for s in range(c.steps):
            graphs[s] = rt.capture(st, lambda: e2e_step(s))
    for i in range(warmup):
        rt.launch(graphs[i % c.steps], st)
    order = [(warmup + i) % c.steps for i in range(steps)]
    ms = ctx.timed(lambda s: rt.launch(graphs[s], st), order, st, flush=True)
    for g in graphs.values():
        rt.destroy(g)
    return {"value": round(job_rate(ctx.world, steps, ms), 2), "unit": "steps/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "how": "per-step CUDA graph: H2D of the routing query, the attention query, the partial "
                   "lengths and the appended K/V rows (strided copies) from pinned memory, routing + "
                   "attention calls, D2H of the output; L2 flushed between steps"}


def measure_gist(ctx: Ctx, cfg: R.Gist, steps: int, warmup: int):
    import torch
    args, peaks = ctx.args, ctx.peaks
    gb = GistBench(cfg, ctx.dev, ctx.rank)
    for i in range(max(1, warmup)):
        gb.step(i % cfg.steps)
    torch.cuda.synchronize()
    gb.capture(ctx.rt)
    for i in range(warmup):
        gb.replay(i % cfg.steps)
    order = [(warmup + i) % cfg.steps for i in range(steps)]
    sampler = ctx.sampler()
    ctx.soak(gb.replay, order, gb.stream, args.soak_seconds / 2, True)
    ms = ctx.timed(gb.replay, order, gb.stream, flush=True)
    clocks = sampler.stop() if sampler else None
    route_ms, attn_ms = gb.part_times(ctx)
    launches = sum(ctx.rt.kernel_nodes[gb.graphs[s].value] for s in order)
    value = job_rate(ctx.world, steps, ms)
    route_bytes = cfg.B * cfg.n_chunks * cfg.d * 2
    compare = None
    if cfg.group_size:
        # bytes the two-level routing reads: every meta key, the kept groups' and trailing chunks' gist keys
        n_groups = cfg.n_chunks // cfg.group_size
        cand = min(cfg.k_groups, n_groups) * cfg.group_size + cfg.n_chunks - n_groups * cfg.group_size
        route_bytes = cfg.B * (n_groups + cand) * cfg.d * 2
        graphs = {}
        with torch.cuda.stream(gb.stream):
            for s in range(cfg.steps):
                graphs[s] = ctx.rt.capture(gb.stream, lambda: gb.step(s, single_level=True))
        ms1 = ctx.timed(lambda s: ctx.rt.launch(graphs[s], gb.stream), order, gb.stream, flush=True)
        for g in graphs.values():
            ctx.rt.destroy(g)
        compare = {"single_level_ms_per_step": round(ms1 / steps, 5), "two_level_ms_per_step": round(ms / steps, 5),
                   "what": "the same steps routed over every gist key (sa_gist_route_unfold) instead of meta "
                           "keys then the kept groups' gist keys (sa_hier_gist_route_unfold); the chosen chunks "
                           "differ, so this compares cost only"}
    mean_rows = cfg.k_chunks * (cfg.chunk_len + 1) + statistics.mean(s % cfg.steps + 1 for s in order)
    attn_bytes = int(cfg.B * mean_rows * cfg.Hkv * cfg.D * 2 * 2 + cfg.B * cfg.Hq * cfg.D * 2 * 2
                     + cfg.B * mean_rows * 4)
    step_bytes = route_bytes + attn_bytes
    route_gbs = route_bytes / (route_ms * 1e-3) / 1e9
    attn_gbs = attn_bytes / (attn_ms * 1e-3) / 1e9
    if attn_ms >= route_ms:
        roof = {"kernel": "attn_decode_split_kernel + attn_decode_merge_kernel (the attention call)",
                "achieved": round(attn_gbs, 1), "algorithmic_bytes_per_launch": attn_bytes,
                "launch_ms": round(attn_ms, 5)}
    else:
        roof = {"kernel": ("hier_gist_kernel (the two-level routing call)" if cfg.group_size else
                           "score_decode_kernel + split_topk_kernel (the routing call)"),
                "achieved": round(route_gbs, 1), "algorithmic_bytes_per_launch": route_bytes,
                "launch_ms": round(route_ms, 5)}
    roof.update({"bound": "hbm", "peak": peaks["hbm_gbs"], "unit": "GB/s",
                 "frac": _frac(roof["achieved"], peaks["hbm_gbs"]),
                 "traffic": traffic_for(cfg.name, "attn" if attn_ms >= route_ms else "route"),
                 "peak_source": peaks["source"]})
    resident = sum(gb.inp[x].numel() * 2 for x in ("K", "V", "gist_key"))
    line = {
        "metric": "decode steps/s", "value": round(value, 2), "unit": "steps/s", "n_gpus": ctx.world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(ms / steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter-hash generator; integer routing query and gist keys, "
                "Irwin-Hall normal K/V/q)",
        "config": {"workload": cfg.name, "batch": cfg.B, "chunks": cfg.n_chunks, "chunk_len": cfg.chunk_len,
                   "raw_tokens": cfg.n_chunks * cfg.chunk_len, "d_route": cfg.d, "top_k_chunks": cfg.k_chunks,
                   "q_heads": cfg.Hq, "kv_heads": cfg.Hkv, "head_dim": cfg.D,
                   "parallelism": f"replicas{ctx.world}", "l2": _l2_note(step_bytes, resident, True),
                   "timing": "CUDA graph per step, an event pair around each step, L2 flushed between "
                             "steps outside the pairs, max over ranks"},
        "roofline": roof,
        "kernels": {"route_ms": round(route_ms, 5), "route_GBps": round(route_gbs, 1),
                    "attn_decode_ms": round(attn_ms, 5), "attn_GBps": round(attn_gbs, 1),
                    "step_algorithmic_MiB": round(step_bytes / MIB, 2),
                    "step_hbm_frac": round(step_bytes / (ms / steps * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if compare is not None:
        line["compare"] = compare
        line["config"].update({"group_size": cfg.group_size, "meta_gists": cfg.n_chunks // cfg.group_size,
                               "top_k_groups": cfg.k_groups})
    line["e2e"] = None if args.no_e2e else gist_e2e(gb, ctx, steps, warmup)
    if ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_gist(cfg, args.cpu_seconds, gb)
    gb.close()
    return line


# ------------------------------------------------------------- CPU oracle
#
# Each baseline times the oracle on a bounded sample of its workload: inputs
# are prepared untimed (generated on the host, or -- inside a native run --
# copied from the device generator's tensors, which are bit-identical to the
# host generator's), the oracle's own selection decides which K/V rows are
# regenerated, and only the oracle's arithmetic is timed.

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def _bits(t):
    """A bf16 device tensor's bit patterns as a host uint16 array."""
    import numpy as np
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _time_loop(fn, budget_s: float, max_reps: int = 1000):
    reps, t0 = 0, time.perf_counter()
    while True:
        fn()
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= max_reps:
            return reps, el


class OracleDecode:
    """One decode step of the oracle on chosen groups, layers and sequences."""

    def __init__(self, cfg: R.Decode, step: int, groups, layers, batches, bench: DecodeBench | None = None):
        import numpy as np
        import oracle
        from gen import counter_hash as ch
        self.cfg = cfg
        self.Tk = Tk = cfg.N + step + 1
        self.k_idx, self.q_idx, self.w_idx, self.q, self.rows = {}, {}, {}, {}, {}
        bl = list(batches)
        for g in groups:
            if bench is not None:
                # bf16 bit patterns, or E4M3 codes (uint8) for an fp8 indexer
                raw = (lambda t: t.contiguous().cpu().numpy()) if cfg.fp8_idx else _bits
                self.k_idx[g] = raw(bench.inp["k_idx"][g][bl])
                self.q_idx[g] = raw(bench.inp["q_idx"][g][step][bl])
                if cfg.H_idx > 1:
                    self.w_idx[g] = bench.inp["w_idx"][g][step][bl].cpu().numpy()
            else:
                n = cfg.B * cfg.Tk_max * cfg.d
                self.k_idx[g] = ch.int_bf16(cfg.seed, R.tid(R.KIND_K_IDX, g), count=n) \
                    .reshape(cfg.B, cfg.Tk_max, cfg.d)[bl]
                self.q_idx[g] = R.decode_q_idx_host(cfg, g, step)[bl]
                if cfg.fp8_idx:
                    to8 = lambda bits: ch.e4m3_codes(ch.bf16_bits_to_f64(bits))
                    self.k_idx[g], self.q_idx[g] = to8(self.k_idx[g]), to8(self.q_idx[g])
                if cfg.H_idx > 1:
                    self.w_idx[g] = R.decode_w_idx_host(cfg, g, step)[bl]
        sel = {g: self._topk(g) for g in groups}
        for l in layers:
            g = l // cfg.share_every
            idx, cnt = sel[g]
            Kr, Vr = [], []
            for i, b in enumerate(bl):
                rows = idx[i, 0, : cnt[i, 0]]
                if bench is not None:
                    import torch
                    r = torch.as_tensor(np.asarray(rows, dtype=np.int64), device=bench.dev)
                    Kr.append(_bits(bench.inp["K"][l][b][r]))
                    Vr.append(_bits(bench.inp["V"][l][b][r]))
                else:
                    lk = 0 if cfg.shared_kv else l
                    Kr.append(R.host_rows(cfg.seed, R.tid(R.KIND_K, lk), (cfg.Hkv, cfg.D), rows, True, b, cfg.Tk_max))
                    Vr.append(R.host_rows(cfg.seed, R.tid(R.KIND_V, lk), (cfg.Hkv, cfg.D), rows, True, b, cfg.Tk_max))
            self.q[l] = _bits(bench.inp["q"][l][step][bl]) if bench is not None else R.decode_q_host(cfg, l, step)[bl]
            self.rows[l] = (Kr, Vr)

    def _topk(self, g):
        import oracle
        w = self.w_idx[g][:, None] if g in self.w_idx else None
        return oracle.index_topk(self.q_idx[g][:, None], self.k_idx[g], self.Tk, self.Tk - 1, self.cfg.k, w=w)

    def run(self):
        import oracle
        for g in self.k_idx:
            self._topk(g)
        for l, (Kr, Vr) in self.rows.items():
            oracle.sparse_attention_decode(self.q[l], Kr, Vr)


def cpu_baseline_decode(cfg: R.Decode, budget_s: float, bench: DecodeBench | None = None):
    """The whole step when the groups are few; otherwise the first group and
    its layers, scaled by the number of groups."""
    if cfg.n_groups <= 1:
        groups, layers, scale = range(cfg.n_groups), range(cfg.n_layers), 1
        what = f"decode step 0 of {cfg.name} (all {cfg.B} sequences, all groups and layers)"
    else:
        groups, layers, scale = [0], range(cfg.share_every), cfg.n_groups
        what = (f"decode step 0 of {cfg.name}: indexer group 0 and its {cfg.share_every} layers, "
                f"scaled by the {cfg.n_groups} groups")
    o = OracleDecode(cfg, 0, groups, layers, range(cfg.B), bench)
    reps, el = _time_loop(o.run, budget_s, 100)
    return {"value": round(reps / (el * scale), 5), "unit": "steps/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{what}, repeated {reps} times in {el:.1f} s; numpy fp64; input preparation and "
                      "row regeneration untimed"}


class OraclePrefill:
    """The oracle on sampled query rows of a prefill: indexer scores and
    top-k of each sampled row against its causal candidates, then each
    layer's attention of that row over its selection."""

    def __init__(self, cfg: R.Prefill, rows, bench: PrefillBench | None = None):
        import numpy as np
        import oracle
        self.cfg, self.rows = cfg, list(rows)
        if bench is not None:
            self.qi = {g: _bits(bench.inp["q_idx"][g][0]) for g in bench.inp["q_idx"]}
            self.ki = {g: _bits(bench.inp["k_idx"][g][0]) for g in bench.inp["k_idx"]}
        else:
            host = R.prefill_host_inputs(cfg, with_attention=False)
            self.qi = {g: host["q_idx"][g][0] for g in range(cfg.n_groups)}
            self.ki = {g: host["k_idx"][g][0] for g in range(cfg.n_groups)}
        self.att = {}
        for g in range(cfg.n_groups):
            s = oracle.index_scores(self.qi[g][self.rows], self.ki[g])
            sels = [oracle.topk_select(s[i, : t + 1], cfg.k) for i, t in enumerate(self.rows)]
            for layer in range(g * cfg.share_every, min(cfg.n_layers, (g + 1) * cfg.share_every)):
                for t, sel in zip(self.rows, sels):
                    if bench is not None:
                        import torch
                        r = torch.as_tensor(np.asarray(sel, dtype=np.int64), device=bench.dev)
                        q = _bits(bench.inp["q"][layer][0, t])
                        Kr = _bits(bench.inp["K"][layer][0][r])
                        Vr = _bits(bench.inp["V"][layer][0][r])
                    else:
                        q = R.host_rows(cfg.seed, R.tid(R.KIND_Q, layer), (cfg.Hq, cfg.D), np.array([t]), True,
                                        0, cfg.L)[0]
                        Kr = R.host_rows(cfg.seed, R.tid(R.KIND_K, layer), (cfg.Hkv, cfg.D), sel, True, 0, cfg.L)
                        Vr = R.host_rows(cfg.seed, R.tid(R.KIND_V, layer), (cfg.Hkv, cfg.D), sel, True, 0, cfg.L)
                    self.att[(layer, t)] = (q, Kr, Vr)

    def run(self):
        import oracle
        for g in self.qi:
            s = oracle.index_scores(self.qi[g][self.rows], self.ki[g])
            for i, t in enumerate(self.rows):
                oracle.topk_select(s[i, : t + 1], self.cfg.k)
        for (q, Kr, Vr) in self.att.values():
            oracle.attention_over_rows(q, Kr, Vr)


def _prefill_sample_rows(cfg: R.Prefill, n: int):
    """n query rows evenly spread over the sequence (their mean cost is the
    mean per-token cost: scoring grows with the row's position)."""
    if n >= cfg.L:
        return list(range(cfg.L))
    return [int((i + 0.5) * cfg.L / n) for i in range(n)]


def cpu_baseline_prefill(cfg: R.Prefill, budget_s: float, bench: PrefillBench | None = None, n_rows: int = 0):
    n_rows = n_rows or (cfg.L if cfg.L <= 2048 else 16)
    rows = _prefill_sample_rows(cfg, n_rows)
    o = OraclePrefill(cfg, rows, bench)
    reps, el = _time_loop(o.run, budget_s, 100)
    return {"value": round(reps * len(rows) * cfg.B / el, 3), "unit": "tokens/s", "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"{len(rows)} of {cfg.L} query rows (evenly spread) of {cfg.name}: indexer scores + "
                      f"top-k of each row and its attention in all {cfg.n_layers} layers, repeated {reps} "
                      f"times in {el:.1f} s; numpy fp64; input preparation and row regeneration untimed"}


class OracleGist:
    """One gist decode step of the oracle for every sequence."""

    def __init__(self, cfg: R.Gist, step: int, bench: GistBench | None = None):
        import numpy as np
        import oracle
        from gen import counter_hash as ch
        self.cfg, self.step = cfg, step
        self.mk = None
        if bench is not None:
            self.gk = _bits(bench.inp["gist_key"])
            self.qr = _bits(bench.inp["q_route"][step])
            self.q = _bits(bench.inp["q"][step])
            if cfg.group_size:
                self.mk = _bits(bench.inp["meta_key"])
        else:
            self.gk = ch.int_bf16(cfg.seed, R.tid(R.KIND_GIST_KEY), count=cfg.B * cfg.n_chunks * cfg.d) \
                .reshape(cfg.B, cfg.n_chunks, cfg.d)
            self.qr = R.gist_q_route_host(cfg, step)
            self.q = R.gist_q_host(cfg, step)
            if cfg.group_size:
                ng = cfg.n_chunks // cfg.group_size
                self.mk = ch.int_bf16(cfg.seed, R.tid(R.KIND_META_KEY), count=cfg.B * ng * cfg.d).reshape(cfg.B, ng, cfg.d)
        self.rows = []
        for b in range(cfg.B):
            rr = self._route(b)
            if bench is not None:
                import torch
                r = torch.as_tensor(np.asarray(rr, dtype=np.int64), device=bench.dev)
                self.rows.append((_bits(bench.inp["K"][b][r]), _bits(bench.inp["V"][b][r])))
            else:
                self.rows.append((R.host_rows(cfg.seed, R.tid(R.KIND_K, 0), (cfg.Hkv, cfg.D), rr, True, b, cfg.Tk_max),
                                  R.host_rows(cfg.seed, R.tid(R.KIND_V, 0), (cfg.Hkv, cfg.D), rr, True, b, cfg.Tk_max)))

    def _route(self, b):
        import oracle
        c = self.cfg
        if c.group_size:
            return oracle.hier_gist_route_unfold(self.qr[b], self.mk[b], self.gk[b], c.group_size, c.chunk_len,
                                                 c.k_groups, c.k_chunks, self.step + 1)[0]
        return oracle.gist_route_unfold(self.qr[b], self.gk[b], c.chunk_len, c.k_chunks, self.step + 1)[0]

    def run(self):
        import oracle
        c = self.cfg
        for b in range(c.B):
            self._route(b)
        oracle.sparse_attention_decode(self.q, [r[0] for r in self.rows], [r[1] for r in self.rows])


def cpu_baseline_gist(cfg: R.Gist, budget_s: float, bench: GistBench | None = None):
    o = OracleGist(cfg, 0, bench)
    reps, el = _time_loop(o.run, budget_s, 200)
    return {"value": round(reps / el, 4), "unit": "steps/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"gist decode step 0 of {cfg.name} (all {cfg.B} sequences: routing over every gist, "
                      f"unfolding, attention), repeated {reps} times in {el:.1f} s; numpy fp64; input "
                      "preparation and row regeneration untimed"}


def run_reference(args, cfg, rank, world):
    """The oracle as the reference arm: same metric, unit and config, each
    step a bounded sample of the workload, scaled to whole steps."""
    if rank != 0:
        return None
    cores = _blas_threads()
    if isinstance(cfg, R.Decode):
        # one sequence of the step; with several indexer groups, group 0 and its layers
        few = cfg.n_groups <= 1
        o = OracleDecode(cfg, 0, range(cfg.n_groups) if few else [0],
                         range(cfg.n_layers) if few else range(cfg.share_every), [0])
        scale = cfg.B * (1 if few else cfg.n_groups)
        metric, unit, per = "decode steps/s", "steps/s", 1.0
        sample = (f"sequence 0 of {cfg.B}" + ("" if few else f", indexer group 0 of {cfg.n_groups} and its layers")
                  + f" per step (scaled by {scale}); oracle in numpy fp64")
        config = {"workload": cfg.name, "batch": cfg.B, "context": cfg.N, "layers": cfg.n_layers,
                  "share_every": cfg.share_every, "d_idx": cfg.d, "q_heads": cfg.Hq, "kv_heads": cfg.Hkv,
                  "head_dim": cfg.D, "top_k": cfg.k, "parallelism": "host cores"}
    elif isinstance(cfg, R.Prefill):
        rows = _prefill_sample_rows(cfg, cfg.L if cfg.L <= 2048 else 4)
        o = OraclePrefill(cfg, rows, None)
        scale = cfg.B * cfg.L / len(rows)
        metric, unit, per = "prefill tokens/s", "tokens/s", float(cfg.B * cfg.L)
        sample = (f"{len(rows)} of {cfg.L} query rows per step (evenly spread; scaled to the whole "
                  "prefill); oracle in numpy fp64")
        config = {"workload": cfg.name, "batch": cfg.B, "seq_len": cfg.L, "layers": cfg.n_layers,
                  "share_every": cfg.share_every, "d_idx": cfg.d, "q_heads": cfg.Hq, "kv_heads": cfg.Hkv,
                  "head_dim": cfg.D, "top_k": cfg.k, "needles": cfg.n_needles, "parallelism": "host cores"}
    else:
        o = OracleGist(cfg, 0, None)
        scale = 1.0
        metric, unit, per = "decode steps/s", "steps/s", 1.0
        sample = f"the whole step (all {cfg.B} sequences); oracle in numpy fp64"
        config = {"workload": cfg.name, "batch": cfg.B, "chunks": cfg.n_chunks, "chunk_len": cfg.chunk_len,
                  "d_route": cfg.d, "top_k_chunks": cfg.k_chunks, "q_heads": cfg.Hq, "kv_heads": cfg.Hkv,
                  "head_dim": cfg.D, "parallelism": "host cores"}
    for _ in range(args.warmup):
        o.run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        o.run()
    el = time.perf_counter() - t0
    s_per_step = el * scale / args.steps
    value = per / s_per_step
    return {"impl": "reference", "metric": metric, "value": round(value, 5), "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(s_per_step * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": {"value": round(value, 5), "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 5), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- driver

def measure(ctx: Ctx, name: str, headline: bool):
    import torch
    args = ctx.args
    cfg = CONFIGS[name]
    if args.layers is not None and isinstance(cfg, R.Decode) and headline:
        cfg = R.Decode(**{**cfg.__dict__, "n_layers": args.layers, "name": f"{cfg.name}_first{args.layers}layers"})
    steps, warmup = args.steps, args.warmup
    if not headline and name == "prefill_64k":
        steps, warmup = min(steps, 10), 3      # ~0.23 s per step
    try:
        if isinstance(cfg, R.Decode):
            return measure_decode(ctx, cfg, steps, warmup, headline)
        if isinstance(cfg, R.Prefill):
            return measure_prefill(ctx, cfg, steps, warmup)
        return measure_gist(ctx, cfg, steps, warmup)
    finally:
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def run_native(args, rank, world):
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    ctx = Ctx(args, rank, world, dev, load_peaks())
    line = measure(ctx, args.config, headline=True)
    if args.config == "decode_32k" and not args.no_workloads and args.layers is None:
        # each workload has its own timed region, launch count and clocks
        line["workloads"] = {CONFIGS[n].name: measure(ctx, n, headline=False) for n in SUB_WORKLOADS}
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--config", choices=sorted(CONFIGS), default="decode_32k")
    ap.add_argument("--no-workloads", action="store_true",
                    help="headline only (skip the other workloads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=None,
                    help="decode only: run fewer layers (small profiling cases; not the headline)")
    ap.add_argument("--cpu-seconds", type=float, default=8.0)
    ap.add_argument("--soak-seconds", type=float, default=1.0,
                    help="busy time before the timed region so clocks are sampled under load")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end legs (profiling runs)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per launch of the headline's roofline kernel from an ncu capture")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    cfg = CONFIGS[args.config]
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
        line = run_native(args, rank, world)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
