"""The debug build (libsa_debug.so, compiled with SA_DEBUG), on the GPU.

It checks every gathered row index a call uses against the cache and puts a
canary after each workspace's used bytes; a violation is recorded in a
device record (read back through sa_debug_read) and never traps -- the
access is clamped exactly as in the release build.  The bad indices below
are therefore safe to pass: both builds clamp them into the cache, so the
calls read a valid row; only the debug build reports them."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gen import counter_hash as ch
from shared_top_routing_b200 import sa as S
from tests.gpu_util import assert_close_attn, dev, i32, to_dev

pytestmark = pytest.mark.gpu


def _normals(seed, tid, shape):
    return ch.normal_bf16(seed, tid, count=int(np.prod(shape))).reshape(shape)


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _decode(L, q, K, V, idx, cnt):
    B, Hq, D = q.shape
    Tk_max, Hkv = K.shape[1], K.shape[2]
    k = idx.shape[1]
    ws = torch.zeros(L.sa_sparse_attn_decode_workspace(B, Hq, Hkv, D, k), dtype=torch.uint8, device=dev())
    out = torch.empty_like(q)
    st = L.sa_sparse_attn_decode(_p(q), _p(K), _p(V), _p(idx), _p(cnt), B, Tk_max, Hq, Hkv, D, k, 0.0, _p(out),
                                 None, _p(ws), ws.numel(), _stream())
    assert st == S.SA_OK
    return out, ws


def test_debug_build_flags_an_out_of_range_decode_index_and_clamps_it():
    LD, LR = S.lib_debug(), S.lib()
    assert LD.sa_debug_enabled() == 1 and LR.sa_debug_enabled() == 0
    S.debug_read(LD, reset=True)
    B, Hq, Hkv, Tk_max, k = 2, 8, 2, 500, 64
    q = _normals(1, 1, (B, Hq, 128))
    K = _normals(1, 2, (B, Tk_max, Hkv, 128))
    V = _normals(1, 3, (B, Tk_max, Hkv, 128))
    idx = np.tile(np.arange(k, dtype=np.int32) * 3, (B, 1))
    cnt = [k, k - 10]
    # clean call: nothing recorded
    out_ok, _ = _decode(LD, to_dev(q), to_dev(K), to_dev(V), i32(idx), i32(cnt))
    torch.cuda.synchronize()
    assert S.debug_read(LD) == [0, 0, 0, 0]
    # one used index past the cache (row 7 of sequence 1): recorded, and clamped to the last row
    bad = idx.copy()
    bad[1, 7] = Tk_max + 5
    outs = []
    for L in (LD, LR):
        o, _ = _decode(L, to_dev(q), to_dev(K), to_dev(V), i32(bad), i32(cnt))
        outs.append(o)
    torch.cuda.synchronize()
    rec = S.debug_read(LD)
    assert rec[0] == 2 and rec[1] == Tk_max + 5 and rec[2] == Tk_max and rec[3] >= 1
    clamped = bad.copy()
    clamped[1, 7] = Tk_max - 1
    ref, _ = oracle.sparse_attention_decode(q, [K[b, clamped[b, :c]] for b, c in enumerate(cnt)],
                                            [V[b, clamped[b, :c]] for b, c in enumerate(cnt)])
    for o in outs:
        assert_close_attn(o.float().cpu().numpy(), ref, "clamped decode")
    # an index past the count is never used, so never reported
    unused = idx.copy()
    unused[1, k - 1] = -100
    _decode(LD, to_dev(q), to_dev(K), to_dev(V), i32(unused), i32(cnt))
    torch.cuda.synchronize()
    assert S.debug_read(LD) == [0, 0, 0, 0]


def test_debug_build_flags_bad_prefill_and_gather_indices():
    LD = S.lib_debug()
    S.debug_read(LD, reset=True)
    B, T, Hq, Hkv, k = 1, 40, 4, 2, 8
    q = to_dev(_normals(2, 1, (B, T, Hq, 128)))
    K = to_dev(_normals(2, 2, (B, T, Hkv, 128)))
    V = to_dev(_normals(2, 3, (B, T, Hkv, 128)))
    idx = np.zeros((B, T, k), np.int32)
    cnt = np.full((B, T), 1, np.int32)
    idx[0, 5, 0] = -3
    out = torch.empty_like(q)
    st = LD.sa_sparse_attn_prefill(_p(q), _p(K), _p(V), _p(i32(idx)), _p(i32(cnt)), B, T, T, Hq, Hkv, 128, k, 0.0,
                                   _p(out), None, _stream())
    assert st == S.SA_OK
    torch.cuda.synchronize()
    assert S.debug_read(LD)[:3] == [1, -3, T]
    gi = np.arange(k, dtype=np.int32)[None].repeat(B, 0)
    gi[0, 2] = T
    kr = torch.empty((B, k, Hkv * 128 + 8), dtype=torch.bfloat16, device=dev())
    vr = torch.empty_like(kr)
    st = LD.sa_gather_rows(_p(K), _p(V), _p(i32(gi)), _p(i32([k])), B, T, Hkv, 128, k, _p(kr), _p(vr), _stream())
    assert st == S.SA_OK
    torch.cuda.synchronize()
    assert S.debug_read(LD)[:3] == [3, T, T]


def test_debug_build_canaries():
    """Every workspace call leaves its canary intact after its kernels; a
    changed canary byte is reported with the call and the byte."""
    LD = S.lib_debug()
    S.debug_read(LD, reset=True)
    B, Hq, Hkv, Tk_max, k = 4, 32, 8, 3000, 2048
    q = to_dev(_normals(3, 1, (B, Hq, 128)))
    K = to_dev(_normals(3, 2, (B, Tk_max, Hkv, 128)))
    V = to_dev(_normals(3, 3, (B, Tk_max, Hkv, 128)))
    idx = i32(np.sort(np.random.default_rng(3).choice(Tk_max, (B, k)), axis=1))
    _, ws = _decode(LD, q, K, V, idx, i32([k, 1000, 0, 7]))
    torch.cuda.synchronize()
    assert S.debug_read(LD) == [0, 0, 0, 0]
    need = ws.numel()
    canary = ws[need - 256:].cpu().numpy()
    assert (canary == 0xA5).all()                        # armed by the call, intact after its kernels
    assert LD.sa_debug_check_canary(_p(ws), need - 256, 3, _stream()) == S.SA_OK
    torch.cuda.synchronize()
    assert S.debug_read(LD) == [0, 0, 0, 0]
    ws[need - 256 + 77] = 0                              # damage one byte
    assert LD.sa_debug_check_canary(_p(ws), need - 256, 3, _stream()) == S.SA_OK
    torch.cuda.synchronize()
    assert S.debug_read(LD)[:3] == [4, 3, 77]


def test_debug_build_indexer_and_gist_leave_their_canaries_intact():
    LD = S.lib_debug()
    S.debug_read(LD, reset=True)
    B, T, d, k = 3, 20000, 128, 2048
    qi = to_dev(ch.int_bf16(4, 1, count=B * d).reshape(B, d))
    ki = to_dev(ch.int_bf16(4, 2, count=B * T * d).reshape(B, T, d))
    ws = torch.zeros(LD.sa_index_score_topk_workspace(B, 1, T, d, k), dtype=torch.uint8, device=dev())
    idx = torch.empty((B, 1, k), dtype=torch.int32, device=dev())
    cnt = torch.empty((B, 1), dtype=torch.int32, device=dev())
    assert LD.sa_index_score_topk(_p(qi), _p(ki), B, 1, T, T, d, k, T - 1, None, _p(idx), _p(cnt), None, _p(ws),
                                  ws.numel(), _stream()) == S.SA_OK
    gk = to_dev(ch.int_bf16(4, 3, count=B * 8192 * d).reshape(B, 8192, d))
    wsg = torch.zeros(LD.sa_gist_route_unfold_workspace(B, 8192, d, 64), dtype=torch.uint8, device=dev())
    rows = torch.empty((B, 64 * 17 + 16), dtype=torch.int32, device=dev())
    rc = torch.empty((B,), dtype=torch.int32, device=dev())
    assert LD.sa_gist_route_unfold(_p(qi), _p(gk), B, 8192, 16, d, 64, None, _p(rows), _p(rc), None, _p(wsg),
                                   wsg.numel(), _stream()) == S.SA_OK
    torch.cuda.synchronize()
    assert S.debug_read(LD) == [0, 0, 0, 0]
    ridx, _ = oracle.index_topk(ch.int_bf16(4, 1, count=B * d).reshape(B, 1, d),
                                ch.int_bf16(4, 2, count=B * T * d).reshape(B, T, d), T, T - 1, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
