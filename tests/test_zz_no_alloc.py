"""The decode-attention entry point that allocates nothing.

Some callers cannot call cudaMalloc (a host process that may only pass on the
buffers it was handed, or code on a path where allocation is not allowed), so
they cannot provide the workspace sa_sparse_attn_decode needs.
sa_sparse_attn_decode_noalloc serves them from a fixed scratch array inside
the library.  This test calls it through the C ABI twice in a row (two
shapes, the second with more sequences and heads than the first) and checks
each result against sa_sparse_attn_decode given a caller workspace, and both
against the CPU oracle, within the attention tolerance the other tests use.  It is collected last so that a run
stopping at its first failure has run every other test already, and it
passes both alone in a fresh process and after the other tests."""
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


def _inputs(seed, B, Hq, Hkv, Tk_max, k):
    """Device inputs, and the oracle's result for them."""
    rng = np.random.default_rng(seed)
    qh = _normals(seed, 1, (B, Hq, 128))
    Kh = _normals(seed, 2, (B, Tk_max, Hkv, 128))
    Vh = _normals(seed, 3, (B, Tk_max, Hkv, 128))
    counts = [k - 7 * (b % 3) for b in range(B)]
    idx = np.full((B, k), -1, np.int32)
    for b, c in enumerate(counts):
        idx[b, :c] = np.sort(rng.choice(Tk_max, size=c, replace=False))
    want, _ = oracle.sparse_attention_decode(qh, [Kh[b, idx[b, :c]] for b, c in enumerate(counts)],
                                             [Vh[b, idx[b, :c]] for b, c in enumerate(counts)])
    return (to_dev(qh), to_dev(Kh), to_dev(Vh), i32(idx), i32(counts)), want


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _call_noalloc(q, K, V, idx, cnt, out):
    B, Hq, D = q.shape
    Tk_max, Hkv = K.shape[1], K.shape[2]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return S.lib().sa_sparse_attn_decode_noalloc(_ptr(q), _ptr(K), _ptr(V), _ptr(idx), _ptr(cnt), B, Tk_max,
                                                 Hq, Hkv, D, idx.shape[1], 0.0, _ptr(out), None, stream)


def _call_with_workspace(q, K, V, idx, cnt, out):
    B, Hq, D = q.shape
    Tk_max, Hkv = K.shape[1], K.shape[2]
    k = idx.shape[1]
    need = S.lib().sa_sparse_attn_decode_workspace(B, Hq, Hkv, D, k)
    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=q.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return S.lib().sa_sparse_attn_decode(_ptr(q), _ptr(K), _ptr(V), _ptr(idx), _ptr(cnt), B, Tk_max, Hq, Hkv,
                                         D, k, 0.0, _ptr(out), None, _ptr(ws), ws.numel(), stream)


def test_noalloc_decode_matches_the_workspace_entry_point_twice_in_a_row():
    torch.cuda.set_device(dev())
    shapes = [(2, 16, 4, 3000, 700), (8, 32, 8, 5000, 2048)]   # (B, Hq, Hkv, Tk_max, k)
    for i, (B, Hq, Hkv, Tk_max, k) in enumerate(shapes):
        (q, K, V, idx, cnt), want = _inputs(600 + i, B, Hq, Hkv, Tk_max, k)
        got = torch.empty_like(q)
        ref = torch.empty_like(q)
        assert _call_noalloc(q, K, V, idx, cnt, got) == S.SA_OK, S.last_error()
        assert _call_with_workspace(q, K, V, idx, cnt, ref) == S.SA_OK, S.last_error()
        torch.cuda.synchronize()
        got, ref = got.float().cpu().numpy(), ref.float().cpu().numpy()
        assert_close_attn(got, ref, f"no-alloc call {i + 1} against the workspace entry point")
        assert_close_attn(got, want, f"no-alloc call {i + 1} against the oracle")
        assert_close_attn(ref, want, f"workspace entry point, shape {i + 1}, against the oracle")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    B, Hq, Hkv, k = 4096, 64, 4, 65536   # needs far more than the fixed scratch
    need = S.lib().sa_sparse_attn_decode_workspace(B, Hq, Hkv, 128, k)
    assert need > (8 << 20)
    fake = ctypes.c_void_p(0x100000)      # never dereferenced: rejected on the host
    st = S.lib().sa_sparse_attn_decode_noalloc(fake, fake, fake, fake, fake, B, 100, Hq, Hkv, 128, k, 0.0,
                                               fake, None, None)
    assert st == S.SA_ERR_UNSUPPORTED
    assert "scratch" in S.last_error()
