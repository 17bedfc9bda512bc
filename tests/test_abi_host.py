"""C ABI checks that need no GPU: the library loads and exports every symbol
include/sa.h declares, host-side validation rejects bad arguments before
any CUDA call, and the shared index cache follows its full/shared rules.

Only calls that fail validation, size queries and the host-only index cache
are made here; nothing computes."""
import ctypes
import os
import re

import pytest

from shared_top_routing_b200 import sa as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sa.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z_]+)\s*\(", txt)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("sa_index_score_topk", "sa_sparse_attn_prefill", "sa_sparse_attn_decode",
                 "sa_gist_route_unfold", "sa_index_cache_create", "sa_index_cache_get",
                 "sa_index_cache_update"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(S.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    # the binding knows every declared entry point
    assert set(_declared()) <= set(S.SIGNATURES)


def test_status_strings_and_version():
    assert S.lib().sa_version() == 100
    for code in range(7):
        assert S.status_string(code)
    assert "unknown" in S.status_string(99)


FAKE = ctypes.c_void_p(0x100000)   # never dereferenced: every call below fails validation


def _topk(**kw):
    a = dict(q=FAKE, k=FAKE, B=1, Tq=1, Tk=10, Tk_max=10, d=64, kk=8, q_pos0=9, kv_len=None,
             idx=FAKE, cnt=FAKE, score=None, ws=None, ws_bytes=0)
    a.update(kw)
    return S.lib().sa_index_score_topk(a["q"], a["k"], a["B"], a["Tq"], a["Tk"], a["Tk_max"], a["d"],
                                       a["kk"], a["q_pos0"], a["kv_len"], a["idx"], a["cnt"],
                                       a["score"], a["ws"], a["ws_bytes"], None)


def test_index_topk_validation():
    assert _topk(Tk=11) == S.SA_ERR_INVALID_ARG                 # Tk > Tk_max
    assert _topk(B=-1) == S.SA_ERR_INVALID_ARG
    assert _topk(Tq=0) == S.SA_ERR_INVALID_ARG
    assert _topk(kk=0) == S.SA_ERR_INVALID_ARG
    assert _topk(kk=S.SA_MAX_K + 1) == S.SA_ERR_UNSUPPORTED
    assert _topk(d=96) == S.SA_ERR_UNSUPPORTED
    assert _topk(q=None) == S.SA_ERR_INVALID_ARG
    assert _topk(k=ctypes.c_void_p(0x100008)) == S.SA_ERR_INVALID_ARG  # misaligned
    assert "aligned" in S.last_error()
    assert _topk(ws=None, ws_bytes=0) == S.SA_ERR_WORKSPACE
    assert _topk(ws=ctypes.c_void_p(0x100010), ws_bytes=1 << 30) == S.SA_ERR_WORKSPACE
    assert _topk(ws=FAKE, ws_bytes=16) == S.SA_ERR_WORKSPACE
    assert "bytes" in S.last_error()
    assert _topk(B=0) == S.SA_OK                                # nothing to do, no launch


def _fp8(**kw):
    a = dict(q=FAKE, w=None, k=FAKE, B=1, H=1, Tk=10, Tk_max=10, d=64, kk=4, q_pos0=9, kv_len=None, idx=FAKE,
             cnt=FAKE, score=None, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    return S.lib().sa_index_score_topk_fp8(a["q"], a["w"], a["k"], a["B"], a["H"], a["Tk"], a["Tk_max"], a["d"],
                                           a["kk"], a["q_pos0"], a["kv_len"], a["idx"], a["cnt"], a["score"],
                                           a["ws"], a["ws_bytes"], None)


def test_fp8_index_topk_validation():
    """The fp8 indexer checks its arguments on the host, before any launch."""
    assert _fp8(H=2) == S.SA_ERR_INVALID_ARG                    # several heads need weights
    assert "weights" in S.last_error()
    assert _fp8(H=0) == S.SA_ERR_INVALID_ARG
    assert _fp8(H=33, w=FAKE) == S.SA_ERR_UNSUPPORTED
    assert _fp8(d=96) == S.SA_ERR_UNSUPPORTED
    assert _fp8(Tk=11) == S.SA_ERR_INVALID_ARG
    assert _fp8(kk=S.SA_MAX_K + 1) == S.SA_ERR_UNSUPPORTED
    assert _fp8(k=ctypes.c_void_p(0x100008)) == S.SA_ERR_INVALID_ARG   # misaligned keys
    assert _fp8(H=4, w=ctypes.c_void_p(0x100002)) == S.SA_ERR_INVALID_ARG   # misaligned weights
    assert _fp8(ws=FAKE, ws_bytes=16) == S.SA_ERR_WORKSPACE
    assert _fp8(B=0) == S.SA_OK
    L = S.lib()
    assert L.sa_index_score_topk_fp8_workspace(8, 32832, 16, 128, 2048) == \
        L.sa_index_score_topk_workspace(8, 1, 32832, 128, 2048)


def test_workspace_status_validation():
    """A NULL workspace is refused on the host; the timeout status has its
    own string."""
    assert S.lib().sa_workspace_status(None, None) == S.SA_ERR_INVALID_ARG
    assert "workspace" in S.last_error()
    assert "wait" in S.status_string(S.SA_ERR_TIMEOUT)


def test_workspace_sizes():
    L = S.lib()
    small = L.sa_index_score_topk_workspace(8, 1, 4096, 128, 2048)
    big = L.sa_index_score_topk_workspace(8, 1, 32832, 128, 2048)
    assert 0 < small < big
    assert big % 256 == 0
    assert L.sa_index_score_topk_workspace(0, 1, 100, 64, 8) == 0
    # prefill: key and candidate-position slabs of at most 1 GiB, plus group
    # maxima (2048 rows x 8224 16-bit entries) and per-row words
    ws = L.sa_index_score_topk_workspace(1, 65536, 65536, 64, 2048)
    assert (1 << 30) < ws <= (1 << 30) + (40 << 20)
    assert L.sa_sparse_attn_decode_workspace(8, 32, 8, 128, 2048) > 0
    assert L.sa_gist_route_unfold_workspace(4, 8192, 128, 64) > 0


def test_attention_validation():
    L = S.lib()

    def pre(**kw):
        a = dict(B=1, T=4, Tk_max=16, Hq=8, Hkv=2, D=128, k=8, q=FAKE, out=FAKE)
        a.update(kw)
        return L.sa_sparse_attn_prefill(a["q"], FAKE, FAKE, FAKE, FAKE, a["B"], a["T"], a["Tk_max"],
                                        a["Hq"], a["Hkv"], a["D"], a["k"], 0.0, a["out"], None, None)

    assert pre(D=64) == S.SA_ERR_UNSUPPORTED
    assert pre(Hq=6, Hkv=4) == S.SA_ERR_INVALID_ARG
    assert pre(Hq=64, Hkv=2) == S.SA_ERR_UNSUPPORTED           # G = 32 > 16
    assert pre(q=None) == S.SA_ERR_INVALID_ARG
    assert pre(out=ctypes.c_void_p(0x100002)) == S.SA_ERR_INVALID_ARG
    assert pre(T=0) == S.SA_OK
    st = L.sa_sparse_attn_decode(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 16, 8, 2, 128, 8, 0.0, FAKE, None,
                                 None, 0, None)
    assert st == S.SA_ERR_WORKSPACE


def test_gist_validation():
    L = S.lib()

    def gist(**kw):
        a = dict(B=1, n=64, cl=16, d=128, kc=4, ws=None, wsb=0)
        a.update(kw)
        return L.sa_gist_route_unfold(FAKE, FAKE, a["B"], a["n"], a["cl"], a["d"], a["kc"], FAKE, FAKE,
                                      FAKE, None, a["ws"], a["wsb"], None)

    assert gist(cl=0) == S.SA_ERR_UNSUPPORTED
    assert gist(kc=0) == S.SA_ERR_INVALID_ARG
    assert gist(d=32) == S.SA_ERR_UNSUPPORTED
    assert gist(n=-1) == S.SA_ERR_INVALID_ARG
    assert gist() == S.SA_ERR_WORKSPACE
    assert gist(B=0) == S.SA_OK


def _cache(n_layers, pattern=None, share_every=4):
    h = ctypes.c_void_p()
    pat = pattern.encode() if pattern else None
    st = S.lib().sa_index_cache_create(n_layers, pat, share_every, 2, 1, 16, FAKE, FAKE, ctypes.byref(h))
    return st, h


def test_index_cache_schedule_and_staleness():
    """Page "清华提出IndexCache技术…", §二 and §六: full layers write one
    buffer, shared layers read the nearest preceding full layer's index."""
    L = S.lib()
    st, h = _cache(8, share_every=4)
    assert st == S.SA_OK
    try:
        assert [L.sa_index_cache_is_full(h, l) for l in range(8)] == [1, 0, 0, 0, 1, 0, 0, 0]
        assert [L.sa_index_cache_owner(h, l) for l in range(8)] == [0, 0, 0, 0, 4, 4, 4, 4]
        assert L.sa_index_cache_is_full(h, 8) == -1
        ip, cp, ver = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_uint64()
        get = lambda l: L.sa_index_cache_get(h, l, ctypes.byref(ip), ctypes.byref(cp), ctypes.byref(ver))
        assert L.sa_index_cache_begin_step(h) == S.SA_OK
        assert get(1) == S.SA_ERR_STALE_INDEX                   # layer 0 has not run yet
        assert L.sa_index_cache_mark_written(h, 1) == S.SA_ERR_INVALID_ARG  # shared layer
        assert L.sa_index_cache_mark_written(h, 0) == S.SA_OK
        versions = []
        for l in range(4):
            assert get(l) == S.SA_OK
            assert ip.value == FAKE.value and cp.value == FAKE.value
            versions.append(ver.value)
        assert len(set(versions)) == 1                           # one index for the group
        assert get(4) == S.SA_ERR_STALE_INDEX
        assert L.sa_index_cache_mark_written(h, 4) == S.SA_OK
        assert get(5) == S.SA_OK and ver.value == versions[0] + 1
        assert get(2) == S.SA_ERR_STALE_INDEX                   # overwritten by layer 4
        assert L.sa_index_cache_begin_step(h) == S.SA_OK
        assert get(4) == S.SA_ERR_STALE_INDEX                   # new step
        # update on a shared layer is refused before any launch
        st = L.sa_index_cache_update(h, 3, FAKE, FAKE, 10, 10, 64, 9, None, None, 0, None)
        assert st == S.SA_ERR_INVALID_ARG
    finally:
        L.sa_index_cache_destroy(h)


def test_index_cache_pattern_rules():
    L = S.lib()
    st, h = _cache(6, pattern="FSSFSF")
    assert st == S.SA_OK
    assert [L.sa_index_cache_owner(h, l) for l in range(6)] == [0, 0, 0, 3, 3, 5]
    L.sa_index_cache_destroy(h)
    for bad in ("SFFFFF", "FSXFFF", "FSSFSFF"):   # starts shared, bad letter, wrong length
        st, h = _cache(6, pattern=bad)
        assert st == S.SA_ERR_INVALID_ARG
    st, h = _cache(4, pattern=None, share_every=0)
    assert st == S.SA_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert S.lib().sa_index_cache_create(4, None, 4, 1, 1, S.SA_MAX_K + 1, FAKE, FAKE,
                                         ctypes.byref(h)) == S.SA_ERR_UNSUPPORTED


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(S, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(S, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        S.lib()


GIB = 1 << 30


@pytest.mark.parametrize("B,Tq,Tk_max,k", [(1, 2048, 2048, 256), (1, 65536, 65536, 2048), (2, 300, 20480, 1000),
                                           (3, 100000, 131072, 4096), (1, 4600, 8200, 4096),
                                           (64, 4096, 200000, 2048)])
def test_prefill_workspace_properties(B, Tq, Tk_max, k):
    """Properties of the prefill workspace size: 256-byte multiples; room for
    the two [rows, Tk_max] u32 slabs of at least one batch of min(Tq, 128)
    rows per sequence (the whole prefill when it fits under the cap); the
    slabs capped at 1 GiB unless the 128-row minimum forces more, with the
    per-row extras (group maxima, bound, run counts) small beside them."""
    L = S.lib()
    got = L.sa_index_score_topk_workspace(B, Tq, Tk_max, 64, k)
    assert got % 256 == 0
    assert got >= 2 * B * min(Tq, 128) * Tk_max * 4
    ld = (Tk_max + 255) // 256 * 256
    if B * Tq * ld * 8 <= GIB:
        assert got >= 2 * B * Tq * Tk_max * 4
    if B * 128 * ld * 8 <= GIB:
        assert got <= GIB * 5 // 4
    else:
        assert got <= B * 128 * ld * 8 * 5 // 4


def test_prefill_workspace_grows_with_the_shape_while_one_batch_holds_every_row():
    L = S.lib()
    for B, Tq, k in [(1, 300, 256), (2, 1000, 2048)]:
        sizes = [L.sa_index_score_topk_workspace(B, Tq, T, 64, k) for T in (2048, 4096, 8192, 16384, 40000)]
        assert sizes == sorted(sizes)
    sizes = [L.sa_index_score_topk_workspace(b, 300, 8192, 64, 256) for b in (1, 2, 3, 4)]
    assert sizes == sorted(sizes)


def test_greedy_pattern_search_matches_the_oracle():
    """The library's host-side layer-role search ([IC] §三, with the index
    overlap as the measure) picks the oracle's pattern on random and block
    structured overlap matrices."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(5)
    for L, n_full in ((6, 2), (12, 3), (28, 7), (47, 12), (4, 4), (5, 1)):
        ov = rng.uniform(0.2, 1.0, (L, L))
        np.fill_diagonal(ov, 1.0)
        assert S.sa_index_pattern_greedy(ov, n_full) == oracle.greedy_pattern(ov, n_full)
    blocks = np.full((8, 8), 0.1)   # two blocks of layers: {0, 1, 2} and {3, ..., 7}
    blocks[:3, :3] = blocks[3:, 3:] = 0.95
    np.fill_diagonal(blocks, 1.0)
    assert S.sa_index_pattern_greedy(blocks, 2) == "FSSFSSSS"
    buf = ctypes.create_string_buffer(9)
    assert S.lib().sa_index_pattern_greedy(None, 8, 2, buf) == S.SA_ERR_INVALID_ARG
    assert S.lib().sa_index_overlap(None, None, None, None, 3, 16, None, None) == S.SA_ERR_INVALID_ARG


def test_debug_library_loads_and_reports_itself():
    """libsa_debug.so exports the same ABI; it says it is a debug build, the
    release library says it is not, and both refuse a NULL record."""
    LD = S.lib_debug()
    assert LD.sa_debug_enabled() == 1
    assert S.lib().sa_debug_enabled() == 0
    assert LD.sa_debug_read(None, 0) == S.SA_ERR_INVALID_ARG
    assert S.lib().sa_debug_check_canary(None, 0, 1, None) == S.SA_ERR_INVALID_ARG
    # the debug workspaces carry the 256-byte canary
    assert LD.sa_sparse_attn_decode_workspace(8, 32, 8, 128, 2048) == \
        S.lib().sa_sparse_attn_decode_workspace(8, 32, 8, 128, 2048) + 256
