"""Full-size parity of the five benchmark workloads, in the launch
configuration bench.py times.

Device inputs come from the device generator; the oracle regenerates the
host side bit for bit (the generators are cross-checked in
test_gpu_parity.py).  Indices are checked bit-exactly on every row the oracle
affords and on sampled rows otherwise; attention on sampled rows and heads."""
import numpy as np
import pytest
import torch

import oracle
import shared_top_routing_b200 as sa
from gen import counter_hash as ch
from gen import recipes as R
from gen import torch_inputs as TI
from tests.gpu_util import assert_close_attn, dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


# ----------------------------------------------------------------- decode

def _check_decode(cfg, steps, check_groups, check_layers):
    d = dev()
    inp = TI.decode_inputs(cfg, d)
    cache = sa.IndexCache(cfg.n_layers, cfg.B, 1, cfg.k, share_every=cfg.share_every, device=d)
    L = sa.lib()
    if cfg.fp8_idx:
        ws_bytes = L.sa_index_score_topk_fp8_workspace(cfg.B, cfg.Tk_max, cfg.H_idx, cfg.d, cfg.k)
    elif cfg.H_idx == 1:
        ws_bytes = L.sa_index_score_topk_workspace(cfg.B, 1, cfg.Tk_max, cfg.d, cfg.k)
    else:
        ws_bytes = L.sa_index_score_topk_mh_workspace(cfg.B, 1, cfg.Tk_max, cfg.H_idx, cfg.d, cfg.k)
    ws_idx = torch.zeros(ws_bytes, dtype=torch.uint8, device=d)
    outs = [torch.empty((cfg.B, cfg.Hq, cfg.D), dtype=torch.bfloat16, device=d) for _ in range(cfg.n_layers)]
    host_int = ch.int_e4m3 if cfg.fp8_idx else ch.int_bf16   # E4M3 codes or bf16 bits of the same integers
    host_k = {g: host_int(cfg.seed, R.tid(R.KIND_K_IDX, g), count=cfg.B * cfg.Tk_max * cfg.d)
              .reshape(cfg.B, cfg.Tk_max, cfg.d) for g in check_groups}
    for s in steps:
        # run the whole step, snapshotting each group's index right after its layers
        Tk = cfg.N + s + 1
        cache.begin_step()
        got_idx = {}
        versions = {}
        for layer in range(cfg.n_layers):
            g = layer // cfg.share_every
            if cache.is_full(layer) == 1:
                if cfg.fp8_idx:
                    wi = inp["w_idx"][g][s] if cfg.H_idx > 1 else None
                    sa.sa_index_score_topk_fp8(inp["q_idx"][g][s], inp["k_idx"][g], cfg.k, w=wi, Tk=Tk, q_pos0=Tk - 1,
                                               idx_out=cache.idx_buf.view(cfg.B, cfg.k),
                                               count_out=cache.count_buf.view(cfg.B), ws=ws_idx)
                    cache.mark_written(layer)
                elif cfg.H_idx == 1:
                    cache.update(layer, inp["q_idx"][g][s], inp["k_idx"][g], Tk=Tk, q_pos0=Tk - 1, ws=ws_idx)
                else:
                    sa.sa_index_score_topk_mh(inp["q_idx"][g][s], inp["w_idx"][g][s], inp["k_idx"][g], cfg.k,
                                              Tk=Tk, q_pos0=Tk - 1, idx_out=cache.idx_buf,
                                              count_out=cache.count_buf, ws=ws_idx)
                    cache.mark_written(layer)
                versions[g] = None
            idx, cnt, ver = cache.get_tensors(layer)
            versions[g] = ver if versions[g] is None else versions[g]
            assert ver == versions[g]          # every layer of the group reads the same write
            if cfg.shared_kv:                  # one cache: gather once, every layer over the compact rows
                if layer % cfg.share_every == 0:
                    kr, vr = sa.sa_gather_rows(inp["K"][layer], inp["V"][layer], idx.view(cfg.B, cfg.k),
                                               cnt.view(cfg.B))
                sa.sa_sparse_attn_decode_rows(inp["q"][layer][s], kr, vr, cnt.view(cfg.B), out=outs[layer])
            else:
                sa.sa_sparse_attn_decode(inp["q"][layer][s], inp["K"][layer], inp["V"][layer],
                                         idx.view(cfg.B, cfg.k), cnt.view(cfg.B), out=outs[layer])
            if g in check_groups and layer % cfg.share_every == 0:
                got_idx[g] = (idx.view(cfg.B, cfg.k).clone(), cnt.view(cfg.B).clone())
            if layer in check_layers:
                outs[layer] = outs[layer].clone()
        torch.cuda.synchronize()
        for g in check_groups:
            qi = R.decode_q_idx_host(cfg, g, s)
            if cfg.fp8_idx:
                qi = ch.e4m3_codes(ch.bf16_bits_to_f64(qi))
            wi = R.decode_w_idx_host(cfg, g, s)[:, None] if cfg.H_idx > 1 else None
            ridx, rcnt = oracle.index_topk(qi[:, None], host_k[g], Tk, Tk - 1, cfg.k, w=wi)
            gi, gc = got_idx[g]
            np.testing.assert_array_equal(gc.cpu().numpy(), rcnt[:, 0])
            np.testing.assert_array_equal(gi.cpu().numpy(), ridx[:, 0])
        for layer in check_layers:
            g = layer // cfg.share_every
            gi = got_idx[g][0].cpu().numpy() if g in got_idx else None
            assert gi is not None
            q = R.decode_q_host(cfg, layer, s)
            lk = 0 if cfg.shared_kv else layer
            Kr = [R.host_rows(cfg.seed, R.tid(R.KIND_K, lk), (cfg.Hkv, cfg.D), gi[b], True, b, cfg.Tk_max)
                  for b in range(cfg.B)]
            Vr = [R.host_rows(cfg.seed, R.tid(R.KIND_V, lk), (cfg.Hkv, cfg.D), gi[b], True, b, cfg.Tk_max)
                  for b in range(cfg.B)]
            ref, _ = oracle.sparse_attention_decode(q, Kr, Vr)
            assert_close_attn(outs[layer].float().cpu().numpy(), ref, f"{cfg.name} step {s} layer {layer}")
    cache.close()
    inp.clear()
    outs.clear()
    del ws_idx
    _free()


def test_decode_32k_batch8_four_layers_share_one_index():
    _check_decode(R.DECODE_32K, steps=[0, 63], check_groups=[0], check_layers=[0, 3])


def test_decode_1m_28_layers_seven_groups():
    _check_decode(R.DECODE_1M, steps=[0, 15], check_groups=[0, 6], check_layers=[0, 27])


def test_decode_32k_one_cache_gathered_once():
    """The bench's one-cache workload (YOCO + CLSA): one gather per step, four
    layers over the compact rows, checked at full size."""
    _check_decode(R.YOCO_32K, steps=[0, 63], check_groups=[0], check_layers=[0, 3])


def test_decode_32k_batch8_sixteen_head_indexer():
    """The batch-8 decode step with the 16-head weighted indexer (the bench's
    multi-head workload): indices bit-exact, two layers' attention checked."""
    _check_decode(R.DECODE_32K_MH16, steps=[0, 63], check_groups=[0], check_layers=[0, 3])


def test_decode_32k_batch8_sixteen_head_fp8_indexer():
    """The 16-head decode step with the indexer's queries and keys in E4M3
    (the bench's fp8 workload): indices bit-exact against the oracle on the
    same codes, one layer's attention checked."""
    _check_decode(R.DECODE_32K_MH16_FP8, steps=[0, 63], check_groups=[0], check_layers=[0])


# ---------------------------------------------------------------- prefill

def _prefill_run(cfg):
    d = dev()
    inp = TI.prefill_inputs(cfg, d)
    cache = sa.IndexCache(cfg.n_layers, cfg.B, cfg.L, cfg.k, share_every=cfg.share_every, device=d)
    ws = torch.zeros(sa.lib().sa_index_score_topk_workspace(cfg.B, cfg.L, cfg.L, cfg.d, cfg.k),
                     dtype=torch.uint8, device=d)
    cache.begin_step()
    outs = {}
    for layer in range(cfg.n_layers):
        if cache.is_full(layer) == 1:
            g = layer // cfg.share_every
            cache.update(layer, inp["q_idx"][g], inp["k_idx"][g], ws=ws)
        idx, cnt, _ = cache.get_tensors(layer)
        outs[layer] = sa.sa_sparse_attn_prefill(inp["q"][layer], inp["K"][layer], inp["V"][layer], idx, cnt)
    torch.cuda.synchronize()
    idx, cnt, _ = cache.get_tensors(0)
    res = (idx.cpu().numpy(), cnt.cpu().numpy(), {l: o for l, o in outs.items()})
    cache.close()
    inp.clear()
    del ws
    _free()
    return res


def test_prefill_2k_full_parity():
    cfg = R.PREFILL_2K
    idx, cnt, outs = _prefill_run(cfg)
    host = R.prefill_host_inputs(cfg)
    ridx, rcnt = oracle.index_topk(host["q_idx"][0], host["k_idx"][0], cfg.L, 0, cfg.k)
    np.testing.assert_array_equal(cnt, rcnt)
    np.testing.assert_array_equal(idx, ridx)
    ref, _ = oracle.sparse_attention(host["q"][0], host["K"][0], host["V"][0], ridx, rcnt)
    assert_close_attn(outs[0].float().cpu().numpy(), ref, "prefill_2k")


def test_prefill_64k_needles_sampled_rows():
    """Indices bit-exact on the first and last row of every 2048-row batch
    the indexer runs (the bounded passes work batch by batch), on every
    needle row and on random rows; every needle retrieved; attention checked
    on sampled rows of all four layers (different rows per layer)."""
    cfg = R.PREFILL_64K
    idx, cnt, outs = _prefill_run(cfg)
    host = R.prefill_host_inputs(cfg, with_attention=False)
    qi, ki = host["q_idx"][0][0], host["k_idx"][0][0]
    pairs = R.needle_pairs(cfg)
    rng = np.random.default_rng(0)
    batch = 2048
    edges = [r for b0 in range(0, cfg.L, batch) for r in (b0, b0 + 1, b0 + batch - 1)]
    rows = sorted(set([255, 256, 8191, 8192, 8193] + edges + [t for _, t in pairs]
                      + list(rng.integers(0, cfg.L, 40))))
    s = oracle.index_scores(qi[rows], ki)
    for n_i, t in enumerate(rows):
        sel = oracle.topk_select(s[n_i, : t + 1], cfg.k)
        assert cnt[0, t] == sel.size
        np.testing.assert_array_equal(idx[0, t, : sel.size], sel)
        assert np.all(idx[0, t, sel.size:] == -1)
    for p, t in pairs:                       # every needle retrieved
        assert p in set(idx[0, t, : cnt[0, t]].tolist())
    # attention: 10 rows per layer, together spanning the batches
    for layer in range(cfg.n_layers):
        o = outs[layer].float().cpu().numpy()
        att_rows = rows[layer::max(1, len(rows) // 10)][:10]
        for t in att_rows:
            sel = idx[0, t, : cnt[0, t]]
            q = R.host_rows(cfg.seed, R.tid(R.KIND_Q, layer), (cfg.Hq, cfg.D), np.array([t]), True, 0, cfg.L)[0]
            Kr = R.host_rows(cfg.seed, R.tid(R.KIND_K, layer), (cfg.Hkv, cfg.D), sel, True, 0, cfg.L)
            Vr = R.host_rows(cfg.seed, R.tid(R.KIND_V, layer), (cfg.Hkv, cfg.D), sel, True, 0, cfg.L)
            ref, _ = oracle.attention_over_rows(q, Kr, Vr)
            assert_close_attn(o[0, t], ref, f"prefill_64k layer {layer} row {t}")


# -------------------------------------------------------------------- gist

def _check_gist(cfg):
    d = dev()
    inp = TI.gist_inputs(cfg, d)
    host_gk = ch.int_bf16(cfg.seed, R.tid(R.KIND_GIST_KEY), count=cfg.B * cfg.n_chunks * cfg.d) \
        .reshape(cfg.B, cfg.n_chunks, cfg.d)
    ng = cfg.n_chunks // cfg.group_size if cfg.group_size else 0
    host_mk = ch.int_bf16(cfg.seed, R.tid(R.KIND_META_KEY), count=cfg.B * ng * cfg.d).reshape(cfg.B, ng, cfg.d) \
        if cfg.group_size else None
    for s in (0, cfg.steps - 1):
        if cfg.group_size:
            rows, cnt = sa.sa_hier_gist_route_unfold(inp["q_route"][s], inp["meta_key"], inp["gist_key"],
                                                     cfg.chunk_len, cfg.group_size, cfg.k_groups, cfg.k_chunks,
                                                     inp["partial_len"][s])
        else:
            rows, cnt = sa.sa_gist_route_unfold(inp["q_route"][s], inp["gist_key"], cfg.chunk_len,
                                                cfg.k_chunks, inp["partial_len"][s])
        out = sa.sa_sparse_attn_decode(inp["q"][s], inp["K"], inp["V"], rows, cnt)
        torch.cuda.synchronize()
        rows, cnt, out = rows.cpu().numpy(), cnt.cpu().numpy(), out.float().cpu().numpy()
        qr = R.gist_q_route_host(cfg, s)
        q = R.gist_q_host(cfg, s)
        Kr, Vr = [], []
        for b in range(cfg.B):
            if cfg.group_size:
                rr = oracle.hier_gist_route_unfold(qr[b], host_mk[b], host_gk[b], cfg.group_size, cfg.chunk_len,
                                                   cfg.k_groups, cfg.k_chunks, s + 1)[0]
            else:
                rr, _ = oracle.gist_route_unfold(qr[b], host_gk[b], cfg.chunk_len, cfg.k_chunks, s + 1)
            assert cnt[b] == rr.size == cfg.k_chunks * 17 + s + 1
            np.testing.assert_array_equal(rows[b, : rr.size], rr)
            Kr.append(R.host_rows(cfg.seed, R.tid(R.KIND_K, 0), (cfg.Hkv, cfg.D), rr, True, b, cfg.Tk_max))
            Vr.append(R.host_rows(cfg.seed, R.tid(R.KIND_V, 0), (cfg.Hkv, cfg.D), rr, True, b, cfg.Tk_max))
        ref, _ = oracle.sparse_attention_decode(q, Kr, Vr)
        assert_close_attn(out, ref, f"{cfg.name} step {s}")
    inp.clear()
    _free()


def test_gist_decode_128k():
    _check_gist(R.GIST_128K)


def test_hier_gist_decode_128k_meta16():
    """The bench's two-level gist workload: 512 meta keys, 8 groups kept,
    64 of their 128 chunks unfolded, then attention."""
    _check_gist(R.HGIST_128K)
