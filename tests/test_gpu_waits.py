"""Bounded waits on the GPU, without a fault.

Every pipeline kernel of the library waits on mbarrier phases with a poll
limit, so a wait that can never complete gives up, records an error code and
lets the kernel wind down instead of hanging the GPU.  The library's probe
kernel makes one wait run out on purpose (a barrier phase nothing completes,
a short poll limit) and checks that a wait that does complete still
succeeds."""
import pytest
import torch

from shared_top_routing_b200 import sa

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit", [1, 64, 4096])
def test_a_wait_that_cannot_complete_gives_up_with_its_code(limit):
    err = sa.sa_self_test_bounded_wait(limit)
    torch.cuda.synchronize()
    assert err.cpu().tolist() == [77, 0, 0, 1, 1]


def test_bad_arguments_are_refused_on_the_host():
    st = sa.lib().sa_self_test_bounded_wait(None, 16, None)
    assert st == sa.SA_ERR_INVALID_ARG


# ---------------------------------------------------------------- sentinel
#
# A wait in the indexer's kernels that gives up leaves a nonzero error word
# at the start of the call's workspace.  The tests below write that word
# themselves (as a wait that ran out would), so no wait has to fail: every
# row must then come out as the failure sentinel, and a zero-filled
# workspace must give the exact selection again.

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from gen import counter_hash as ch  # noqa: E402
from tests.gpu_util import dev, i32, to_dev  # noqa: E402


def _ws(nbytes):
    return torch.zeros(max(256, nbytes), dtype=torch.uint8, device=dev())


def _set_err(ws, code):
    ws[:4].view(torch.int32)[0] = code


@pytest.mark.parametrize("B,Tq,T,d,k", [(3, 1, 20000, 128, 2048),    # decode, streamed row scan
                                        (2, 1, 3000, 64, 256),       # decode, whole row in shared memory
                                        (1, 300, 300, 64, 64),       # prefill, key slab
                                        (1, 200, 9000, 64, 512)])    # prefill, bounded passes
def test_indexer_error_word_gives_the_sentinel(B, Tq, T, d, k):
    qi = ch.int_bf16(71, 1, count=B * Tq * d).reshape(B, Tq, d)
    ki = ch.int_bf16(71, 2, count=B * T * d).reshape(B, T, d)
    q_pos0 = T - Tq
    ws = _ws(sa.lib().sa_index_score_topk_workspace(B, Tq, T, d, k))
    ref_idx, ref_cnt = oracle.index_topk(qi, ki, T, q_pos0, k)
    for code in (0, 31, 0):
        _set_err(ws, code)
        idx, cnt, sc = sa.sa_index_score_topk(to_dev(qi), to_dev(ki), k, Tk=T, q_pos0=q_pos0, ws=ws,
                                              with_scores=True)
        torch.cuda.synchronize()
        if code == 0:
            np.testing.assert_array_equal(cnt.cpu().numpy(), ref_cnt)
            np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
            assert sa.sa_workspace_status(ws) == sa.SA_OK
        else:
            assert (cnt.cpu().numpy() == 0).all()
            assert (idx.cpu().numpy() == -1).all()
            assert np.isneginf(sc.cpu().numpy()).all()
            assert ws[:4].view(torch.int32)[0].item() == code   # the word is left for the caller
            # ... and the host reads it as a timed-out wait, naming the code
            assert sa.sa_workspace_status(ws) == sa.SA_ERR_TIMEOUT
            assert str(code) in sa.last_error()


def test_gist_error_word_gives_the_sentinel():
    B, n_chunks, chunk_len, d, kc = 2, 9000, 16, 128, 64
    qr = ch.int_bf16(72, 1, count=B * d).reshape(B, d)
    gk = ch.int_bf16(72, 2, count=B * n_chunks * d).reshape(B, n_chunks, d)
    part = i32([5, 16])
    ws = _ws(sa.lib().sa_gist_route_unfold_workspace(B, n_chunks, d, kc))
    for code in (0, 31, 0):
        _set_err(ws, code)
        rows, cnt = sa.sa_gist_route_unfold(to_dev(qr), to_dev(gk), chunk_len, kc, part, ws=ws)
        torch.cuda.synchronize()
        rows, cnt = rows.cpu().numpy(), cnt.cpu().numpy()
        for b, p in enumerate((5, 16)):
            if code == 0:
                rr, _ = oracle.gist_route_unfold(qr[b], gk[b], chunk_len, kc, p)
                assert cnt[b] == rr.size
                np.testing.assert_array_equal(rows[b, : rr.size], rr)
            else:
                assert cnt[b] == 0 and (rows[b] == -1).all()
        assert sa.sa_workspace_status(ws) == (sa.SA_OK if code == 0 else sa.SA_ERR_TIMEOUT)
