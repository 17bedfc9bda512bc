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
