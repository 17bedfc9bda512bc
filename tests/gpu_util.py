"""Helpers shared by the GPU tests (input plumbing and tolerance checks)."""
import numpy as np
import torch

# Attention tolerance (bf16 in, fp32 accumulate, bf16 out) against the fp64
# oracle: max-abs 2e-2 and mean-abs 2e-3.
ATOL_MAX = 2e-2
ATOL_MEAN = 2e-3


def dev():
    return torch.device("cuda:0")


def to_dev(bits):
    a = np.ascontiguousarray(bits).view(np.int16)
    return torch.from_numpy(a).to(dev()).view(torch.bfloat16)


def i32(x):
    return torch.as_tensor(np.asarray(x, dtype=np.int32), device=dev())


def bits_of(t):
    """bf16 tensor -> host uint16 bit patterns."""
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def assert_close_attn(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= ATOL_MAX, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= ATOL_MEAN, f"{what}: mean abs err {err.mean():.3e}"


def assert_lse_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), f"{what}: -inf pattern differs"
    fin = ~np.isneginf(ref)
    if fin.any():
        d = np.abs(got[fin] - ref[fin])
        assert d.max() <= 1e-3 * max(1.0, np.abs(ref[fin]).max()), f"{what}: lse err {d.max()}"
