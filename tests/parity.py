"""Shared helpers for the GPU-vs-oracle parity tests."""
import numpy as np
import pytest
import torch

# allclose semantics with atol = rtol = 1e-4 against the double-precision
# oracle: the tolerance the l2_p7 trace states for fp32 outputs
# ("atol=rtol=1e-4") and the one both ops are held to.
ATOL = 1e-4
RTOL = 1e-4


def assert_close(got, ref, what="", atol=ATOL, rtol=RTOL):
    got = np.asarray(got.detach().cpu().double() if isinstance(got, torch.Tensor) else got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    if got.size == 0:
        return
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    lim = atol + rtol * np.abs(ref)
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        pytest.fail(f"{what}: {bad.sum()} of {got.size} outside atol=rtol=1e-4; worst at {i}: "
                    f"gpu {got[i]!r} oracle {ref[i]!r} (|err| {err[i]:.3e})")


def sample_indices(shape, n, seed, corners=True):
    """n random multi-indices into `shape`, plus every corner (first/last along each axis)."""
    r = np.random.default_rng(seed)
    idx = np.stack([r.integers(0, s, n) for s in shape], axis=1)
    if corners:
        import itertools
        cs = np.array(list(itertools.product(*[(0, s - 1) for s in shape])))
        idx = np.concatenate([cs, idx], axis=0)
    return idx.astype(np.int64)


requires_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
