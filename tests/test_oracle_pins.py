"""The CPU oracle against facts other than its own code (shapes printed on the
pages, torch float64 library routines, brute force, closed forms, invariants)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(lib, pin):
    name, ok, detail = pin(lib)
    assert ok, f"{name}: {detail}"


def test_thread_count_positive(lib):
    assert oracle.num_threads(lib) >= 1


def test_domain_errors(lib):
    import numpy as np
    x = np.zeros((1, 1, 2, 5), np.float32)
    w = np.zeros((1, 1, 3, 3), np.float32)
    b = np.zeros((1,), np.float32)
    with pytest.raises(ValueError):
        oracle.conv2d_pool_sigmoid_sum(x, w, b, 2, lib)  # H < 3
    with pytest.raises(ValueError):
        oracle.conv1d_out_len(4, 9, 1, 0, lib)  # T + 2p < K
    with pytest.raises(ValueError):
        oracle.conv1d_out_len(4, 3, 0, 0, lib)  # stride 0
