"""The CPU oracle against its pins (no GPU needed)."""
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def o():
    return oracle.default()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(o, pin):
    pin(o)


def test_thread_count_does_not_change_results(o):
    import numpy as np
    import workloads
    p = workloads.dense_problem(9, 300, 512, seed=3)
    n0 = o.num_threads()
    try:
        o.set_num_threads(1)
        d1, a1 = o.gemm_nt(p.a, p.sfa, p.b, p.sfb)
        o.set_num_threads(max(2, n0))
        d2, a2 = o.gemm_nt(p.a, p.sfa, p.b, p.sfb)
    finally:
        o.set_num_threads(n0)
    assert np.array_equal(d1, d2) and np.array_equal(a1, a2)


def test_bad_arguments_are_rejected(o):
    import numpy as np
    a = np.zeros((2, 100), np.uint8)
    with pytest.raises(AssertionError):
        o.gemm_nt(a, np.ones((2, 1), np.float32), a, np.ones((1, 1), np.float32))
    m_idx = np.array([0, 5], np.int32)              # expert 5 does not exist
    with pytest.raises(ValueError):
        o.grouped_contiguous(np.zeros((2, 128), np.uint8), np.ones((2, 1), np.float32),
                             np.zeros((2, 16, 128), np.uint8), np.ones((2, 1, 1), np.float32), m_idx)
