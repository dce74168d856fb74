"""Host-side logic of bench.py (no GPU): the closed form it reports beside the
measured collapse fraction must be the oracle's, and the FLOP and throughput
conventions must be the ones the metric is quoted in."""
import math
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402


@pytest.mark.parametrize("S", [1.0, 16.0, 256.0, 448.0])
def test_reported_closed_form_is_the_oracles(S):
    for delta in range(0, 13):
        for k in (1, 2, 3, 4):
            assert math.isclose(bench.closed_form_F(delta, S, k),
                                oracle.underflow_fraction_closed(delta, S, k),
                                rel_tol=1e-8, abs_tol=1e-12), (delta, S, k)


def test_flop_convention():
    # causal: 2 B H N^2 d (visible pairs, diagonal excess ignored); non-causal 4 B H N^2 d
    assert bench.algorithmic_flops(1, 32, 32768, 128, True) == 2 * 32 * 32768 ** 2 * 128
    assert bench.algorithmic_flops(4, 32, 8192, 128, False) == 4 * 4 * 32 * 8192 ** 2 * 128
    # the prefill is 8.796 TFLOP per launch
    assert abs(bench.algorithmic_flops(1, 32, 32768, 128, True) / 1e12 - 8.796) < 1e-3


def test_job_throughput_uses_the_slowest_rank():
    # two ranks, 1 TFLOP each, the slower rank took 2 ms: 2 TFLOP / 2 ms = 1000 TFLOP/s
    assert math.isclose(bench.job_tflops(1e12, 2, 2.0), 1000.0)
