"""The benchmark's roofline arithmetic (CPU only): the bound is whichever of
the algorithmic bytes at the HBM copy bandwidth and the algorithmic flops at
the dense bf16 tensor peak takes longer, and the fraction is that time over
the measured launch time."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from long_context_fwd_b200 import inputs as I  # noqa: E402


def test_memory_bound_launch():
    # 10 GB and 1 TFLOP on a 5000 GB/s, 1000 TFLOP/s part: 2 ms vs 1 ms -> HBM
    r = bench.roofline(10e9, 1e12, 4.0, 5000.0, 1000.0)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(2500.0)
    assert r["frac"] == pytest.approx(0.5)
    assert r["hbm_bound_ms"] == pytest.approx(2.0) and r["tensor_bound_ms"] == pytest.approx(1.0)


def test_compute_bound_launch():
    # 1 GB and 3 TFLOP: 0.2 ms vs 3 ms -> tensor
    r = bench.roofline(1e9, 3e12, 6.0, 5000.0, 1000.0)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(500.0)
    assert r["frac"] == pytest.approx(0.5)


def test_prefill_workloads_are_memory_bound_on_b200():
    # 102 flop/B at 128-token blocks, below the 1683 / 6543 ~ 257 flop/B ridge
    for w in (I.PREFILL_8K, I.PREFILL_32K, I.PREFILL_1M):
        assert bench.prefill_bytes(w) == w.B * w.H * w.N * 1280
        r = bench.roofline(bench.prefill_bytes(w), bench.prefill_flops(w), 1.0, 6543.4, 1683.0)
        assert r["bound"] == "hbm"
