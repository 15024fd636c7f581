"""The benchmark's measured-traffic figure (CPU only): the DRAM bytes of the
committed ncu summary of the prefill kernel, scaled per (b, h, token), taken
from the capture of the same way of splitting the work, and withheld when the
kernel source no longer matches the capture."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from long_context_fwd_b200 import inputs as I  # noqa: E402


def _fields():
    out = {}
    with open(bench.PROFILE) as f:
        for line in f:
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                out[k.strip()] = v.strip().strip("`")
    return out


@pytest.fixture
def current(monkeypatch):
    """The summary taken as matching the kernel source (the scaling is under test)."""
    monkeypatch.setattr(bench, "kernel_hash", lambda: _fields()["kernel_sha"])


def test_handover_workload_uses_the_whole_sequence_capture(current):
    f = _fields()
    w = I.PREFILL_32K
    want = float(f["dram_bytes_per_launch"]) / float(f["token_heads_per_launch"]) * w.B * w.H * w.N
    assert bench.measured_traffic(w, 148) == pytest.approx(want, rel=1e-12)


@pytest.mark.parametrize("w", [I.PREFILL_8K, I.PREFILL_1M])
def test_split_scan_workloads_use_the_split_capture(current, w):
    f = _fields()
    want = (float(f["split_dram_bytes_per_launch"]) / float(f["split_token_heads_per_launch"]) *
            w.B * w.H * w.N)
    assert bench.measured_traffic(w, 148) == pytest.approx(want, rel=1e-12)
    # ~1546 B per token-head: q, k, v, out plus the local-state pass
    assert 1400 < bench.measured_traffic(w, 148) / (w.B * w.H * w.N) < 1700


def test_other_split_counts_and_stale_captures_give_none(current, monkeypatch):
    # 32 sequences split differently from the 64-sequence capture
    assert bench.measured_traffic(I.Workload("x", 1, 32, 65536, 128, 128, "bf16", index=950), 148) is None
    monkeypatch.setattr(bench, "kernel_hash", lambda: "0" * 16)
    assert bench.measured_traffic(I.PREFILL_32K, 148) is None


def test_kernel_hash_ignores_comments_only():
    code = "int f(int x) {  // doubles\n  /* a block\n comment */ return 2 * x;\n}\n\n"
    assert bench._code_only(code) == "int f(int x) {\n   return 2 * x;\n}"
    assert bench._code_only(code.replace("doubles", "twice")) == bench._code_only(code)
    assert bench._code_only(code.replace("2 * x", "3 * x")) != bench._code_only(code)
