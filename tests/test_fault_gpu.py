"""Failure detection on the GPU without a fault: a chunked prefill in which no
chunk 0 is ever processed, so every chunk-1 item waits on a publication flag
that nothing sets.  The bounded waits give up after 100 ms, the kernel reports
LA_ERR_TIMEOUT through the device status word and returns, and the context
stays usable for a normal, correct call right after."""
import time

import numpy as np
import pytest
import torch

import oracle
from long_context_fwd_b200 import inputs as I
from long_context_fwd_b200 import ops
from parity import TOL_BF16, bf16_to_dev, f32_to_dev, rel

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def test_scan_stall_times_out_and_context_survives():
    w = I.Workload("stall", 1, 3, 1024, 128, 128, "bf16", index=600)
    q, k, v = I.prefill_inputs(w)
    sl = np.array([0.5, 0.1, 0.0], np.float32)
    tq, tk, tv, ts = (bf16_to_dev(q, DEV), bf16_to_dev(k, DEV), bf16_to_dev(v, DEV),
                      f32_to_dev(sl, DEV))
    out = torch.zeros((1, 3, 1024, 128), dtype=torch.float32, device=DEV)
    assert ops.device_status(reset=True) == 0
    t0 = time.time()
    ops.fault_test_scan_stall(tq, tk, tv, ts, out, chunk=256, wait_limit_ms=100)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert ops.device_status(reset=True) == 6  # LA_ERR_TIMEOUT
    assert elapsed < 10.0
    assert ops.device_status(reset=True) == 0  # reset took effect
    got = ops.fwd(tq, tk, tv, ts, chunk=256)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    assert rel(got.cpu().numpy(), oracle.recurrent(q, k, v, sl)) <= TOL_BF16
