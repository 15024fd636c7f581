"""GPU test of the allocation-free prefill entry point (lightning_attn_fwd_noalloc).

That entry point exists for callers that cannot allocate device memory while
they run (a process whose device memory is partitioned up front by its own
allocator, or a latency-critical loop where an allocation could block or
fail).  It keeps the chunk-scan scratch in one fixed device array compiled
into the library instead of calling cudaMallocAsync.  This test calls it
through the C ABI twice in a row on different inputs -- the second call reuses
the array the first one left behind -- and checks each result against the
allocating entry point on the same inputs and against the float64 oracle, with
the bf16 tolerance used by the other prefill tests.  The file is named so that
pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_fwd_b200 import inputs as I
from long_context_fwd_b200 import ops
from parity import TOL_BF16, bf16_to_dev, f32_to_dev, rel, worst_head

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _case(seed, B, H, N, slopes):
    w = I.Workload(f"noalloc{seed}", B, H, N, 128, 128, "bf16", index=400 + seed)
    q, k, v = I.prefill_inputs(w)
    sl = np.asarray(slopes, np.float32)
    return (bf16_to_dev(q, DEV), bf16_to_dev(k, DEV), bf16_to_dev(v, DEV), f32_to_dev(sl, DEV),
            oracle.recurrent(q, k, v, sl))


@pytest.mark.parametrize("chunk", [0, 256])
def test_noalloc_matches_allocating_entry_point_twice(chunk):
    # B*H = 6 is below the SM count, so the sequences are split into chunks and
    # the chunk scan runs through the fixed scratch array.
    cases = [_case(1, 2, 3, 3000, [0.9, 0.05, 0.0]), _case(2, 1, 6, 2500, [0.3] * 5 + [0.0])]
    if chunk == 0:
        # more sequences than SMs: the balanced split hands sequences over
        # between CTAs through the same fixed array
        cases.append(_case(3, 1, 150, 1100, [0.5, 0.02, 0.0] * 50))
    for q, k, v, sl, want in cases:
        out_na = torch.full(q.shape[:3] + (128,), float("nan"), dtype=torch.float32, device=DEV)
        ops.fwd_noalloc(q, k, v, sl, out_na, chunk=chunk)
        ref = ops.fwd(q, k, v, sl, chunk=chunk)
        torch.cuda.synchronize()
        assert ops.device_status(reset=True) == 0
        a, b = out_na.cpu().numpy(), ref.cpu().numpy()
        assert np.isfinite(a).all()
        assert rel(a, b) <= TOL_BF16
        assert rel(a, want) <= TOL_BF16
        assert worst_head(a, want) <= TOL_BF16


def test_noalloc_rejects_scratch_beyond_limit():
    # 200 sequences split into 128-token chunks would need 25 MiB of chunk states.
    q = torch.zeros((1, 200, 256, 128), dtype=torch.bfloat16, device=DEV)
    sl = torch.zeros(200, dtype=torch.float32, device=DEV)
    with pytest.raises(ops.LightningAttnError) as err:
        ops.fwd_noalloc(q, q, q, sl, chunk=128)
    assert err.value.code == 7  # LA_ERR_WORKSPACE
