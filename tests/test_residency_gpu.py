"""GPU: the static work splits under a capped grid and beside another launch.

The hand-over and the split scan have CTAs that wait for states published by
other CTAs of the same launch, so those launches are cooperative (all CTAs
resident, or the launch fails).  These tests run both splits

* on grids smaller than the SM count (lightning_attn_set_cta_limit), which
  the schedule plans for -- the results must still match the float64 oracle;
* as two prefills issued on two streams with no ordering between them, each
  of which alone fills the GPU -- neither may be left waiting for CTAs that
  cannot start (device-side waits are bounded, so a failure here reads as a
  time-out in the device status word, not a hang).
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


def _case(seed, B, H, N):
    w = I.Workload(f"resid{seed}", B, H, N, 128, 128, "bf16", index=1300 + seed)
    q, k, v = I.prefill_inputs(w)
    sl = I.alibi_slopes(H)
    sl[7::8] = 0.0
    return q, k, v, sl


@pytest.fixture
def cta_limit():
    prev = ops.set_cta_limit(0)
    yield ops.set_cta_limit
    ops.set_cta_limit(prev)


@pytest.mark.parametrize("B,H,N,ctas,mode", [
    (1, 64, 3000, 100, 2),   # split scan on 100 CTAs
    (1, 64, 2500, 37, 1),    # 64 sequences >= 37 CTAs: hand-over
    (2, 80, 1100, 100, 1),   # hand-over on 100 CTAs
    (1, 9, 20000, 60, 2),    # split scan, long chains (60 / 9 CTAs per sequence)
    (1, 4, 9000, 16, 2),     # split scan on 16 CTAs
    (1, 2, 9000, 40, 0),     # chunk scan (fewer than CTAs / 8 sequences)
])
def test_capped_grid_matches_oracle(B, H, N, ctas, mode, cta_limit):
    assert ops.fwd_plan(B, H, N, 0, ctas)[0]["mode"] == mode
    q, k, v, sl = _case(ctas + N, B, H, N)
    cta_limit(ctas)
    st = torch.zeros((B, H, 128, 128), dtype=torch.float32, device=DEV)
    out = ops.fwd(bf16_to_dev(q, DEV), bf16_to_dev(k, DEV), bf16_to_dev(v, DEV),
                  f32_to_dev(sl, DEV), final_state=st)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    ref, sref = oracle.recurrent(q, k, v, sl, return_state=True)
    got = out.cpu().numpy()
    assert rel(got, ref) <= TOL_BF16
    assert worst_head(got, ref) <= TOL_BF16
    assert rel(st.cpu().numpy(), sref) <= TOL_BF16


@pytest.mark.parametrize("B,H,N", [(1, 64, 8192), (2, 80, 1100)])
def test_two_streams_without_ordering(B, H, N):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert ops.fwd_plan(B, H, N, 0, sms)[0]["mode"] in (1, 2)
    cases = [_case(s, B, H, N) for s in (1, 2)]
    dev = [tuple(bf16_to_dev(x, DEV) for x in c[:3]) + (f32_to_dev(c[3], DEV),) for c in cases]
    outs = [torch.empty((B, H, N, 128), dtype=torch.float32, device=DEV) for _ in cases]
    streams = [torch.cuda.Stream(device=DEV) for _ in cases]
    torch.cuda.synchronize()
    for rep in range(3):
        for (q, k, v, sl), o, s in zip(dev, outs, streams):
            ops.fwd(q, k, v, sl, o, stream=s)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    for (q, k, v, sl), o in zip(cases, outs):
        ref = oracle.recurrent(q, k, v, sl)
        assert rel(o.cpu().numpy(), ref) <= TOL_BF16


@pytest.mark.parametrize("entry", ["fused", "anticausal", "noalloc"])
def test_other_entries_on_a_capped_grid(entry, cta_limit):
    # the fused layer, the reverse-time operator and the allocation-free entry
    # plan their splits for the capped grid too (split scan at 40 CTAs)
    B, H, N = 1, 24, 3000
    assert ops.fwd_plan(B, H, N, 0, 40)[0]["mode"] == 2
    q, k, v, sl = _case(7, B, H, N)
    cta_limit(40)
    tq, tk, tv = (bf16_to_dev(x, DEV) for x in (q, k, v))
    ts = f32_to_dev(sl, DEV)
    if entry == "fused":
        g = I.f32_to_bf16_bits(np.random.default_rng(3).standard_normal(q.shape).astype(np.float32))
        w = np.ones((H, 128), np.float32)
        got = ops.fwd_fused(tq, tk, tv, bf16_to_dev(g, DEV), ts, f32_to_dev(w, DEV), 1e-6)
        ref = oracle.fused_layer(q, k, v, g, sl, w, 1e-6)
    elif entry == "anticausal":
        got = ops.fwd_anticausal(tq, tk, tv, ts)
        ref = oracle.recurrent_anticausal(q, k, v, sl)
    else:
        got = ops.fwd_noalloc(tq, tk, tv, ts)
        ref = oracle.recurrent(q, k, v, sl)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    got = got.float().cpu().numpy()
    assert rel(got, ref) <= TOL_BF16
    assert worst_head(got, ref) <= TOL_BF16


@pytest.mark.parametrize("ctas", [1, 3, 37])
def test_backward_on_capped_grid(ctas, cta_limit):
    """The backward pass on grids of 1 CTA (dk and dv then take a launch each),
    3 CTAs (one pair: dk and dv side by side) and 37 (18 pairs)."""
    B, H, N = 1, 64, 1300
    cta_limit(ctas)
    w = I.Workload("capbwd", B, H, N, 128, 128, "bf16", index=880 + ctas)
    q, k, v = I.prefill_inputs(w)
    g = I.f32_to_bf16_bits(np.random.default_rng(ctas).standard_normal((B, H, N, 128))
                           .astype(np.float32))
    sl = I.alibi_slopes(H)
    dq, dk, dv = ops.bwd(*(bf16_to_dev(x, DEV) for x in (q, k, v, g)), f32_to_dev(sl, DEV))
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    refs = oracle.backward(q, k, v, g, sl)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        a = got.cpu().numpy()
        assert rel(a, ref) <= TOL_BF16, name
        assert worst_head(a, ref) <= TOL_BF16, name
