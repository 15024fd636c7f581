"""GPU parity of the anti-causal prefill and the backward pass against the oracle.

lightning_attn_fwd_anticausal runs the tensor-core kernel in reversed time;
lightning_attn_bwd composes dq (causal on (dout, v, k)) with dk and dv
(anti-causal on (v, dout, q) and (k, q, dout)), the last two in one paired
launch when D == E (alternate CTAs, each role planned for half the grid) and
in two launches otherwise.  Both are compared element by
element with the float64 oracle (its anti-causal sum and its gradients of
L = sum dout . o, pinned in tests/test_oracle_backward.py) on the same seeded
bf16 inputs, across the kernel's work splits (whole sequences, explicit
chunks, split scan, hand-over), ragged lengths and 64-wide heads.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_fwd_b200 import inputs as I
from long_context_fwd_b200 import ops
from parity import (TOL_BF16, bf16_to_dev, f32_to_dev, fill_heads_from_host, host_workers, rel,
                    worst_head)

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _case(B, H, N, D, E, seed):
    w = I.Workload(f"bwd{seed}", B, H, N, D, E, "bf16", index=700 + seed)
    q, k, v = I.prefill_inputs(w)
    g = I.f32_to_bf16_bits(np.random.default_rng(900 + seed).standard_normal((B, H, N, E))
                           .astype(np.float32))
    sl = I.alibi_slopes(H)
    sl[2::5] = 0.0
    return q, k, v, g, sl


ANTI_CASES = [
    # B, H, N, D, E, chunk
    (2, 3, 777, 128, 128, 0),
    (1, 4, 3000, 128, 128, 512),
    (1, 64, 2500, 128, 128, 0),
    (2, 80, 1100, 128, 128, 0),
    (1, 2, 129, 128, 128, 0),
    (1, 1, 1, 128, 128, 0),
    (1, 3, 1000, 64, 128, 0),
    (1, 2, 640, 128, 64, 256),
]


@pytest.mark.parametrize("B,H,N,D,E,chunk", ANTI_CASES)
def test_anticausal_parity(B, H, N, D, E, chunk):
    q, k, v, _, sl = _case(B, H, N, D, E, seed=N % 97 + H + D // 64)
    out = ops.fwd_anticausal(bf16_to_dev(q, DEV), bf16_to_dev(k, DEV), bf16_to_dev(v, DEV),
                             f32_to_dev(sl, DEV), chunk=chunk)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    got = out.cpu().numpy()
    ref = oracle.recurrent_anticausal(q, k, v, sl)
    assert np.isfinite(got).all()
    assert rel(got, ref) <= TOL_BF16
    assert worst_head(got, ref) <= TOL_BF16


@pytest.mark.parametrize("B,H,N,chunk", [(1, 3, 1500, 0), (1, 3, 1500, 256), (1, 64, 1200, 0)])
def test_anticausal_initial_and_final_state(B, H, N, chunk):
    q, k, v, _, sl = _case(B, H, N, 128, 128, seed=31 + chunk // 128 + H)
    s0 = (np.random.default_rng(8).standard_normal((B, H, 128, 128)) * 0.02).astype(np.float32)
    fin = torch.zeros((B, H, 128, 128), dtype=torch.float32, device=DEV)
    out = ops.fwd_anticausal(bf16_to_dev(q, DEV), bf16_to_dev(k, DEV), bf16_to_dev(v, DEV),
                             f32_to_dev(sl, DEV), init_state=f32_to_dev(s0, DEV),
                             final_state=fin, chunk=chunk)
    torch.cuda.synchronize()
    ref, sref = oracle.recurrent_anticausal(q, k, v, sl, s0=s0.astype(np.float64),
                                            return_state=True)
    assert rel(out.cpu().numpy(), ref) <= TOL_BF16
    assert rel(fin.cpu().numpy(), sref) <= TOL_BF16


BWD_CASES = [
    # B, H, N, D, E
    (1, 2, 1000, 128, 128),
    (2, 3, 777, 128, 128),
    (1, 64, 2000, 128, 128),
    (2, 80, 600, 128, 128),
    (1, 4, 900, 64, 128),
    (1, 3, 513, 128, 64),
]


@pytest.mark.parametrize("B,H,N,D,E", BWD_CASES)
def test_backward_parity(B, H, N, D, E):
    q, k, v, g, sl = _case(B, H, N, D, E, seed=50 + H + N % 31)
    dq, dk, dv = ops.bwd(*(bf16_to_dev(x, DEV) for x in (q, k, v, g)), f32_to_dev(sl, DEV))
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    refs = oracle.backward(q, k, v, g, sl)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        a = got.cpu().numpy()
        assert np.isfinite(a).all(), name
        assert rel(a, ref) <= TOL_BF16, name
        assert worst_head(a, ref) <= TOL_BF16, name


def test_backward_adjoint_identity_on_device():
    """sum q . dq = sum k . dk = sum v . dv = sum dout . o (o linear in each input)."""
    B, H, N = 1, 4, 1024
    q, k, v, g, sl = _case(B, H, N, 128, 128, seed=77)
    dq_, dk_, dv_, dg_ = (bf16_to_dev(x, DEV) for x in (q, k, v, g))
    ds = f32_to_dev(sl, DEV)
    o = ops.fwd(dq_, dk_, dv_, ds)
    dq, dk, dv = ops.bwd(dq_, dk_, dv_, dg_, ds)
    torch.cuda.synchronize()
    L = (dg_.double() * o.double()).sum(dim=(2, 3))
    for x, dx in ((dq_, dq), (dk_, dk), (dv_, dv)):
        lx = (x.double() * dx.double()).sum(dim=(2, 3))
        assert torch.allclose(lx, L, rtol=2e-2, atol=1e-3 * float(L.abs().max()))


@pytest.mark.parametrize("B,H,N,mode", [
    (2, 80, 600, 1),    # hand-over
    (1, 64, 2000, 2),   # split scan
    (1, 4, 3000, 0),    # chunk scan: each role draws its own tickets
    (1, 2, 1000, 0),    # whole sequences
    (1, 1, 1, 0),       # one token
])
def test_backward_paired_launch_every_split(B, H, N, mode):
    """dk and dv from the paired launch, whose roles each plan for half the
    CTAs, in every work split of that plan."""
    sms = torch.cuda.get_device_properties(DEV).multi_processor_count
    assert ops.fwd_plan(B, H, N, 0, sms // 2)[0]["mode"] == mode
    q, k, v, g, sl = _case(B, H, N, 128, 128, seed=300 + H + N % 29)
    dq, dk, dv = ops.bwd(*(bf16_to_dev(x, DEV) for x in (q, k, v, g)), f32_to_dev(sl, DEV))
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    refs = oracle.backward(q, k, v, g, sl)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        a = got.cpu().numpy()
        assert np.isfinite(a).all(), name
        assert rel(a, ref) <= TOL_BF16, name
        assert worst_head(a, ref) <= TOL_BF16, name


def test_backward_32k_workload_shapes_sampled_sequences():
    """The backward pass on the benchmark's shapes (B=4, H=64, N=32768, lambda = 0
    on heads h % 8 == 7; the dq launch and the paired dk/dv launch as the
    benchmark times them), every input drawn on the host: dq, dk and dv of 12
    sequences -- four lambda = 0 heads and eight decaying ones in the first and
    last batch rows -- in full against the oracle's gradients."""
    w = I.PREFILL_32K
    sl = I.slopes_for(w)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    checked = {(b, h) for b in (0, 3) for h in (7, 15, 0, 20, 41, 62)}
    assert sum(sl[h] == 0.0 for _, h in checked) == 4

    def draw(b, h):
        dout = np.random.default_rng(5000 + b * w.H + h).standard_normal((w.N, w.E))
        return (*I.head_inputs(w, b, h), I.f32_to_bf16_bits(dout.astype(np.float32)))

    def reference(b, h, hq, hk, hv, hg):
        if (b, h) not in checked:
            return None
        grads = oracle.backward(hq[None, None], hk[None, None], hv[None, None], hg[None, None],
                                sl[h:h + 1], threads=1)
        return [x[0, 0] for x in grads]

    q, k, v, g = (torch.empty((w.B, w.H, w.N, 128), dtype=torch.bfloat16, device=DEV)
                  for _ in range(4))
    refs = fill_heads_from_host(draw, (q, k, v, g), heads, reference, host_workers(0.3e9))
    dq, dk, dv = ops.bwd(q, k, v, g, f32_to_dev(sl, DEV))
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    del q, k, v, g
    for (b, h) in sorted(checked):
        for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs[(b, h)]):
            a = got[b, h].cpu().numpy()
            assert np.isfinite(a).all(), (b, h, name)
            assert rel(a, ref) <= TOL_BF16, (b, h, name)
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()
