"""GPU parity of the strided prefill entry point (lightning_attn_fwd_strided).

q, k, v and out are laid out as a model produces and consumes them --
token-major [B][N][H][D], or slices of one fused [B][N][3][H][D] projection
output -- and the result is compared element by element with the float64
oracle on the head-major copies of the same seeded inputs.  Each case runs
through one of the kernel's work splits: whole sequences, the balanced
hand-over (B*H >= SMs), the split scan (fewer sequences than SMs) and the
explicit chunk scan.
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


def _case(B, H, N, seed, D=128, E=128):
    w = I.Workload(f"layout{seed}", B, H, N, D, E, "bf16", index=500 + seed)
    q, k, v = I.prefill_inputs(w)
    sl = I.alibi_slopes(H)
    sl[::3] = 0.0
    return q, k, v, sl


def _token_major(x_bits, dtype=torch.bfloat16):
    """Head-major host array [B,H,N,D] -> device token-major [B,N,H,D] and its
    [B,H,N,D] view."""
    t = bf16_to_dev(x_bits, DEV) if dtype == torch.bfloat16 else f32_to_dev(x_bits, DEV)
    tm = t.permute(0, 2, 1, 3).contiguous()
    return tm, tm.permute(0, 2, 1, 3)


LAYOUT_CASES = [
    # B, H, N, chunk: whole sequences, split scan, hand-over, chunk scan, ragged
    (2, 3, 777, 0),
    (1, 64, 2500, 0),
    (2, 80, 1100, 0),
    (1, 4, 3000, 512),
    (1, 2, 129, 0),
]


@pytest.mark.parametrize("B,H,N,chunk", LAYOUT_CASES)
def test_token_major_inputs_and_output(B, H, N, chunk):
    q, k, v, sl = _case(B, H, N, seed=N % 89 + H)
    _, qv = _token_major(q)
    _, kv = _token_major(k)
    _, vv = _token_major(v)
    out_tm = torch.full((B, N, H, 128), float("nan"), dtype=torch.float32, device=DEV)
    ops.fwd_strided(qv, kv, vv, f32_to_dev(sl, DEV), out_tm.permute(0, 2, 1, 3), chunk=chunk)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    got = out_tm.permute(0, 2, 1, 3).cpu().numpy()
    ref = oracle.recurrent(q, k, v, sl)
    assert np.isfinite(got).all()
    assert rel(got, ref) <= TOL_BF16
    assert worst_head(got, ref) <= TOL_BF16


@pytest.mark.parametrize("B,H,N", [(2, 5, 1000), (1, 64, 2048)])
def test_fused_qkv_projection_buffer(B, H, N):
    """q, k, v as slices of one [B][N][3][H][D] buffer; head-major fp32 out."""
    q, k, v, sl = _case(B, H, N, seed=7 + H)
    buf = torch.empty((B, N, 3, H, 128), dtype=torch.bfloat16, device=DEV)
    for i, x in enumerate((q, k, v)):
        buf[:, :, i].copy_(bf16_to_dev(x, DEV).permute(0, 2, 1, 3))
    views = [buf[:, :, i].permute(0, 2, 1, 3) for i in range(3)]
    assert views[0].stride() == (N * 3 * H * 128, 128, 3 * H * 128, 1)
    out = torch.empty((B, H, N, 128), dtype=torch.float32, device=DEV)
    ops.fwd_strided(*views, f32_to_dev(sl, DEV), out)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    ref = oracle.recurrent(q, k, v, sl)
    assert rel(out.cpu().numpy(), ref) <= TOL_BF16


def test_strided_matches_contiguous_bitwise():
    """Head-major strides through the strided entry point give the same bits as
    the contiguous entry point (same kernel, same work split)."""
    q, k, v, sl = _case(1, 6, 3000, seed=3)
    dq, dk, dv = (bf16_to_dev(x, DEV) for x in (q, k, v))
    ds = f32_to_dev(sl, DEV)
    a = ops.fwd(dq, dk, dv, ds)
    b = torch.empty_like(a)
    ops.fwd_strided(dq, dk, dv, ds, b)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_token_major_initial_and_final_state():
    B, H, N = 1, 64, 1500
    q, k, v, sl = _case(B, H, N, seed=11)
    s0 = (np.random.default_rng(4).standard_normal((B, H, 128, 128)) * 0.02).astype(np.float32)
    fin = torch.zeros((B, H, 128, 128), dtype=torch.float32, device=DEV)
    _, qv = _token_major(q)
    _, kv = _token_major(k)
    _, vv = _token_major(v)
    out_tm = torch.empty((B, N, H, 128), dtype=torch.float32, device=DEV)
    ops.fwd_strided(qv, kv, vv, f32_to_dev(sl, DEV), out_tm.permute(0, 2, 1, 3),
                    init_state=f32_to_dev(s0, DEV), final_state=fin)
    torch.cuda.synchronize()
    ref, sref = oracle.recurrent(q, k, v, sl, s0=s0.astype(np.float64), return_state=True)
    assert rel(out_tm.permute(0, 2, 1, 3).cpu().numpy(), ref) <= TOL_BF16
    assert rel(fin.cpu().numpy(), sref) <= TOL_BF16


def test_token_major_with_64_wide_q_k():
    B, H, N, D, E = 1, 64, 2000, 64, 128
    q, k, v, sl = _case(B, H, N, seed=13, D=D, E=E)
    _, qv = _token_major(q)
    _, kv = _token_major(k)
    _, vv = _token_major(v)
    out_tm = torch.empty((B, N, H, E), dtype=torch.float32, device=DEV)
    ops.fwd_strided(qv, kv, vv, f32_to_dev(sl, DEV), out_tm.permute(0, 2, 1, 3))
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    ref = oracle.recurrent(q, k, v, sl)
    assert rel(out_tm.permute(0, 2, 1, 3).cpu().numpy(), ref) <= TOL_BF16
