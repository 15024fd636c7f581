"""GPU parity of the model-facing fused layer against the float64 oracle.

lightning_attn_fwd_fused_ex takes the raw projections in the layouts a QKV
projection writes (token-major, or slices of one fused buffer) and hands the
recurrent state in and out; lightning_attn_decode_fused continues a sequence
one token at a time from that state.  Compared element by element (bf16
outputs upcast) with oracle.fused_layer -- SiLU on q, k, v, the operator,
per-head RMSNorm, weight and sigmoid gate -- whose state in/out is pinned in
tests/test_oracle_layer.py.
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


def _case(B, H, N, D, E, seed):
    rng = np.random.default_rng(2000 + seed)
    bits = lambda shape, scale=1.0: I.f32_to_bf16_bits(
        (rng.standard_normal(shape) * scale).astype(np.float32))
    q, k = bits((B, H, N, D)), bits((B, H, N, D))
    v, g = bits((B, H, N, E)), bits((B, H, N, E), 2.0)
    w = (1.0 + 0.25 * rng.standard_normal((H, E))).astype(np.float32)
    sl = I.alibi_slopes(H)
    sl[1::4] = 0.0
    return q, k, v, g, w, sl


def _token_major(x):
    """Head-major host bits [B,H,N,W] -> device token-major buffer [B,N,H,W] and
    its [B,H,N,W] view."""
    t = bf16_to_dev(np.ascontiguousarray(x.transpose(0, 2, 1, 3)), DEV)
    return t, t.permute(0, 2, 1, 3)


def _done():
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0


@pytest.mark.parametrize("B,H,N,D,E", [(2, 3, 777, 128, 128), (1, 64, 2500, 128, 128),
                                       (2, 80, 600, 128, 128), (1, 4, 9000, 128, 128),
                                       (1, 3, 1000, 64, 128), (2, 2, 700, 128, 64)])
def test_token_major_layer(B, H, N, D, E):
    q, k, v, g, w, sl = _case(B, H, N, D, E, seed=N % 31 + H)
    views = [_token_major(x)[1] for x in (q, k, v, g)]
    out_buf = torch.empty((B, N, H, E), dtype=torch.bfloat16, device=DEV)
    ops.fwd_fused_ex(*views, f32_to_dev(sl, DEV), f32_to_dev(w, DEV), 1e-6,
                     out_buf.permute(0, 2, 1, 3))
    _done()
    got = out_buf.permute(0, 2, 1, 3).float().cpu().numpy()
    ref = oracle.fused_layer(q, k, v, g, sl, w, 1e-6)
    assert rel(got, ref) <= TOL_BF16
    assert worst_head(got, ref) <= TOL_BF16


def test_fused_projection_buffer_layer():
    # q, k, v interleaved in one [B, N, 3, H, D] buffer, the gate in another
    # token-major buffer, head-major output
    B, H, N, D = 2, 4, 1500, 128
    q, k, v, g, w, sl = _case(B, H, N, D, D, seed=5)
    qkv = np.stack([x.transpose(0, 2, 1, 3) for x in (q, k, v)], axis=2)  # [B, N, 3, H, D]
    buf = bf16_to_dev(np.ascontiguousarray(qkv), DEV)
    qv, kv, vv = (buf[:, :, i].permute(0, 2, 1, 3) for i in range(3))
    gv = _token_major(g)[1]
    out = ops.fwd_fused_ex(qv, kv, vv, gv, f32_to_dev(sl, DEV), f32_to_dev(w, DEV), 1e-6)
    _done()
    got = out.float().cpu().numpy()
    assert rel(got, oracle.fused_layer(q, k, v, g, sl, w, 1e-6)) <= TOL_BF16


@pytest.mark.parametrize("N1,chunk", [(640, 0), (1280, 256), (3000, 0)])
def test_layer_in_two_pieces_through_the_state(N1, chunk):
    B, H, N, D = 1, 6, 5000, 128
    q, k, v, g, w, sl = _case(B, H, N, D, D, seed=N1)
    ts, tw = f32_to_dev(sl, DEV), f32_to_dev(w, DEV)
    st = torch.empty((B, H, D, D), dtype=torch.float32, device=DEV)
    fin = torch.empty_like(st)
    part = lambda x, a, b: bf16_to_dev(np.ascontiguousarray(x[:, :, a:b]), DEV)
    y1 = ops.fwd_fused_ex(*(part(x, 0, N1) for x in (q, k, v, g)), ts, tw, 1e-6,
                          final_state=st, chunk=chunk)
    y2 = ops.fwd_fused_ex(*(part(x, N1, N) for x in (q, k, v, g)), ts, tw, 1e-6,
                          init_state=st, final_state=fin, chunk=chunk)
    _done()
    ref, sref = oracle.fused_layer(q, k, v, g, sl, w, 1e-6, return_state=True)
    got = np.concatenate([y1.float().cpu().numpy(), y2.float().cpu().numpy()], axis=2)
    assert rel(got, ref) <= TOL_BF16
    assert worst_head(got, ref) <= TOL_BF16
    assert rel(fin.cpu().numpy(), sref) <= TOL_BF16


def test_prefill_then_decode_continues_the_layer():
    # prefill N tokens through the fused layer, then decode T tokens one at a
    # time from its final state: together they must equal the layer over N + T
    B, H, N, T, D = 2, 3, 900, 12, 128
    q, k, v, g, w, sl = _case(B, H, N + T, D, D, seed=77)
    ts, tw = f32_to_dev(sl, DEV), f32_to_dev(w, DEV)
    state = torch.empty((B, H, D, D), dtype=torch.float32, device=DEV)
    head = lambda x: bf16_to_dev(np.ascontiguousarray(x[:, :, :N]), DEV)
    y = ops.fwd_fused_ex(*(head(x) for x in (q, k, v, g)), ts, tw, 1e-6, final_state=state)
    outs = [y.float().cpu().numpy()]
    for t in range(N, N + T):
        step = [bf16_to_dev(np.ascontiguousarray(x[:, :, t]), DEV) for x in (q, k, v, g)]
        outs.append(ops.decode_fused(*step, state, ts, tw, 1e-6).float().cpu().numpy()[:, :, None])
    _done()
    ref, sref = oracle.fused_layer(q, k, v, g, sl, w, 1e-6, return_state=True)
    got = np.concatenate(outs, axis=2)
    assert rel(got, ref) <= TOL_BF16
    assert rel(got[:, :, N:], ref[:, :, N:]) <= TOL_BF16
    assert rel(state.cpu().numpy(), sref) <= TOL_BF16


@pytest.mark.parametrize("D,E", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_decode_layer_chain_from_random_states(D, E):
    # inputs read from one fused [B, 3, H, D] projection row per token (q, k, v)
    # and a separate gate; states ~ N(0, 0.02^2) as in the decode workload
    B, H, steps = 3, 5, 8
    w_ = I.Workload("declayer", B, H, 1, D, E, "bf16", steps=steps, kind="decode", index=90 + D + E)
    s0 = I.decode_state(w_)
    rng = np.random.default_rng(D * 3 + E)
    w = (1.0 + 0.25 * rng.standard_normal((H, E))).astype(np.float32)
    sl = I.alibi_slopes(H)
    sl[2] = 0.0
    ts, tw = f32_to_dev(sl, DEV), f32_to_dev(w, DEV)
    state = f32_to_dev(s0, DEV)
    sref = s0.astype(np.float64)
    W = max(D, E)
    for t in range(steps):
        raw = I.f32_to_bf16_bits(rng.standard_normal((B, 3, H, W)).astype(np.float32))
        g = I.f32_to_bf16_bits((2.0 * rng.standard_normal((B, H, E))).astype(np.float32))
        buf = bf16_to_dev(raw, DEV)
        qd, kd, vd = buf[:, 0, :, :D], buf[:, 1, :, :D], buf[:, 2, :, :E]
        y = ops.decode_fused(qd, kd, vd, bf16_to_dev(g, DEV), state, ts, tw, 1e-5)
        q, k, v = (np.ascontiguousarray(raw[:, i, :, :n])[:, :, None]
                   for i, n in ((0, D), (1, D), (2, E)))
        ref, sref = oracle.fused_layer(q, k, v, g[:, :, None], sl, w, 1e-5, s0=sref,
                                       return_state=True)
        assert rel(y.float().cpu().numpy(), ref[:, :, 0]) <= TOL_BF16
    _done()
    assert rel(state.cpu().numpy(), sref) <= 1e-4


@pytest.mark.parametrize("D,E", [(64, 64), (64, 128), (128, 64)])
def test_token_major_layer_narrow_heads_with_state(D, E):
    # 64-wide heads through the 4-D tensor maps (zero-filled second halves),
    # token-major in and out, with an initial state and the final state
    B, H, N = 2, 3, 1000
    q, k, v, g, w, sl = _case(B, H, N, D, E, seed=D + 2 * E)
    s0 = (0.05 * np.random.default_rng(D * E).standard_normal((B, H, D, E))).astype(np.float32)
    views = [_token_major(x)[1] for x in (q, k, v, g)]
    out_buf = torch.empty((B, N, H, E), dtype=torch.bfloat16, device=DEV)
    fin = torch.empty((B, H, D, E), dtype=torch.float32, device=DEV)
    ops.fwd_fused_ex(*views, f32_to_dev(sl, DEV), f32_to_dev(w, DEV), 1e-6,
                     out_buf.permute(0, 2, 1, 3), init_state=f32_to_dev(s0, DEV), final_state=fin)
    _done()
    ref, sref = oracle.fused_layer(q, k, v, g, sl, w, 1e-6, s0=s0.astype(np.float64),
                                   return_state=True)
    got = out_buf.permute(0, 2, 1, 3).float().cpu().numpy()
    assert rel(got, ref) <= TOL_BF16
    assert worst_head(got, ref) <= TOL_BF16
    assert rel(fin.cpu().numpy(), sref) <= TOL_BF16


def test_decode_layer_strided_output_rows():
    # the step's output written into every other row of a wider buffer
    # (strides {2 H E, E}), inputs token-major slices of one [B, H, 4, 128] row
    B, H, D, E = 4, 6, 128, 128
    w_ = I.Workload("declayer_s", B, H, 1, D, E, "bf16", steps=1, kind="decode", index=97)
    s0 = I.decode_state(w_)
    rng = np.random.default_rng(11)
    raw = I.f32_to_bf16_bits(rng.standard_normal((B, H, 4, 128)).astype(np.float32))
    buf = bf16_to_dev(raw, DEV)
    w = (1.0 + 0.25 * rng.standard_normal((H, E))).astype(np.float32)
    sl = I.alibi_slopes(H)
    state = f32_to_dev(s0, DEV)
    wide = torch.zeros((B, 2 * H, E), dtype=torch.bfloat16, device=DEV)
    outv = wide[:, ::2]
    ops.decode_fused(buf[:, :, 0], buf[:, :, 1], buf[:, :, 2], buf[:, :, 3], state,
                     f32_to_dev(sl, DEV), f32_to_dev(w, DEV), 1e-6, outv)
    _done()
    q, k, v, g = (np.ascontiguousarray(raw[:, :, i])[:, :, None] for i in range(4))
    ref, sref = oracle.fused_layer(q, k, v, g, sl, w, 1e-6, s0=s0.astype(np.float64),
                                   return_state=True)
    assert rel(outv.float().cpu().numpy(), ref[:, :, 0]) <= TOL_BF16
    assert torch.all(wide[:, 1::2] == 0)
    assert rel(state.cpu().numpy(), sref) <= 1e-4


@pytest.mark.parametrize("D,E", [(64, 128), (128, 64), (128, 128)])
def test_split_scan_layer_with_state(D, E):
    """The fused layer in the split scan (64 sequences on the grid), entering
    from a caller's state: the items that start inside a sequence combine that
    state with the chained pieces (group X's combine, including the rows and
    columns past 64-wide heads), and the final state is handed back."""
    B, H, N = 1, 64, 2500
    sms = torch.cuda.get_device_properties(DEV).multi_processor_count
    assert ops.fwd_plan(B, H, N, 0, sms)[0]["mode"] == 2
    q, k, v, g, w, sl = _case(B, H, N, D, E, seed=60 + D + E)
    s0 = 0.05 * np.random.default_rng(D + 2 * E).standard_normal((B, H, D, E))
    fin = torch.zeros((B, H, D, E), dtype=torch.float32, device=DEV)
    out = ops.fwd_fused_ex(*(bf16_to_dev(x, DEV) for x in (q, k, v, g)), f32_to_dev(sl, DEV),
                           f32_to_dev(w, DEV), 1e-6, init_state=f32_to_dev(s0.astype(np.float32), DEV),
                           final_state=fin)
    _done()
    ref, sref = oracle.fused_layer(q, k, v, g, sl, w, 1e-6, s0=s0, return_state=True)
    got = out.float().cpu().numpy()
    assert rel(got, ref) <= TOL_BF16
    assert worst_head(got, ref) <= TOL_BF16
    assert rel(fin.cpu().numpy(), sref) <= TOL_BF16
