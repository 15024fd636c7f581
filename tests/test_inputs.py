"""Host-side checks of the seeded input generator (CPU only)."""
import numpy as np
import torch

from long_context_fwd_b200 import inputs as I


def test_alibi_slopes_values():
    s = I.alibi_slopes(64)
    assert s.dtype == np.float32 and s.shape == (64,)
    np.testing.assert_allclose(s[0], 2.0 ** (-1.0 / 8.0), rtol=1e-7)
    np.testing.assert_allclose(s[-1], 2.0 ** -8, rtol=1e-7)
    assert np.all(np.diff(s) < 0)
    np.testing.assert_allclose(I.alibi_slopes(2), [2.0 ** -4, 2.0 ** -8], rtol=1e-7)


def test_depth_scaled_slopes():
    H, L = 64, 80
    np.testing.assert_array_equal(I.depth_scaled_slopes(H, 0, L), I.alibi_slopes(H))
    assert np.all(I.depth_scaled_slopes(H, L - 1, L) == 0.0)
    per = np.stack([I.depth_scaled_slopes(H, l, L).astype(np.float64) for l in range(L)])
    # linear in depth: constant first difference, every head
    d = np.diff(per, axis=0)
    np.testing.assert_allclose(d, np.broadcast_to(d[0], d.shape), rtol=1e-5, atol=1e-9)
    assert np.all(d <= 0)
    np.testing.assert_allclose(per[40], per[0] * (1 - 40 / 79), rtol=1e-6)
    np.testing.assert_array_equal(I.depth_scaled_slopes(8, 0, 1), I.alibi_slopes(8))


def test_zero_decay_heads():
    s = I.slopes_for(I.PREFILL_32K)
    zero = np.flatnonzero(s == 0.0)
    assert list(zero) == [h for h in range(64) if h % 8 == 7]
    assert np.all(I.slopes_for(I.TINY_F32_NODECAY) == 0.0)


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 7.0
    x[:4] = [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]  # exact ties
    ours = I.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = I.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_head_inputs_row_ranges_are_consistent():
    w = I.Workload("t", 1, 2, 10000, 16, 8, "bf16", index=9)
    q, k, v = I.head_inputs(w, 0, 1)
    q2, k2, v2 = I.head_inputs(w, 0, 1, 4000, 8300)
    assert np.array_equal(q[4000:8300], q2) and np.array_equal(v[4000:8300], v2)
    assert q.dtype == np.uint16 and q.shape == (10000, 16) and v.shape == (10000, 8)
    qa, _, _ = I.head_inputs(w, 0, 0)
    assert not np.array_equal(qa, q)


def test_distributions():
    w = I.Workload("t", 1, 1, 8192, 128, 128, "bf16", index=8)
    q, k, v = (I.bf16_bits_to_f32(x) for x in I.head_inputs(w, 0, 0))
    # SiLU(N(0,1)) has mean ~0.2066 and minimum ~ -0.2785; v stays standard normal.
    assert abs(q.mean() - 0.2066) < 0.01 and q.min() > -0.2785 - 1e-3
    assert abs(k.mean() - 0.2066) < 0.01
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1.0) < 0.01
    f = I.Workload("f", 1, 1, 4096, 64, 64, "f32", index=7)
    qf, kf, vf = I.head_inputs(f, 0, 0)
    assert qf.dtype == np.float32 and abs(qf.std() - 1 / 8) < 0.005 and abs(kf.std() - 1) < 0.02


def test_decode_inputs():
    w = I.Workload("d", 4, 3, 1, 16, 8, "bf16", steps=3, kind="decode", index=6)
    s = I.decode_state(w)
    assert s.shape == (4, 3, 16, 8) and abs(s.std() - 0.02) < 0.003
    a = I.decode_step_inputs(w, 0)
    b = I.decode_step_inputs(w, 1)
    assert a[0].shape == (4, 3, 16) and a[2].shape == (4, 3, 8)
    assert not np.array_equal(a[0], b[0])


def test_sample_positions():
    p = I.sample_positions(1048576)
    assert len(p) == 64 and p[0] == 0 and p[-1] == 1048575 and np.all(np.diff(p) > 0)
    assert {127, 128, 129, 8191, 8192}.issubset(set(p.tolist()))
    assert len(I.sample_positions(10)) == 10
