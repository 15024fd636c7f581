"""Pins of the float64 oracle against things other than itself (CPU only).

Each test checks the oracle's forms against a fact fixed by the mathematics of
the definition o_t = sum_{s<=t} exp(-lambda (t-s)) (q_t . k_s) v_s ("MiniMax-M1"
model entry (archdb), linear/SSM layer field; "MiniMax-01" (redeep.blog),
"What Makes 1M Context Hard"): an independent pure-Python brute force, closed
forms, the lambda = 0 textbook matmul, limits, invariants and a hand-worked
example.  They are chosen so that a dropped term, a sign or index error or a
transposed operand in any form fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle.bruteforce import brute_force

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (den if den > 0 else 1.0)


CASES = [
    # (B, H, N, D, E, slopes)
    (1, 1, 1, 1, 1, [0.3]),
    (1, 2, 5, 3, 2, [0.0, 0.9]),
    (2, 2, 17, 4, 3, [0.1, 3.0]),
    (1, 3, 40, 16, 16, [0.0, 0.25, 1.5]),
    (1, 1, 64, 3, 16, [0.05]),
]


@pytest.mark.parametrize("B,H,N,D,E,slopes", CASES)
def test_forms_match_bruteforce(B, H, N, D, E, slopes):
    q = _rand((B, H, N, D), 1)
    k = _rand((B, H, N, D), 2)
    v = _rand((B, H, N, E), 3)
    ref = np.zeros((B, H, N, E))
    for b in range(B):
        for h in range(H):
            lam = float(np.float32(slopes[h]))
            ref[b, h] = np.array(brute_force(q[b, h], k[b, h], v[b, h], lam)).reshape(N, E)
    got = {"masked": oracle.masked(q, k, v, slopes),
           "recurrent": oracle.recurrent(q, k, v, slopes)}
    for blk in sorted({1, 3, 7, 64, max(N, 1)}):
        got[f"blocked{blk}"] = oracle.blocked(q, k, v, slopes, blk)
    for name, out in got.items():
        assert _rel(out, ref) <= 1e-12, name


@pytest.mark.parametrize("seed", range(6))
def test_forms_match_bruteforce_random_shapes(seed):
    """Seeded random shapes, slopes (including 0 and large) and block sizes:
    every C form against the pure-Python brute force."""
    rng = np.random.default_rng(700 + seed)
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 4))
    N, D, E = int(rng.integers(1, 48)), int(rng.integers(1, 10)), int(rng.integers(1, 10))
    slopes = [float(x) for x in rng.choice([0.0, 0.01, 0.3, 1.0, 4.0], size=H)]
    q, k, v = (_rand((B, H, N, n), 10 * seed + i, scale) for i, (n, scale) in
               enumerate(((D, 1.0), (D, 0.5), (E, 2.0))))
    ref = np.zeros((B, H, N, E))
    for b in range(B):
        for h in range(H):
            ref[b, h] = np.array(brute_force(q[b, h], k[b, h], v[b, h],
                                             float(np.float32(slopes[h])))).reshape(N, E)
    forms = {"masked": oracle.masked(q, k, v, slopes), "recurrent": oracle.recurrent(q, k, v, slopes)}
    for blk in {1, int(rng.integers(1, N + 1)), N}:
        forms[f"blocked{blk}"] = oracle.blocked(q, k, v, slopes, blk)
    for name, out in forms.items():
        assert _rel(out, ref) <= 1e-12, (name, B, H, N, D, E, slopes)


@pytest.mark.parametrize("lam", [0.0, 0.05, 0.7, 2.0])
def test_closed_form_unit_inputs(lam):
    # D = E = 1, q = k = v = 1: o_t = sum_{s<=t} gamma^(t-s) = (1 - gamma^(t+1)) / (1 - gamma),
    # and t + 1 when lambda = 0.
    N = 300
    ones = np.ones((1, 1, N, 1), np.float32)
    g = math.exp(-float(np.float32(lam)))
    t = np.arange(N, dtype=np.float64)
    expect = t + 1.0 if lam == 0.0 else (1.0 - g ** (t + 1.0)) / (1.0 - g)
    for out in (oracle.masked(ones, ones, ones, [lam]), oracle.recurrent(ones, ones, ones, [lam]),
                oracle.blocked(ones, ones, ones, [lam], 64)):
        np.testing.assert_allclose(out[0, 0, :, 0], expect, rtol=1e-13, atol=0)


def test_lambda_zero_is_causal_matmul():
    # lambda = 0: O = (Q K^T masked to s <= t) V, a plain numpy matmul.
    N, D, E = 96, 8, 5
    q, k, v = _rand((1, 1, N, D), 4), _rand((1, 1, N, D), 5), _rand((1, 1, N, E), 6)
    Q, K, V = (x[0, 0].astype(np.float64) for x in (q, k, v))
    expect = (np.tril(Q @ K.T)) @ V
    for out in (oracle.masked(q, k, v, [0.0]), oracle.recurrent(q, k, v, [0.0]),
                oracle.blocked(q, k, v, [0.0], 32)):
        assert _rel(out[0, 0], expect) <= 1e-13


def test_decay_matrix_matches_matmul():
    # General lambda: O = ((Q K^T) * M) V with M_ts = exp(-lambda (t - s)) for s <= t, else 0.
    N, D, E, lam = 70, 6, 4, 0.3
    q, k, v = _rand((1, 1, N, D), 7), _rand((1, 1, N, D), 8), _rand((1, 1, N, E), 9)
    Q, K, V = (x[0, 0].astype(np.float64) for x in (q, k, v))
    t = np.arange(N)
    lam32 = float(np.float32(lam))
    M = np.where(t[:, None] >= t[None, :], np.exp(-lam32 * (t[:, None] - t[None, :])), 0.0)
    expect = ((Q @ K.T) * M) @ V
    for out in (oracle.masked(q, k, v, [lam]), oracle.recurrent(q, k, v, [lam]),
                oracle.blocked(q, k, v, [lam], 16)):
        assert _rel(out[0, 0], expect) <= 1e-13


def test_infinite_decay_keeps_diagonal():
    # gamma -> 0: only s = t survives, o_t = (q_t . k_t) v_t.
    N, D, E = 33, 5, 3
    q, k, v = _rand((1, 1, N, D), 10), _rand((1, 1, N, D), 11), _rand((1, 1, N, E), 12)
    Q, K, V = (x[0, 0].astype(np.float64) for x in (q, k, v))
    expect = np.sum(Q * K, axis=1)[:, None] * V
    for out in (oracle.masked(q, k, v, [1e4]), oracle.recurrent(q, k, v, [1e4]),
                oracle.blocked(q, k, v, [1e4], 8)):
        assert _rel(out[0, 0], expect) <= 1e-14


def test_linearity_in_v_and_q():
    N, D, E, sl = 50, 6, 7, [0.2]
    q1, q2 = _rand((1, 1, N, D), 13), _rand((1, 1, N, D), 14)
    k = _rand((1, 1, N, D), 15)
    v1, v2 = _rand((1, 1, N, E), 16), _rand((1, 1, N, E), 17)
    a, b = np.float32(0.75), np.float32(-1.5)
    for f in (oracle.masked, oracle.recurrent, lambda *x: oracle.blocked(*x, 9)):
        lhs = f(q1, k, (a * v1 + b * v2).astype(np.float32), sl)
        rhs = a * f(q1, k, v1, sl) + b * f(q1, k, v2, sl)
        assert _rel(lhs, rhs) <= 1e-6  # fp32 rounding of a*v1 + b*v2 in the input
        lhs = f((a * q1 + b * q2).astype(np.float32), k, v1, sl)
        rhs = a * f(q1, k, v1, sl) + b * f(q2, k, v1, sl)
        assert _rel(lhs, rhs) <= 1e-6


def test_zero_key_prefix_leaves_later_outputs():
    # Tokens with k = 0 add nothing to the state: prepending P of them leaves the
    # outputs of the original tokens unchanged.
    N, P, D, E, sl = 30, 11, 4, 3, [0.4]
    q, k, v = _rand((1, 1, N, D), 18), _rand((1, 1, N, D), 19), _rand((1, 1, N, E), 20)
    qp = np.concatenate([_rand((1, 1, P, D), 21), q], axis=2)
    kp = np.concatenate([np.zeros((1, 1, P, D), np.float32), k], axis=2)
    vp = np.concatenate([_rand((1, 1, P, E), 22), v], axis=2)
    for f in (oracle.masked, oracle.recurrent, lambda *x: oracle.blocked(*x, 8)):
        base = f(q, k, v, sl)
        pre = f(qp, kp, vp, sl)
        assert _rel(pre[:, :, P:], base) <= 1e-14
        assert np.all(pre[:, :, :P] == 0.0)


def test_causality_bitwise():
    N, D, E, t0, sl = 40, 5, 4, 23, [0.3]
    q, k, v = _rand((1, 1, N, D), 23), _rand((1, 1, N, D), 24), _rand((1, 1, N, E), 25)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[..., t0, :] += 1.0
    k2[..., t0, :] -= 2.0
    v2[..., t0, :] *= 3.0
    for f in (oracle.masked, oracle.recurrent, lambda *x: oracle.blocked(*x, 8)):
        a, b = f(q, k, v, sl), f(q2, k2, v2, sl)
        assert np.array_equal(a[:, :, :t0], b[:, :, :t0])
        assert not np.array_equal(a[:, :, t0], b[:, :, t0])


def test_decode_chain_equals_prefill():
    B, H, N, D, E = 2, 3, 25, 6, 5
    sl = [0.0, 0.3, 1.2]
    q, k, v = _rand((B, H, N, D), 26), _rand((B, H, N, D), 27), _rand((B, H, N, E), 28)
    pre, sfin = oracle.recurrent(q, k, v, sl, return_state=True)
    state = np.zeros((B, H, D, E))
    for t in range(N):
        o = oracle.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], sl, state)
        assert _rel(o, pre[:, :, t]) <= 1e-13
    assert _rel(state, sfin) <= 1e-13
    # masked form agrees too (independent arithmetic)
    assert _rel(oracle.masked(q, k, v, sl), pre) <= 1e-12


def test_decode_from_state_and_state_api():
    B, H, N, D, E = 1, 2, 12, 4, 6
    sl = [0.5, 0.0]
    s0 = np.random.default_rng(29).standard_normal((B, H, D, E)) * 0.02
    q, k, v = _rand((B, H, N, D), 30), _rand((B, H, N, D), 31), _rand((B, H, N, E), 32)
    pre, sfin = oracle.recurrent(q, k, v, sl, s0=s0, return_state=True)
    state = s0.copy()
    for t in range(N):
        o = oracle.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], sl, state)
        assert _rel(o, pre[:, :, t]) <= 1e-13
    # From S0 the output is the zero-state output plus exp(-lambda (t+1)) q_t S0.
    z = oracle.recurrent(q, k, v, sl)
    for h in range(H):
        g = math.exp(-float(np.float32(sl[h])))
        extra = np.stack([g ** (t + 1) * (q[0, h, t].astype(np.float64) @ s0[0, h])
                          for t in range(N)])
        assert _rel(pre[0, h], z[0, h] + extra) <= 1e-12
    # Splitting the sequence and carrying the state reproduces the whole.
    a, sa = oracle.recurrent(q[:, :, :5], k[:, :, :5], v[:, :, :5], sl, s0=s0, return_state=True)
    b2, sb = oracle.recurrent(q[:, :, 5:], k[:, :, 5:], v[:, :, 5:], sl, s0=sa, return_state=True)
    assert _rel(np.concatenate([a, b2], axis=2), pre) <= 1e-13
    assert _rel(sb, sfin) <= 1e-13


def test_decode_infinite_decay_state_is_outer_product():
    B, H, D, E = 2, 2, 5, 3
    q, k, v = _rand((B, H, D), 33), _rand((B, H, D), 34), _rand((B, H, E), 35)
    state = np.random.default_rng(36).standard_normal((B, H, D, E))
    o = oracle.decode_step(q, k, v, [1e4, 1e4], state)
    outer = k.astype(np.float64)[..., :, None] * v.astype(np.float64)[..., None, :]
    assert np.allclose(state, outer, rtol=1e-15, atol=0)
    assert _rel(o, np.einsum("bhd,bhde->bhe", q.astype(np.float64), outer)) <= 1e-14


def test_hand_worked_example():
    with open(os.path.join(GOLDEN, "worked_example_n3.json")) as f:
        g = json.load(f)
    q = np.array(g["q"], np.float32)[None, None]
    k = np.array(g["k"], np.float32)[None, None]
    v = np.array(g["v"], np.float32)[None, None]
    for case in g["cases"]:
        expect = np.array(case["out"], np.float64)
        for f in (oracle.masked, oracle.recurrent, lambda *x: oracle.blocked(*x, 2)):
            out = f(q, k, v, [case["lambda"]])[0, 0]
            np.testing.assert_allclose(out, expect, rtol=case["tol"], atol=case["tol"])
        out = np.array(brute_force(q[0, 0], k[0, 0], v[0, 0],
                                   float(np.float32(case["lambda"]))))
        np.testing.assert_allclose(out, expect, rtol=case["tol"], atol=case["tol"])


def test_bf16_input_path_is_exact_upcast():
    from long_context_fwd_b200.inputs import bf16_bits_to_f32, f32_to_bf16_bits
    N, D, E, sl = 20, 4, 4, [0.3]
    bits = [f32_to_bf16_bits(_rand((1, 1, N, w), s)) for w, s in ((D, 37), (D, 38), (E, 39))]
    f32 = [bf16_bits_to_f32(b) for b in bits]
    for f in (oracle.masked, oracle.recurrent, lambda *x: oracle.blocked(*x, 8)):
        assert np.array_equal(f(*bits, sl), f(*f32, sl))


def test_sampled_recurrence_matches_full():
    B, H, N, D, E = 1, 2, 300, 8, 8
    sl = [0.02, 0.0]
    q, k, v = _rand((B, H, N, D), 40), _rand((B, H, N, D), 41), _rand((B, H, N, E), 42)
    full = oracle.recurrent(q, k, v, sl)
    pos = [299, 0, 128, 127, 5]
    samp = oracle.recurrent_sampled(q, k, v, sl, pos)
    assert _rel(samp, full[:, :, pos]) <= 1e-14


def test_oracle_rejects_bad_arguments():
    q = np.zeros((1, 1, 4, 2), np.float32)
    with pytest.raises(TypeError):
        oracle.masked(q, q.astype(np.float64), q, [0.1])
    with pytest.raises(ValueError):
        oracle.recurrent_sampled(q, q, q, [0.1], [4])
    with pytest.raises(ValueError):
        oracle.blocked(q, q, q, [0.1], 0)
