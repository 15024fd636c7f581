"""Pins of the oracle's fused layer (CPU only).

The layer around the operator ("MiniMax-M1" model entry, linear-layer field:
SiLU on Q, K, V; RMSNorm on the output; a sigmoid gate on the output after
the RMSNorm, before the output projection):

    y = w * RMSNorm_E(o) * sigmoid(g),   o = operator(silu(q), silu(k), silu(v))

checked against an independent pure-Python statement built on the brute force
of the operator, against closed forms of SiLU, sigmoid and RMSNorm, and
against invariances (per-head independence, weight homogeneity, gate limits), so that a
missing activation, a norm over the wrong axis or a misplaced weight fails.
"""
import math

import numpy as np
import pytest

import oracle
from oracle.bruteforce import brute_force


def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (den if den > 0 else 1.0)


def _python_layer(q, k, v, g, lam, w, eps):
    """Pure Python: SiLU by its definition, the brute-force operator, then the
    norm over the row's E outputs, the weight and the gate."""
    silu = lambda x: x / (1.0 + math.exp(-x))
    qs = [[silu(float(x)) for x in row] for row in q]
    ks = [[silu(float(x)) for x in row] for row in k]
    vs = [[silu(float(x)) for x in row] for row in v]
    o = brute_force(qs, ks, vs, lam)
    out = []
    for t, row in enumerate(o):
        ms = sum(x * x for x in row) / len(row)
        r = 1.0 / math.sqrt(ms + eps)
        out.append([float(w[e]) * row[e] * r / (1.0 + math.exp(-float(g[t][e])))
                    for e in range(len(row))])
    return out


@pytest.mark.parametrize("N,D,E,lam,eps", [(1, 3, 4, 0.2, 1e-6), (9, 4, 3, 0.0, 0.0),
                                           (17, 3, 5, 1.1, 1e-5)])
def test_layer_matches_python_statement(N, D, E, lam, eps):
    H = 2
    q, k, v = _rand((1, H, N, D), 1), _rand((1, H, N, D), 2), _rand((1, H, N, E), 3)
    g = _rand((1, H, N, E), 4, 2.0)
    w = _rand((H, E), 5) + 1.0
    sl = [lam, 0.5]
    got = oracle.fused_layer(q, k, v, g, sl, w, eps)
    for h in range(H):
        ref = _python_layer(q[0, h], k[0, h], v[0, h], g[0, h], float(np.float32(sl[h])),
                            w[h], eps)
        assert _rel(got[0, h], np.array(ref)) <= 1e-12


def test_unit_gate_weight_gives_unit_rms():
    # w = 1, sigmoid(g) -> 1 (g = 60), eps = 0: every row has mean square 1
    B, H, N, D, E = 1, 3, 30, 8, 6
    q, k, v = _rand((B, H, N, D), 6), _rand((B, H, N, D), 7), _rand((B, H, N, E), 8)
    g = np.full((B, H, N, E), 60.0, np.float32)
    y = oracle.fused_layer(q, k, v, g, [0.0, 0.3, 2.0], np.ones((H, E)), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-12)


def test_gate_limits_and_sigmoid_at_zero():
    B, H, N, D, E = 1, 1, 12, 4, 4
    q, k, v = _rand((B, H, N, D), 9), _rand((B, H, N, D), 10), _rand((B, H, N, E), 11)
    w = np.ones((H, E))
    hi = oracle.fused_layer(q, k, v, np.full((B, H, N, E), 60.0, np.float32), [0.1], w, 1e-6)
    zero = oracle.fused_layer(q, k, v, np.zeros((B, H, N, E), np.float32), [0.1], w, 1e-6)
    lo = oracle.fused_layer(q, k, v, np.full((B, H, N, E), -60.0, np.float32), [0.1], w, 1e-6)
    np.testing.assert_allclose(zero, 0.5 * hi, rtol=1e-12)  # sigmoid(0) = 1/2
    assert np.max(np.abs(lo)) < 1e-25 * max(1.0, np.max(np.abs(hi)))


def test_rmsnorm_is_per_head_and_weight_homogeneous():
    # The norm of each (t, head) row comes from that row alone: changing head 0's
    # v leaves head 1's output bit-identical.  The weight multiplies after the
    # norm: scaling it by 2 scales the output by exactly 2.
    B, H, N, D, E = 1, 2, 20, 4, 4
    q, k, v = _rand((B, H, N, D), 12), _rand((B, H, N, D), 13), _rand((B, H, N, E), 14)
    g = _rand((B, H, N, E), 15)
    w = _rand((H, E), 16)
    sl = [0.2, 0.6]
    base = oracle.fused_layer(q, k, v, g, sl, w, 0.0)
    v2 = v.copy()
    v2[0, 0] *= 3.0
    out2 = oracle.fused_layer(q, k, v2, g, sl, w, 0.0)
    np.testing.assert_array_equal(out2[0, 1], base[0, 1])
    assert not np.allclose(out2[0, 0], base[0, 0])
    np.testing.assert_allclose(oracle.fused_layer(q, k, v, g, sl, 2.0 * w, 0.0), 2.0 * base,
                               rtol=1e-14)


def test_silu_values():
    # single token, D = E = 1, q = k = 1, v = x: o = silu(1)^2 silu(x); RMSNorm
    # of a 1-vector with eps = 0 is its sign, so y = w sign(silu(x)) sigmoid(g)
    one = np.ones((1, 1, 1, 1), np.float32)
    for x in (-3.0, -0.5, 0.7, 4.0):
        v = np.full((1, 1, 1, 1), x, np.float32)
        y = oracle.fused_layer(one, one, v, np.zeros_like(v), [0.0], [[1.0]], 0.0)
        assert y[0, 0, 0, 0] == pytest.approx(0.5 * math.copysign(1.0, x), rel=1e-14)
    # with eps = 1, y = o / sqrt(o^2 + 1) * sigmoid(0), o = silu(1)^2 silu(x)
    s1 = 1.0 / (1.0 + math.exp(-1.0))
    for x in (-3.0, 0.7):
        v = np.full((1, 1, 1, 1), x, np.float32)
        o = s1 * s1 * (float(np.float32(x)) / (1.0 + math.exp(-float(np.float32(x)))))
        y = oracle.fused_layer(one, one, v, np.zeros_like(v), [0.0], [[1.0]], 1.0)
        assert y[0, 0, 0, 0] == pytest.approx(0.5 * o / math.sqrt(o * o + 1.0), rel=1e-13)


def test_layer_rejects_bad_arguments():
    q = _rand((1, 1, 4, 2), 1)
    with pytest.raises(ValueError):
        oracle.fused_layer(q, q, q, q, [0.1], np.ones(3), 1e-6)
    with pytest.raises(TypeError):
        oracle.fused_layer(q, q, q, q.astype(np.float64), [0.1], np.ones(2), 1e-6)
    with pytest.raises(ValueError):
        oracle.fused_layer(q, q, q, q, [0.1], np.ones(2), -1.0)


def _python_layer_state(q, k, v, g, lam, w, eps, s0):
    """Pure Python, from an initial state S_0 (D x E): the operator's output gains
    gamma^(t+1) silu(q_t) S_0, and the final state is
    gamma^N S_0 + sum_s gamma^(N-1-s) silu(k_s)^T silu(v_s)."""
    silu = lambda x: x / (1.0 + math.exp(-x))
    N, D, E = len(q), len(q[0]), len(v[0])
    gam = math.exp(-lam)
    qs = [[silu(float(x)) for x in row] for row in q]
    ks = [[silu(float(x)) for x in row] for row in k]
    vs = [[silu(float(x)) for x in row] for row in v]
    o = brute_force(qs, ks, vs, lam)
    y = []
    for t in range(N):
        row = [o[t][e] + gam ** (t + 1) * sum(qs[t][d] * float(s0[d][e]) for d in range(D))
               for e in range(E)]
        r = 1.0 / math.sqrt(sum(x * x for x in row) / E + eps)
        y.append([float(w[e]) * row[e] * r / (1.0 + math.exp(-float(g[t][e]))) for e in range(E)])
    sf = [[gam ** N * float(s0[d][e]) +
           sum(gam ** (N - 1 - s) * ks[s][d] * vs[s][e] for s in range(N))
           for e in range(E)] for d in range(D)]
    return y, sf


@pytest.mark.parametrize("N,D,E,lam", [(1, 3, 4, 0.3), (11, 4, 3, 0.0), (6, 2, 5, 1.7)])
def test_layer_state_in_and_out_match_python_statement(N, D, E, lam):
    H = 2
    q, k, v = _rand((1, H, N, D), 21), _rand((1, H, N, D), 22), _rand((1, H, N, E), 23)
    g = _rand((1, H, N, E), 24, 2.0)
    w = _rand((H, E), 25) + 1.0
    s0 = _rand((1, H, D, E), 26, 0.5).astype(np.float64)
    sl = [lam, 0.4]
    y, sf = oracle.fused_layer(q, k, v, g, sl, w, 1e-6, s0=s0, return_state=True)
    for h in range(H):
        ry, rs = _python_layer_state(q[0, h], k[0, h], v[0, h], g[0, h],
                                     float(np.float32(sl[h])), w[h], 1e-6, s0[0, h])
        assert _rel(y[0, h], np.array(ry)) <= 1e-12
        assert _rel(sf[0, h], np.array(rs)) <= 1e-12


def test_layer_continues_a_sequence_from_its_state():
    # the layer over N tokens equals the layer over the first N1 tokens followed
    # by the layer over the rest started from the state the first part returned;
    # the last N - N2 tokens one at a time (decode steps of the layer) too
    B, H, N, N1, N2, D, E = 2, 3, 40, 17, 35, 6, 5
    q, k, v = _rand((B, H, N, D), 31), _rand((B, H, N, D), 32), _rand((B, H, N, E), 33)
    g = _rand((B, H, N, E), 34, 2.0)
    w = _rand((H, E), 35) + 1.0
    sl = [0.0, 0.2, 1.3]
    full, sfull = oracle.fused_layer(q, k, v, g, sl, w, 1e-6, return_state=True)
    a, sa = oracle.fused_layer(q[:, :, :N1], k[:, :, :N1], v[:, :, :N1], g[:, :, :N1], sl, w,
                               1e-6, return_state=True)
    b, sb = oracle.fused_layer(q[:, :, N1:N2], k[:, :, N1:N2], v[:, :, N1:N2], g[:, :, N1:N2],
                               sl, w, 1e-6, s0=sa, return_state=True)
    parts = [a, b]
    s = sb
    for t in range(N2, N):
        y, s = oracle.fused_layer(q[:, :, t:t + 1], k[:, :, t:t + 1], v[:, :, t:t + 1],
                                  g[:, :, t:t + 1], sl, w, 1e-6, s0=s, return_state=True)
        parts.append(y)
    assert _rel(np.concatenate(parts, axis=2), full) <= 1e-13
    assert _rel(s, sfull) <= 1e-13
    # a zero initial state is the same as none
    np.testing.assert_array_equal(
        oracle.fused_layer(q, k, v, g, sl, w, 1e-6, s0=np.zeros((B, H, D, E))), full)
