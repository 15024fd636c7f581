"""Pins of the oracle's anti-causal sum and gradients (CPU only).

The backward pass of Lightning Attention (for training with long contexts: the
abstract trains on 1M-token contexts) needs the gradients of
L = sum_t dout_t . o_t with respect to q, k and v, and the anti-causal sum
o_t = sum_{s >= t} exp(-lambda (s - t)) (q_t . k_s) v_s that two of them are.
These tests check the oracle's forms against facts other than themselves:
central finite differences of the independent pure-Python brute force of the
forward definition, closed forms, the decay-matrix matmul, the adjoint
identities of a function linear in each of q, k and v, and reversal symmetry.
A transposed operand, a wrong time direction or a dropped decay fails one.
"""
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


def _decay_matrix(N, lam):
    t = np.arange(N)[:, None]
    s = np.arange(N)[None, :]
    return np.where(s <= t, np.exp(-lam * (t - s).astype(np.float64)), 0.0)


@pytest.mark.parametrize("lam", [0.0, 0.2, 1.7])
def test_anticausal_closed_form_unit_inputs(lam):
    # D = E = 1, q = k = v = 1: o_t = sum_{s=t}^{N-1} g^(s-t) = (1 - g^(N-t)) / (1 - g)
    N = 23
    one = np.ones((1, 1, N, 1), np.float32)
    lam32 = float(np.float32(lam))
    g = np.exp(-lam32)
    want = np.array([N - t if lam == 0 else (1 - g ** (N - t)) / (1 - g) for t in range(N)])
    for out in (oracle.masked_anticausal(one, one, one, [lam]),
                oracle.recurrent_anticausal(one, one, one, [lam])):
        np.testing.assert_allclose(out[0, 0, :, 0], want, rtol=1e-13)


@pytest.mark.parametrize("N,D,E,lam", [(1, 2, 3, 0.4), (13, 3, 2, 0.0), (30, 5, 4, 0.7)])
def test_anticausal_is_reversed_bruteforce(N, D, E, lam):
    q, k, v = _rand((1, 1, N, D), 4), _rand((1, 1, N, D), 5), _rand((1, 1, N, E), 6)
    lam32 = float(np.float32(lam))
    rev = np.array(brute_force(q[0, 0, ::-1], k[0, 0, ::-1], v[0, 0, ::-1], lam32))[::-1]
    for out in (oracle.masked_anticausal(q, k, v, [lam]), oracle.recurrent_anticausal(q, k, v, [lam])):
        assert _rel(out[0, 0], rev) <= 1e-12


def test_anticausal_state_at_token_zero():
    # the recurrence's final state is sum_s g^s k_s^T v_s (+ g^N times the given one)
    N, D, E, lam = 19, 4, 3, 0.3
    q, k, v = _rand((1, 1, N, D), 7), _rand((1, 1, N, D), 8), _rand((1, 1, N, E), 9)
    s0 = np.random.default_rng(1).standard_normal((1, 1, D, E))
    lam32 = float(np.float32(lam))
    _, sf = oracle.recurrent_anticausal(q, k, v, [lam], s0=s0, return_state=True)
    w = np.exp(-lam32 * np.arange(N))
    want = np.einsum("s,sd,se->de", w, k[0, 0].astype(np.float64), v[0, 0].astype(np.float64))
    want += np.exp(-lam32 * N) * s0[0, 0]
    assert _rel(sf[0, 0], want) <= 1e-13


GRAD_CASES = [
    # (N, D, E, lam)
    (1, 2, 2, 0.5),
    (7, 3, 2, 0.0),
    (12, 2, 3, 0.9),
    (20, 4, 4, 0.05),
]


@pytest.mark.parametrize("N,D,E,lam", GRAD_CASES)
def test_gradients_match_finite_differences_of_bruteforce(N, D, E, lam):
    """Central differences (float64, h = 1e-5) of L = sum dout . brute_force(q, k, v)."""
    q, k, v, g = (_rand((1, 1, N, D), 11), _rand((1, 1, N, D), 12), _rand((1, 1, N, E), 13),
                  _rand((1, 1, N, E), 14))
    lam32 = float(np.float32(lam))
    base = [x[0, 0].astype(np.float64) for x in (q, k, v)]
    G = g[0, 0].astype(np.float64)

    def loss(arrs):
        return float(np.sum(G * np.array(brute_force(*arrs, lam32))))

    h = 1e-5
    fd = []
    for which in range(3):
        grad = np.zeros_like(base[which])
        for idx in np.ndindex(*grad.shape):
            plus = [a.copy() for a in base]
            minus = [a.copy() for a in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            grad[idx] = (loss(plus) - loss(minus)) / (2 * h)
        fd.append(grad)
    for form in ("masked", "recurrent"):
        got = oracle.backward(q, k, v, g, [lam], form=form)
        for name, a, b in zip("qkv", got, fd):
            assert _rel(a[0, 0], b) <= 1e-7, (form, name)


@pytest.mark.parametrize("lam", [0.0, 0.35])
def test_gradients_equal_decay_matrix_matmuls(lam):
    # with M[t][s] = g^(t-s) (s <= t): dq = (M * (G V^T)) K, dk = (M * (G V^T))^T Q,
    # dv = (M * (Q K^T))^T G -- numpy matmuls, a textbook routine
    N, D, E = 33, 6, 5
    q, k, v, g = (_rand((2, 1, N, D), 21), _rand((2, 1, N, D), 22), _rand((2, 1, N, E), 23),
                  _rand((2, 1, N, E), 24))
    M = _decay_matrix(N, float(np.float32(lam)))
    dq, dk, dv = oracle.backward(q, k, v, g, [lam])
    for b in range(2):
        Q, K, V, G = (x[b, 0].astype(np.float64) for x in (q, k, v, g))
        A = M * (G @ V.T)
        assert _rel(dq[b, 0], A @ K) <= 1e-12
        assert _rel(dk[b, 0], A.T @ Q) <= 1e-12
        assert _rel(dv[b, 0], (M * (Q @ K.T)).T @ G) <= 1e-12


def test_adjoint_identities():
    """o is linear in each of q, k, v, so L = sum dout.o = sum q.dq = sum k.dk = sum v.dv."""
    B, H, N, D, E = 2, 3, 40, 8, 6
    q, k, v, g = (_rand((B, H, N, D), 31), _rand((B, H, N, D), 32), _rand((B, H, N, E), 33),
                  _rand((B, H, N, E), 34))
    sl = [0.0, 0.3, 2.0]
    o = oracle.recurrent(q, k, v, sl)
    dq, dk, dv = oracle.backward(q, k, v, g, sl)
    L = np.sum(g.astype(np.float64) * o, axis=(2, 3))
    for x, dx in ((q, dq), (k, dk), (v, dv)):
        np.testing.assert_allclose(np.sum(x.astype(np.float64) * dx, axis=(2, 3)), L, rtol=1e-11)


def test_gradients_linear_in_dout():
    N, D, E = 25, 4, 3
    q, k, v = _rand((1, 2, N, D), 41), _rand((1, 2, N, D), 42), _rand((1, 2, N, E), 43)
    # dyadic values, so 2 g1 - 3 g2 is exact in float32
    g1, g2 = (np.round(_rand((1, 2, N, E), s) * 8) / 8 for s in (44, 45))
    sl = [0.1, 0.0]
    a = oracle.backward(q, k, v, g1, sl)
    b = oracle.backward(q, k, v, g2, sl)
    c = oracle.backward(q, k, v, (2 * g1 - 3 * g2).astype(np.float32), sl)
    for x, y, z in zip(a, b, c):
        assert _rel(z, 2 * x - 3 * y) <= 1e-12


def test_backward_bf16_inputs_are_exact_upcasts():
    from long_context_fwd_b200 import inputs as I
    N, D, E = 16, 4, 4
    x = [_rand((1, 1, N, D if i < 2 else E), 50 + i) for i in range(4)]
    bits = [I.f32_to_bf16_bits(a) for a in x]
    vals = [I.bf16_bits_to_f32(b) for b in bits]
    a = oracle.backward(*bits, [0.2])
    b = oracle.backward(*vals, [0.2])
    for u, w in zip(a, b):
        np.testing.assert_array_equal(u, w)


def test_backward_rejects_bad_arguments():
    q = _rand((1, 1, 4, 2), 1)
    with pytest.raises(ValueError):
        oracle.backward(q, q, q, _rand((1, 1, 3, 2), 2), [0.1])
    with pytest.raises(TypeError):
        oracle.backward(q, q, q, q.astype(np.float64), [0.1])
