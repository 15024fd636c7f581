"""Float64 CPU oracle for Lightning Attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The CUDA library (``long_context_fwd_b200``) never
imports it and shares no code with it; the only thing both sides share is the
seeded input generator in ``long_context_fwd_b200.inputs``, which holds none
of the method's arithmetic.

The arithmetic lives in ``lightning_oracle.c`` (plain C, double precision,
OpenMP over the independent (b, h) problems); this module compiles it with gcc
on first use and wraps it for numpy arrays.  ``bruteforce.py`` is a second,
independent pure-Python statement of the definition for tiny inputs.

What is computed (one problem per (b, h), layout [B][H][N][*]):

    o_t = sum_{s <= t} exp(-lambda_h (t - s)) (q_t . k_s) v_s

after the "MiniMax-M1" model entry (archdb), linear/SSM layer configuration
field (per-head exponential decay with ALiBi-style slopes, 128x128 state per
head), and "MiniMax-01" (redeep.blog), "What Makes 1M Context Hard"
(linear-complexity attention variant).  For training with long contexts (the
abstract: 1M tokens in training) it also gives the anti-causal sum and the
gradients of L = sum_t dout_t . o_t with respect to q, k and v.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lightning_oracle.c")
_SO = os.path.join(_HERE, "liblaoracle.so")
_lock = threading.Lock()
_lib = None

F32 = 0
BF16 = 1


def build(force: bool = False) -> str:
    """Compiles lightning_oracle.c into liblaoracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O3", "-march=x86-64-v3", "-fopenmp", "-shared", "-fPIC",
               "-o", _SO + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_SO + ".tmp", _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_SO)
            P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            lib.la_oracle_masked.argtypes = [P, P, P, I, P, P, I64, I64, I64, I64, I64, I]
            lib.la_oracle_recurrent.argtypes = [P, P, P, I, P, P, P, P, I64, I64, I64, I64, I64, I]
            lib.la_oracle_recurrent_sampled.argtypes = [P, P, P, I, P, P, I64, P, I64, I64, I64,
                                                        I64, I64, I]
            lib.la_oracle_blocked.argtypes = [P, P, P, I, P, I64, P, I64, I64, I64, I64, I64, I]
            lib.la_oracle_decode_step.argtypes = [P, P, P, I, P, P, P, I64, I64, I64, I64, I]
            lib.la_oracle_max_threads.argtypes = []
            lib.la_oracle_masked_anticausal.argtypes = [P, P, P, I, P, P, I64, I64, I64, I64, I64,
                                                        I]
            lib.la_oracle_recurrent_anticausal.argtypes = [P, P, P, I, P, P, P, P, I64, I64, I64,
                                                           I64, I64, I]
            lib.la_oracle_backward_masked.argtypes = [P, P, P, P, I, P, P, P, P, I64, I64, I64,
                                                      I64, I64, I]
            lib.la_oracle_backward_recurrent.argtypes = [P, P, P, P, I, P, P, P, P, I64, I64, I64,
                                                         I64, I64, I]
            lib.la_oracle_fused_layer.argtypes = [P, P, P, P, I, P, P, ctypes.c_double, P, P, P,
                                                  I64, I64, I64, I64, I64, I]
            for f in ("la_oracle_masked", "la_oracle_recurrent", "la_oracle_recurrent_sampled",
                      "la_oracle_blocked", "la_oracle_decode_step", "la_oracle_max_threads",
                      "la_oracle_masked_anticausal", "la_oracle_recurrent_anticausal",
                      "la_oracle_backward_masked", "la_oracle_backward_recurrent",
                      "la_oracle_fused_layer"):
                getattr(lib, f).restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _inputs(q, k, v):
    """Accepts float32 arrays or bf16 bit patterns (uint16); returns (q, k, v, dtype)."""
    q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
    kinds = {x.dtype for x in (q, k, v)}
    if kinds == {np.dtype(np.float32)}:
        return q, k, v, F32
    if kinds == {np.dtype(np.uint16)}:
        return q, k, v, BF16
    raise TypeError(f"oracle inputs must all be float32 or all bf16 bits (uint16), got {kinds}")


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name} rejected its arguments (code {rc})")


def _slopes(slopes, H):
    s = np.ascontiguousarray(np.asarray(slopes, dtype=np.float32).reshape(-1))
    if s.shape[0] != H:
        raise ValueError("slopes must have H entries")
    return s


def masked(q, k, v, slopes, threads: int = 0) -> np.ndarray:
    """O(N^2) masked sum; q, k [B,H,N,D], v [B,H,N,E] -> float64 [B,H,N,E]."""
    q, k, v, dt = _inputs(q, k, v)
    B, H, N, D = q.shape
    E = v.shape[-1]
    s = _slopes(slopes, H)
    out = np.empty((B, H, N, E), dtype=np.float64)
    _check(_load().la_oracle_masked(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(s), _ptr(out),
                                    B, H, N, D, E, threads), "la_oracle_masked")
    return out


def recurrent(q, k, v, slopes, s0=None, return_state: bool = False, threads: int = 0):
    """O(N D E) recurrence; optional initial state s0 [B,H,D,E] (float64)."""
    q, k, v, dt = _inputs(q, k, v)
    B, H, N, D = q.shape
    E = v.shape[-1]
    s = _slopes(slopes, H)
    out = np.empty((B, H, N, E), dtype=np.float64)
    s0a = None if s0 is None else np.ascontiguousarray(s0, dtype=np.float64).reshape(B, H, D, E)
    sf = np.empty((B, H, D, E), dtype=np.float64) if return_state else None
    _check(_load().la_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(s), _ptr(s0a),
                                       _ptr(sf), _ptr(out), B, H, N, D, E, threads),
           "la_oracle_recurrent")
    return (out, sf) if return_state else out


def recurrent_sampled(q, k, v, slopes, positions, threads: int = 0) -> np.ndarray:
    """Recurrence emitting o_t at the given positions -> float64 [B,H,len(positions),E]."""
    q, k, v, dt = _inputs(q, k, v)
    B, H, N, D = q.shape
    E = v.shape[-1]
    s = _slopes(slopes, H)
    pos = np.ascontiguousarray(np.asarray(positions, dtype=np.int64).reshape(-1))
    out = np.empty((B, H, pos.shape[0], E), dtype=np.float64)
    _check(_load().la_oracle_recurrent_sampled(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(s), _ptr(pos),
                                               pos.shape[0], _ptr(out), B, H, N, D, E, threads),
           "la_oracle_recurrent_sampled")
    return out


def blocked(q, k, v, slopes, blk: int, threads: int = 0) -> np.ndarray:
    """Blocked form (intra + inter + carry) with block size blk."""
    q, k, v, dt = _inputs(q, k, v)
    B, H, N, D = q.shape
    E = v.shape[-1]
    s = _slopes(slopes, H)
    out = np.empty((B, H, N, E), dtype=np.float64)
    _check(_load().la_oracle_blocked(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(s), int(blk), _ptr(out),
                                     B, H, N, D, E, threads), "la_oracle_blocked")
    return out


def decode_step(q, k, v, slopes, state, threads: int = 0) -> np.ndarray:
    """One decode step; q, k [B,H,D], v [B,H,E]; state float64 [B,H,D,E] updated in place."""
    q, k, v, dt = _inputs(q, k, v)
    B, H, D = q.shape
    E = v.shape[-1]
    if state.dtype != np.float64 or not state.flags.c_contiguous or state.shape != (B, H, D, E):
        raise ValueError("state must be a C-contiguous float64 array [B,H,D,E]")
    s = _slopes(slopes, H)
    out = np.empty((B, H, E), dtype=np.float64)
    _check(_load().la_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(s), _ptr(state),
                                         _ptr(out), B, H, D, E, threads), "la_oracle_decode_step")
    return out


def masked_anticausal(q, k, v, slopes, threads: int = 0) -> np.ndarray:
    """o_t = sum_{s >= t} exp(-lambda (s - t)) (q_t . k_s) v_s, term by term."""
    q, k, v, dt = _inputs(q, k, v)
    B, H, N, D = q.shape
    E = v.shape[-1]
    s = _slopes(slopes, H)
    out = np.empty((B, H, N, E), dtype=np.float64)
    _check(_load().la_oracle_masked_anticausal(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(s), _ptr(out),
                                               B, H, N, D, E, threads),
           "la_oracle_masked_anticausal")
    return out


def recurrent_anticausal(q, k, v, slopes, s0=None, return_state: bool = False, threads: int = 0):
    """The anti-causal sum as a recurrence run from the last token down; s0 is
    the state after the last token, the returned state the one at token 0."""
    q, k, v, dt = _inputs(q, k, v)
    B, H, N, D = q.shape
    E = v.shape[-1]
    s = _slopes(slopes, H)
    out = np.empty((B, H, N, E), dtype=np.float64)
    s0a = None if s0 is None else np.ascontiguousarray(s0, dtype=np.float64).reshape(B, H, D, E)
    sf = np.empty((B, H, D, E), dtype=np.float64) if return_state else None
    _check(_load().la_oracle_recurrent_anticausal(_ptr(q), _ptr(k), _ptr(v), dt, _ptr(s),
                                                  _ptr(s0a), _ptr(sf), _ptr(out), B, H, N, D, E,
                                                  threads), "la_oracle_recurrent_anticausal")
    return (out, sf) if return_state else out


def backward(q, k, v, dout, slopes, form: str = "recurrent", threads: int = 0):
    """Gradients (dq, dk, dv) of L = sum_t dout_t . o_t (float64), as recurrences
    (form="recurrent", O(N D E)) or as the written-out sums (form="masked")."""
    q, k, v, dt = _inputs(q, k, v)
    g = np.ascontiguousarray(dout)
    if g.dtype != q.dtype:
        raise TypeError("dout must have the dtype of q, k, v")
    B, H, N, D = q.shape
    E = v.shape[-1]
    if g.shape != (B, H, N, E):
        raise ValueError("dout must be [B,H,N,E]")
    s = _slopes(slopes, H)
    dq = np.empty((B, H, N, D), dtype=np.float64)
    dk = np.empty((B, H, N, D), dtype=np.float64)
    dv = np.empty((B, H, N, E), dtype=np.float64)
    fn = {"recurrent": _load().la_oracle_backward_recurrent,
          "masked": _load().la_oracle_backward_masked}[form]
    _check(fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), dt, _ptr(s), _ptr(dq), _ptr(dk), _ptr(dv),
              B, H, N, D, E, threads), f"la_oracle_backward_{form}")
    return dq, dk, dv


def fused_layer(q, k, v, gate, slopes, norm_weight, eps: float, s0=None,
                return_state: bool = False, threads: int = 0):
    """The layer around the operator, float64 [B,H,N,E]:
    y = w * RMSNorm_E(o) * sigmoid(gate) with o the recurrence on (silu(q),
    silu(k), silu(v)); the RMSNorm runs over each head's E outputs and w is
    per channel, norm_weight [H, E] (or [H * E]).  s0: optional initial state
    [B,H,D,E] of the recurrence (on the activated k, v); with return_state the
    state after the last token is returned too: (y, state)."""
    q, k, v, dt = _inputs(q, k, v)
    g = np.ascontiguousarray(gate)
    if g.dtype != q.dtype:
        raise TypeError("gate must have the dtype of q, k, v")
    B, H, N, D = q.shape
    E = v.shape[-1]
    if g.shape != (B, H, N, E):
        raise ValueError("gate must be [B,H,N,E]")
    w = np.ascontiguousarray(np.asarray(norm_weight, dtype=np.float32).reshape(-1))
    if w.shape[0] != H * E:
        raise ValueError("norm_weight must have H * E entries")
    s = _slopes(slopes, H)
    out = np.empty((B, H, N, E), dtype=np.float64)
    s0a = None if s0 is None else np.ascontiguousarray(s0, dtype=np.float64).reshape(B, H, D, E)
    sf = np.empty((B, H, D, E), dtype=np.float64) if return_state else None
    _check(_load().la_oracle_fused_layer(_ptr(q), _ptr(k), _ptr(v), _ptr(g), dt, _ptr(s),
                                         _ptr(w), float(eps), _ptr(s0a), _ptr(sf), _ptr(out),
                                         B, H, N, D, E, threads),
           "la_oracle_fused_layer")
    return (out, sf) if return_state else out


def max_threads() -> int:
    """Threads an OpenMP region of the oracle uses by default."""
    return int(_load().la_oracle_max_threads())
