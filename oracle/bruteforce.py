"""Pure-Python brute force of the Lightning Attention definition -- TEST INFRASTRUCTURE.

A second statement of the definition, independent of ``lightning_oracle.c``:
an explicit double loop over (t, s) in Python floats, for tiny inputs only
(N <= 64).  Used to pin the C oracle's forms.

    o_t = sum_{s <= t} exp(-lambda (t - s)) (q_t . k_s) v_s

("MiniMax-M1" model entry (archdb), linear/SSM layer field: per-head
exponential decay; "MiniMax-01" (redeep.blog), "What Makes 1M Context Hard":
linear-complexity attention.)
"""
from __future__ import annotations

import math


def brute_force(q, k, v, lam):
    """q, k: N x D, v: N x E (nested sequences or arrays of floats); lam: float.

    Returns an N x E list of Python floats.
    """
    N = len(q)
    E = len(v[0]) if N else 0
    out = [[0.0] * E for _ in range(N)]
    for t in range(N):
        for s in range(t + 1):
            dot = 0.0
            for d in range(len(q[t])):
                dot += float(q[t][d]) * float(k[s][d])
            w = math.exp(-float(lam) * (t - s)) * dot
            for e in range(E):
                out[t][e] += w * float(v[s][e])
    return out
