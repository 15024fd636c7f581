"""Seeded synthetic inputs for Lightning Attention workloads.

This module is the one piece shared by the CUDA path's tests/benchmarks and the
float64 oracle: it draws the inputs and holds none of the method's arithmetic.

Workload shapes and distributions (per (b, h) problem, head-major layout):
  * bf16 prefill workloads: q, k = bf16(SiLU(x)), v = bf16(y), x, y ~ N(0, 1)
    drawn in fp32, SiLU in fp32, then rounded to nearest-even bf16.  The SiLU
    follows the Lightning layer of the "MiniMax-M1" model entry (archdb),
    linear/SSM layer field ("SiLU on Q, K, V"); as in the workload recipe it is
    applied to q and k only, v stays Gaussian.
  * fp32 check workload: q, k, v ~ N(0, 1) fp32, q scaled by D^-1/2.
  * slopes: lambda_h = 2^(-8 (h + 1) / H), h zero-based -- the ALiBi-style
    slopes of the same entry; the "scaled down linearly with depth" part has no
    formula on the page and is not applied.  Optional lambda = 0 heads.
  * decode: states ~ N(0, 0.02^2) fp32 (0.02 read as a standard deviation),
    per-step q, k, v drawn like the prefill inputs.

Every array is drawn from its own numpy PCG64 stream keyed by
(workload, tensor, b, h, step), so any single head of any workload (the
1,048,576-token one included) can be regenerated alone on the host.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

_SEED_BASE = 20250115  # fixed base of every stream

_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "state": 4}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtype and input recipe."""

    name: str
    B: int
    H: int
    N: int
    D: int
    E: int
    dtype: str  # "bf16" or "f32" (input dtype; outputs are fp32)
    zero_decay_every: int = 0  # heads with h % m == m - 1 get lambda = 0 (0: none)
    all_zero_decay: bool = False  # every head lambda = 0
    steps: int = 0  # decode steps (decode workloads only)
    kind: str = "prefill"  # "prefill" or "decode"
    index: int = 0  # stream key of the workload

    @property
    def tokens(self) -> int:
        """Positions processed per pass (a token spans all H heads)."""
        return self.B * self.N if self.kind == "prefill" else self.B


# The five workloads: the fp32 check, the 8K single-group prefill, the batched
# 32K prefill with lambda = 0 heads, the 1,048,576-token prefill and decode.
TINY_F32 = Workload("tiny_f32_b1h2n256d64", 1, 2, 256, 64, 64, "f32", index=0)
TINY_F32_NODECAY = dataclasses.replace(TINY_F32, name="tiny_f32_b1h2n256d64_lambda0",
                                       all_zero_decay=True)
PREFILL_8K = Workload("prefill_b1h64n8192d128", 1, 64, 8192, 128, 128, "bf16", index=1)
PREFILL_32K = Workload("prefill_b4h64n32768d128", 4, 64, 32768, 128, 128, "bf16",
                       zero_decay_every=8, index=2)
PREFILL_1M = Workload("prefill_b1h64n1048576d128", 1, 64, 1048576, 128, 128, "bf16", index=3)
DECODE = Workload("decode_b256h64d128_1024steps", 256, 64, 1, 128, 128, "bf16", steps=1024,
                  kind="decode", index=4)

# Profiling case: one wave of whole sequences (148 = the B200 SM count), the
# unsplit code path of the 32K workload at 1.5 GB instead of 10.7 GB.
PROFILE_148x8K = Workload("profile_prefill_b1h148n8192d128", 1, 148, 8192, 128, 128, "bf16",
                          index=5)

# Profiling case of the split scan (64 sequences on 148 SMs, the code path of
# the 8K and 1M workloads) at 2.7 GB: the local-state pass re-reads the K and V
# of the first 1 - 64/148 of every sequence.
PROFILE_64x32K = Workload("profile_prefill_b1h64n32768d128", 1, 64, 32768, 128, 128, "bf16",
                          index=7)

WORKLOADS = {w.name: w for w in (TINY_F32, TINY_F32_NODECAY, PREFILL_8K, PREFILL_32K,
                                 PREFILL_1M, DECODE, PROFILE_148x8K, PROFILE_64x32K)}


def alibi_slopes(H: int) -> np.ndarray:
    """lambda_h = 2^(-8 (h + 1) / H) for h = 0..H-1, as float32."""
    h = np.arange(H, dtype=np.float64)
    return np.power(2.0, -8.0 * (h + 1.0) / H).astype(np.float32)


def depth_scaled_slopes(H: int, layer: int, n_layers: int) -> np.ndarray:
    """Per-head decay rates of the layer at depth `layer` (0-based) of a model
    with `n_layers` layers: the ALiBi-style rates scaled down linearly with
    depth, lambda_h * (1 - layer / (n_layers - 1)), as float32.

    "MiniMax-M1" model entry, linear-layer field: per-head exponential decay
    with ALiBi-style slopes scaled down linearly with depth.  The field gives no
    formula; this reading runs the factor from 1 at the first layer to 0 at the
    last (whose Lightning layer, if it is one, is then plain causal linear
    attention), counting every layer of the model.
    """
    if not 0 <= layer < n_layers:
        raise ValueError(f"layer {layer} outside [0, {n_layers})")
    factor = 1.0 if n_layers == 1 else 1.0 - layer / (n_layers - 1)
    h = np.arange(H, dtype=np.float64)
    return (np.power(2.0, -8.0 * (h + 1.0) / H) * factor).astype(np.float32)


def slopes_for(w: Workload) -> np.ndarray:
    """The workload's per-head slopes (float32 [H])."""
    s = alibi_slopes(w.H)
    if w.all_zero_decay:
        s[:] = 0.0
    elif w.zero_decay_every:
        m = w.zero_decay_every
        s[(np.arange(w.H) % m) == m - 1] = 0.0
    return s


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact bf16 (uint16 bits) -> fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(
        np.float32)


def _rng(w: Workload, tensor: str, b: int, h: int, step: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence([_SEED_BASE, w.index, _TENSOR_IDS[tensor], b, h, step])
    return np.random.Generator(np.random.PCG64(ss))


def _silu_f32(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float32, copy=False)
    return (x / (np.float32(1.0) + np.exp(-x))).astype(np.float32)


def head_inputs(w: Workload, b: int, h: int, n0: int = 0, n1: Optional[int] = None):
    """q, k, v of problem (b, h), rows [n0, n1) -- bf16 bits (uint16) or float32.

    Rows are drawn in fixed 4096-row pages so that any row range of the
    1,048,576-token workload regenerates identically without drawing the rest.
    """
    if w.kind != "prefill":
        raise ValueError("head_inputs is for prefill workloads")
    n1 = w.N if n1 is None else n1
    if not (0 <= n0 <= n1 <= w.N):
        raise ValueError("row range out of bounds")
    page = 4096
    outs = []
    for name, width in (("q", w.D), ("k", w.D), ("v", w.E)):
        parts = []
        for p in range(n0 // page, (n1 + page - 1) // page):
            rows = min(page, w.N - p * page)
            x = _rng(w, name, b, h, step=p).standard_normal((rows, width), dtype=np.float32)
            lo, hi = max(n0, p * page) - p * page, min(n1, p * page + rows) - p * page
            parts.append(x[lo:hi])
        x = np.concatenate(parts, axis=0) if parts else np.zeros((0, width), np.float32)
        if w.dtype == "bf16":
            x = f32_to_bf16_bits(_silu_f32(x) if name in ("q", "k") else x)
        else:
            if name == "q":
                x = (x * np.float32(1.0 / math.sqrt(w.D))).astype(np.float32)
        outs.append(np.ascontiguousarray(x))
    return tuple(outs)


def prefill_inputs(w: Workload, heads: Optional[Sequence[tuple]] = None, n: Optional[int] = None):
    """Full [B, H, n, *] arrays (n defaults to w.N); unlisted heads are zero.

    heads: iterable of (b, h) to draw; None draws all of them.
    """
    n = w.N if n is None else n
    dt = np.uint16 if w.dtype == "bf16" else np.float32
    q = np.zeros((w.B, w.H, n, w.D), dt)
    k = np.zeros((w.B, w.H, n, w.D), dt)
    v = np.zeros((w.B, w.H, n, w.E), dt)
    todo = heads if heads is not None else [(b, h) for b in range(w.B) for h in range(w.H)]
    for b, h in todo:
        q[b, h], k[b, h], v[b, h] = head_inputs(w, b, h, 0, n)
    return q, k, v


def decode_state(w: Workload) -> np.ndarray:
    """Initial decode states, float32 [B, H, D, E] ~ N(0, 0.02^2)."""
    s = np.empty((w.B, w.H, w.D, w.E), np.float32)
    for b in range(w.B):
        s[b] = (_rng(w, "state", b, 0).standard_normal((w.H, w.D, w.E), dtype=np.float32)
                * np.float32(0.02))
    return s


def decode_step_inputs(w: Workload, step: int, rows: Optional[Sequence[int]] = None):
    """q, k [B, H, D] and v [B, H, E] for one decode step, as bf16 bits.

    Each batch row b has its own stream (keyed by tensor, b and step); rows
    lists the batch rows to draw (others are zero), None draws all.
    """
    out = []
    todo = range(w.B) if rows is None else rows
    for name, width in (("q", w.D), ("k", w.D), ("v", w.E)):
        x = np.zeros((w.B, w.H, width), np.float32)
        for b in todo:
            x[b] = _rng(w, name, b, 0, step=step + 1).standard_normal((w.H, width),
                                                                      dtype=np.float32)
        x = _silu_f32(x) if name in ("q", "k") else x
        out.append(f32_to_bf16_bits(x))
    return tuple(out)


def sample_positions(N: int, blk: int = 128, count: int = 64, seed: int = 7) -> np.ndarray:
    """Sorted distinct positions to check on long sequences: block edges plus uniform draws."""
    fixed = {0, 1, blk - 1, blk, blk + 1, 8191, 8192, N - 1}
    fixed = {p for p in fixed if 0 <= p < N}
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([_SEED_BASE, 99, seed, N])))
    pos = set(fixed)
    while len(pos) < min(count, N):
        pos.add(int(rng.integers(0, N)))
    return np.array(sorted(pos), dtype=np.int64)


def device_prefill_inputs(w: Workload, device, seed: int = 0):
    """Same shapes and distributions, drawn on the device with torch's generator.

    A different random stream from head_inputs(); used where the host draw
    would dominate a benchmark's set-up time.  Returns torch tensors.
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(_SEED_BASE + 1000 * w.index + seed)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def draw(width, silu, scale=None):
        out = torch.empty((w.B, w.H, w.N, width), dtype=tdt, device=device)
        hc = max(1, min(w.H, (1 << 28) // max(1, w.N * width)))  # fp32 temporary <= 1 GiB
        for b in range(w.B):
            for h0 in range(0, w.H, hc):
                h1 = min(w.H, h0 + hc)
                x = torch.empty((h1 - h0, w.N, width), dtype=torch.float32, device=device)
                x.normal_(generator=g)
                if silu:
                    x = torch.nn.functional.silu(x)
                if scale is not None:
                    x.mul_(scale)
                out[b, h0:h1].copy_(x)
        return out

    if w.dtype == "bf16":
        return draw(w.D, True), draw(w.D, True), draw(w.E, False)
    return draw(w.D, False, 1.0 / math.sqrt(w.D)), draw(w.D, False), draw(w.E, False)
