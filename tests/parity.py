"""Helpers shared by the GPU parity tests: error metrics and host<->device moves.

The error metric is the relative Frobenius norm ||out - ref||_F / ||ref||_F over
the compared elements, checked over the whole tensor and per (b, h) head.
"""
import concurrent.futures
import os

import numpy as np
import torch

# Tolerances (relative Frobenius): fp32 inputs vs the float64 oracle, and bf16
# inputs with fp32 accumulation (bf16 tensor-core operands for P, the state copy
# and the decayed Q/K tiles each round to 2^-9 relative).
TOL_F32 = 1e-4
TOL_BF16 = 1e-2
# Decode runs entirely in fp32 on exact bf16 inputs: its error is fp32 rounding,
# a few 1e-7 per step, so a much tighter bound also holds over 1024 steps.
TOL_DECODE_FP32 = 1e-4


def rel(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def worst_head(out, ref) -> float:
    """Largest per-(b, h) relative error over heads whose reference is non-zero."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    worst = 0.0
    for b in range(ref.shape[0]):
        for h in range(ref.shape[1]):
            if np.linalg.norm(ref[b, h]) > 0:
                worst = max(worst, rel(out[b, h], ref[b, h]))
    return worst


def bf16_to_dev(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def f32_to_dev(x: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def host_workers(bytes_per_worker: float, cap: int = 16) -> int:
    """Worker threads for per-head host work: the host's cores, at most `cap`,
    and no more than a third of the available memory allows."""
    n = min(cap, len(os.sched_getaffinity(0)))
    try:
        import psutil
        n = min(n, int(psutil.virtual_memory().available / 3 // bytes_per_worker))
    except ImportError:
        pass
    return max(1, n)


def fill_heads_from_host(draw, tensors, heads, per_head, workers: int):
    """For each (b, h) in `heads`, in worker threads: draws its inputs on the
    host with draw(b, h) (the draw the oracle consumes), copies them into
    tensors[i][b, h] on the device, and computes per_head(b, h, *arrays) --
    typically the oracle's reference.  Numpy's draws, the copies and the
    oracle's C code release the GIL, so heads proceed in parallel; at most
    `workers` heads' inputs are held on the host at a time.
    Returns {(b, h): per_head(...)}."""
    def job(bh):
        b, h = bh
        arrays = draw(b, h)
        for dst, x in zip(tensors, arrays):
            x = np.ascontiguousarray(x)
            if dst.dtype == torch.bfloat16:
                src = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
            else:
                src = torch.from_numpy(x)
            dst[b, h].copy_(src)
        return bh, per_head(b, h, *arrays)

    out = {}
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        for bh, r in ex.map(job, list(heads)):
            out[bh] = r
    torch.cuda.synchronize()
    return out
