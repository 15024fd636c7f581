#!/usr/bin/env python
"""Benchmark of the Lightning Attention hot path on B200 (one JSON line on rank 0).

Default workload (the prefill configuration the throughput target is stated
for, N >= 32K): B=4, H=64, N=32768, D=E=128, bf16 q/k/v, fp32 out, ALiBi-style
slopes with lambda = 0 on heads h % 8 == 7.  A step is one lightning_attn_fwd
call over the whole batch (q, k, v resident in HBM, 10.7 GB moved per step --
larger than L2, so no flush is needed).  The same line carries the decode leg
(256 sequences x 64 heads, fp32 128x128 states, 1024 chained
lightning_attn_decode steps), the end-to-end number through host buffers, the
roofline of the prefill kernel and the float64 oracle timed on the host cores.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs the full workload on
its own GPU -- independent (b, h) problems, no collective on the data path --
and the reported throughput is the whole job's tokens over the slowest rank's
device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "lightning-attn prefill tokens/s (% roofline); decode tokens/s (HBM GB/s)"
BLK = 128  # tokens per block in the prefill kernel


KERNEL_SOURCES = ("long_context_fwd_b200/csrc/la_fwd_sm100.cuh",
                  "long_context_fwd_b200/csrc/sm100_ptx.cuh",
                  "long_context_fwd_b200/csrc/la_schedule.cuh")
PROFILE = os.path.join(ROOT, "profiles", "prefill_bf16_tcgen05.md")


def _code_only(text: str) -> str:
    """C++ source with comments and blank lines removed, lines right-stripped
    (string literals in the kernel sources hold no comment markers)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_hash() -> str:
    """sha256 (first 16 hex) of the prefill kernel's code: a comment edit keeps
    the committed ncu capture valid, any code change invalidates it."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f)) as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def measured_traffic(workload, sms: int) -> "float | None":
    """DRAM bytes per launch of the prefill kernel from the committed ncu summary,
    scaled to `workload` by (b, h, token) units; None unless the summary was
    taken on the current kernel source.  The summary holds one capture per way
    of splitting the work: whole sequences / the balanced hand-over
    (`dram_bytes_per_launch`) and the split scan (`split_dram_bytes_per_launch`,
    whose extra local-state reads scale with tokens only for the same number
    of sequences, 64, as the 8K and 1M workloads).  `sms`: the device's SM
    count, which decides the split."""
    fields = {}
    try:
        with open(PROFILE) as f:
            for line in f:
                if line.startswith("- ") and ":" in line:
                    k, v = line[2:].split(":", 1)
                    fields[k.strip()] = v.strip().strip("`")
    except OSError:
        return None
    if fields.get("kernel_sha") != kernel_hash():
        return None
    from long_context_fwd_b200 import ops
    mode = ops.fwd_plan(workload.B, workload.H, workload.N, 0, sms)[0]["mode"]
    if mode == 2:
        if workload.B * workload.H != int(fields["split_sequences"]):
            return None
        per_unit = (float(fields["split_dram_bytes_per_launch"]) /
                    float(fields["split_token_heads_per_launch"]))
    else:
        per_unit = float(fields["dram_bytes_per_launch"]) / float(fields["token_heads_per_launch"])
    return per_unit * workload.B * workload.H * workload.N


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, source) from the
    measured peaks of this machine's B200s, else the recorded fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        burst = float(d["bf16_tflops"])
        return float(d["hbm_gbs"]), burst, float(d.get("bf16_tflops_sustained", burst)), "measured"
    except (OSError, KeyError, TypeError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_b4h64n32768d128",
                    help="prefill workload timed for the headline value (profiling uses the 8K one)")
    ap.add_argument("--chunk", type=int, default=0, help="prefill chunk length (0 = automatic)")
    ap.add_argument("--layout", choices=["head-major", "token-major"], default="head-major",
                    help="prefill q/k/v/out layout: [B][H][N][D] or [B][N][H][D]")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--e2e-steps", type=int, default=3, help="0 skips the end-to-end leg")
    ap.add_argument("--e2e-groups", type=int, default=16,
                    help="groups of sequences the end-to-end step pipelines (largest divisor "
                         "of B*H not above it that splits whole rows or equal runs of heads)")
    ap.add_argument("--e2e-upload-streams", type=int, default=1,
                    help="streams the end-to-end leg's uploads alternate between (two measured "
                         "slower: 146 vs 134-136 ms per step)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="0 skips the CPU baseline")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--backward-steps", type=int, default=20,
                    help="steps of the backward-pass leg (0 skips it)")
    ap.add_argument("--fused-steps", type=int, default=20,
                    help="steps of the fused-layer leg (0 skips it)")
    ap.add_argument("--sustained-steps", type=int, default=1000,
                    help="a second timing of the headline workload over this many launches "
                         "(clocks settled under the power cap; 0 skips it)")
    ap.add_argument("--extra-workloads",
                    default="prefill_b1h64n8192d128,prefill_b1h64n1048576d128",
                    help="comma-separated prefill workloads timed as legs of the same line")
    ap.add_argument("--state-workloads", default="prefill_b1h64n1048576d128",
                    help="comma-separated workloads whose state pass alone is timed as a leg")
    ap.add_argument("--extra-seconds", type=float, default=0.5,
                    help="about this much roofline time per extra leg")
    ap.add_argument("--extra-max-steps", type=int, default=300)
    return ap.parse_args()


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------
class Dist:
    """One process per GPU (torchrun env vars); NCCL on GPUs, gloo for CPU tests."""

    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.backend = None

    def init(self, backend, timeout_s: int = 300):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
            self.pg = dist
            self.backend = backend

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        """Max over ranks (device timings are reported as the slowest rank's)."""
        if not self.pg:
            return x
        import torch
        dev = "cpu" if self.backend == "gloo" else "cuda"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        self.windows = []

    def mark(self, t0: float, t1: float):
        self.windows.append((t0, t1))

    def stop(self):
        """Ends sampling and parses the samples; summary() then reads them."""
        self.rows = []
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        with open(self.tmp.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                    self.rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
                except (ValueError, IndexError, OverflowError):
                    continue
        os.unlink(self.tmp.name)

    def summary(self, windows=None):
        """Median SM clock, max clock and active throttle reasons of the samples
        taken inside `windows` (host-time intervals; default: every marked one)."""
        rows = getattr(self, "rows", [])
        windows = self.windows if windows is None else windows
        inside = [r for r in rows if any(a - 0.05 <= r[0] <= b + 0.05 for a, b in windows)]
        use = inside if inside else rows[-5:]
        if not use:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "in_timed_region": bool(inside)}


def roofline(bytes_launch: float, flops_launch: float, kernel_ms: float, hbm: float,
             tensor_peak: float, traffic=None, peak_src: str = "measured") -> dict:
    """Roofline of one launch: the bound is the slower of its algorithmic bytes
    at the HBM copy bandwidth and its algorithmic flops at the dense bf16
    tensor peak; achieved and peak are given in the bound's unit and frac is
    that lower-bound time over the measured launch time."""
    t_bytes = bytes_launch / (hbm * 1e9)
    t_flops = flops_launch / (tensor_peak * 1e12)
    secs = kernel_ms / 1e3
    if t_bytes >= t_flops:
        r = {"bound": "hbm", "achieved": bytes_launch / secs / 1e9, "peak": hbm, "unit": "GB/s"}
    else:
        r = {"bound": "tensor", "achieved": flops_launch / secs / 1e12, "peak": tensor_peak,
             "unit": "TFLOP/s"}
    r.update({"frac": max(t_bytes, t_flops) / secs, "traffic": traffic,
              "peak_source": f"{peak_src} ({'copy bandwidth' if r['bound'] == 'hbm' else 'bf16 GEMM'})",
              "bytes_per_launch": bytes_launch, "flops_per_launch": flops_launch,
              "kernel_ms": kernel_ms, "hbm_bound_ms": t_bytes * 1e3,
              "tensor_bound_ms": t_flops * 1e3,
              "tensor_tflops": flops_launch / secs / 1e12})
    return r


# ----------------------------------------------------------------------------
# our implementation
# ----------------------------------------------------------------------------
def timed_launches(dist, stream, steps: int, fn) -> dict:
    """Times `steps` calls of fn back to back with CUDA events on `stream`
    (a barrier and a device synchronisation on both sides; the slowest rank's
    times): the whole region and the mean per call."""
    import torch
    from long_context_fwd_b200 import ops

    dist.barrier()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    t_host0 = time.time()
    for i in range(steps):
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    torch.cuda.synchronize()
    t_host1 = time.time()
    dist.barrier()
    total_ms = starts[0].elapsed_time(ends[-1])
    launch_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))
    return {"total_ms": dist.max(total_ms), "launch_ms": dist.max(launch_ms), "steps": steps,
            "window": (t_host0, t_host1), "status": ops.device_status(reset=True)}


def bench_prefill_leg(dist, w, dev, steps: int, warmup: int) -> dict:
    """One more prefill workload timed on its own (inputs resident on the
    device, head-major, automatic work split): a leg of the JSON line."""
    import torch
    from long_context_fwd_b200 import inputs as I
    from long_context_fwd_b200 import ops

    q, k, v = I.device_prefill_inputs(w, dev)
    sl = torch.from_numpy(I.slopes_for(w)).to(dev)
    out = torch.empty((w.B, w.H, w.N, w.E), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, warmup)):
        ops.fwd(q, k, v, sl, out)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0, "device-side wait timed out during warm-up"
    res = timed_launches(dist, stream, steps, lambda: ops.fwd(q, k, v, sl, out))
    del q, k, v, out
    torch.cuda.empty_cache()
    return res


def bench_state_leg(dist, w, dev, steps: int, warmup: int) -> dict:
    """The state pass alone (lightning_attn_state: K and V in, the state after
    the sequence out) on a prefill workload's shapes, inputs resident."""
    import torch
    from long_context_fwd_b200 import inputs as I
    from long_context_fwd_b200 import ops

    _, k, v = I.device_prefill_inputs(w, dev)  # (q is drawn and dropped: same k, v as the prefill)
    torch.cuda.empty_cache()
    sl = torch.from_numpy(I.slopes_for(w)).to(dev)
    st = torch.empty((w.B, w.H, w.D, w.E), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, warmup)):
        ops.state(k, v, sl, st)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0, "device-side wait timed out during warm-up"
    res = timed_launches(dist, stream, steps, lambda: ops.state(k, v, sl, st))
    del k, v, st
    torch.cuda.empty_cache()
    return res


def bench_prefill(args, dist, w, dev):
    import torch
    from long_context_fwd_b200 import inputs as I
    from long_context_fwd_b200 import ops

    q, k, v = I.device_prefill_inputs(w, dev)
    sl = torch.from_numpy(I.slopes_for(w)).to(dev)
    token_major = args.layout == "token-major"
    if token_major:
        # [B][N][H][D] buffers, as a QKV projection writes them; the kernel
        # reads them through strided views, with no transposing copy per step
        q, k, v = (x.permute(0, 2, 1, 3).contiguous() for x in (q, k, v))
        out = torch.empty((w.B, w.N, w.H, w.E), dtype=torch.float32, device=dev)
    else:
        out = torch.empty((w.B, w.H, w.N, w.E), dtype=torch.float32, device=dev)

    def call(qx, kx, vx, ox):
        if token_major:
            tv = lambda x: x.permute(0, 2, 1, 3)
            ops.fwd_strided(tv(qx), tv(kx), tv(vx), sl, tv(ox), chunk=args.chunk)
        else:
            ops.fwd(qx, kx, vx, sl, ox, chunk=args.chunk)

    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        call(q, k, v, out)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0, "device-side wait timed out during warm-up"
    res = timed_launches(dist, stream, args.steps, lambda: call(q, k, v, out))
    if args.sustained_steps > 0:
        # the same launches again, back to back for long enough that the
        # clocks settle under the power cap
        res["sustained"] = timed_launches(dist, stream, args.sustained_steps,
                                          lambda: call(q, k, v, out))
    if args.e2e_steps <= 0:
        res["e2e_ms"], res["h2d"], res["d2h"] = None, 0, 0
        del q, k, v, out
        torch.cuda.empty_cache()
        return res
    # end to end through host buffers: pinned inputs in, result out, every step
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    del q, k, v
    torch.cuda.empty_cache()
    dq, dk, dv = (torch.empty(x.shape, dtype=x.dtype, device=dev) for x in (hq, hk, hv))

    # The step runs as G groups of consecutive (b, h) sequences (whole batch rows,
    # or equal runs of heads of one row): upload streams (groups taken in turn)
    # copy every group's inputs up back to back, one stream runs each group's
    # prefill once its inputs are in, one copies each group's result down once
    # it is computed, so uploads run continuously and overlap the downloads
    # (PCIe is full duplex).
    nseq = w.B * w.H
    G = next((g for g in range(min(args.e2e_groups, nseq), 1, -1) if nseq % g == 0 and
              (w.H % (nseq // g) == 0 or (nseq // g) % w.H == 0)), 1)
    per = nseq // G
    ups = [torch.cuda.Stream(device=dev) for _ in range(max(1, args.e2e_upload_streams))]
    comp, down = (torch.cuda.Stream(device=dev) for _ in range(2))

    def group_views(i):
        lo = i * per
        rows = per // w.H if per >= w.H else 1
        heads = w.H if per >= w.H else per
        h0 = 0 if per >= w.H else lo % w.H
        shp = lambda t: t.reshape(nseq, *t.shape[2:])[lo:lo + per].reshape(rows, heads, *t.shape[2:])
        return shp, slice(h0, h0 + heads)

    def e2e_step():
        if token_major or G == 1:
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            call(dq, dk, dv, out)
            hout.copy_(out, non_blocking=True)
            return
        start = torch.cuda.Event()
        start.record(stream)
        for st in (*ups, comp, down):
            st.wait_event(start)
        for i in range(G):
            shp, hs = group_views(i)
            gq, gk, gv, go = shp(dq), shp(dk), shp(dv), shp(out)
            up = ups[i % len(ups)]
            with torch.cuda.stream(up):
                gq.copy_(shp(hq), non_blocking=True)
                gk.copy_(shp(hk), non_blocking=True)
                gv.copy_(shp(hv), non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(up)
            comp.wait_event(landed)
            with torch.cuda.stream(comp):
                ops.fwd(gq, gk, gv, sl[hs], go, chunk=args.chunk, stream=comp)
                computed = torch.cuda.Event()
                computed.record(comp)
            down.wait_event(computed)
            with torch.cuda.stream(down):
                shp(hout).copy_(go, non_blocking=True)
        finished = torch.cuda.Event()
        finished.record(down)
        stream.wait_event(finished)

    e2e_step()
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    res["e2e_ms"] = dist.max(e0.elapsed_time(e1)) / args.e2e_steps
    res["e2e_groups"] = G if not token_major else 1
    res["h2d"] = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    res["d2h"] = hout.numel() * hout.element_size()
    del dq, dk, dv, hq, hk, hv, hout, out
    torch.cuda.empty_cache()
    return res


def bench_decode(args, dist, dev, fused: bool = False):
    """1024 chained decode steps of the decode workload (256 sequences x 64
    heads, fp32 128x128 states), inputs resident on the device.  fused: the
    layer's decode step (lightning_attn_decode_fused: raw q, k, v and gate in,
    SiLU, state step, RMSNorm, weight and sigmoid gate, bf16 out)."""
    import torch
    from long_context_fwd_b200 import inputs as I
    from long_context_fwd_b200 import ops

    w = I.DECODE
    steps = args.decode_steps
    g = torch.Generator(device=dev)
    g.manual_seed(4321)
    state = torch.randn((w.B, w.H, w.D, w.E), generator=g, device=dev) * 0.02
    sl = torch.from_numpy(I.slopes_for(w)).to(dev)
    act = (lambda x: x) if fused else torch.nn.functional.silu
    qs = act(torch.randn((steps, w.B, w.H, w.D), generator=g, device=dev)).to(torch.bfloat16)
    ks = act(torch.randn((steps, w.B, w.H, w.D), generator=g, device=dev)).to(torch.bfloat16)
    vs = torch.randn((steps, w.B, w.H, w.E), generator=g, device=dev).to(torch.bfloat16)
    if fused:
        gs = torch.randn((steps, w.B, w.H, w.E), generator=g, device=dev).to(torch.bfloat16)
        nw = torch.ones((w.H, w.E), dtype=torch.float32, device=dev)
        out = torch.empty((w.B, w.H, w.E), dtype=torch.bfloat16, device=dev)
        step = lambda i: ops.decode_fused(qs[i], ks[i], vs[i], gs[i], state, sl, nw, 1e-6, out)
    else:
        out = torch.empty((w.B, w.H, w.E), dtype=torch.float32, device=dev)
        step = lambda i: ops.decode(qs[i], ks[i], vs[i], state, sl, out)
    stream = torch.cuda.current_stream()
    for i in range(max(3, args.warmup)):
        step(i % steps)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_host0 = time.time()
    e0.record(stream)
    for i in range(steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.time()
    dist.barrier()
    ms = dist.max(e0.elapsed_time(e1)) / steps
    if fused:
        # state read + write (fp32), q, k, v and gate in (bf16), out (bf16), the
        # slope; the norm weight [H][E] once per step
        bytes_step = (w.B * w.H * (2 * w.D * w.E * 4 + 2 * w.D * 2 + 2 * w.E + 2 * w.E + 4) +
                      w.H * w.E * 4)
        del gs
    else:
        bytes_step = w.B * w.H * (2 * w.D * w.E * 4 + 2 * w.D * 2 + 2 * w.E + 4 * w.E + 4)
    finite = bool(torch.isfinite(state).all().item())
    del qs, ks, vs, state
    torch.cuda.empty_cache()
    return {"ms": ms, "bytes": bytes_step, "flops": w.B * w.H * 5 * w.D * w.E, "steps": steps,
            "window": (t_host0, t_host1), "finite": finite, "workload": w.name, "tokens": w.B}


def bench_backward(args, dist, w, dev):
    """The backward pass (dq, dk, dv from dout) on the prefill workload's shapes:
    launches of the tensor-core kernel per step: dq causal, then dk and dv
    anti-causal (one paired launch when D == E, else one each), inputs
    resident on the device."""
    import torch
    from long_context_fwd_b200 import inputs as I
    from long_context_fwd_b200 import ops

    q, k, v = I.device_prefill_inputs(w, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(98765)
    dout = torch.randn((w.B, w.H, w.N, w.E), generator=g, device=dev).to(torch.bfloat16)
    sl = torch.from_numpy(I.slopes_for(w)).to(dev)
    dq = torch.empty((w.B, w.H, w.N, w.D), dtype=torch.float32, device=dev)
    dk = torch.empty_like(dq)
    dv = torch.empty((w.B, w.H, w.N, w.E), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        ops.bwd(q, k, v, dout, sl, dq, dk, dv)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0, "device-side wait timed out during warm-up"
    dist.barrier()
    steps = args.backward_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_host0 = time.time()
    e0.record(stream)
    for _ in range(steps):
        ops.bwd(q, k, v, dout, sl, dq, dk, dv)
    e1.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.time()
    dist.barrier()
    ms = dist.max(e0.elapsed_time(e1)) / steps
    status = ops.device_status(reset=True)
    del q, k, v, dout, dq, dk, dv
    torch.cuda.empty_cache()
    units = w.B * w.H * w.N
    # streamed operands: the dq launch reads dout, v, k and writes dq; the
    # paired dk/dv launch reads q, k, v, dout (each q and dout tile from DRAM
    # once when the second role's read hits L2) and writes dk, dv; unpaired,
    # dk and dv each read three operands
    paired = w.D == w.E
    moved = units * (2 * (2 * w.E + w.D) + 4 * w.D)
    if paired:
        moved += units * (2 * (2 * w.D + 2 * w.E) + 4 * w.D + 4 * w.E)
    else:
        moved += units * (2 * (2 * w.D + w.E) + 4 * w.D + 2 * (2 * w.D + w.E) + 4 * w.E)
    return {"ms": ms, "steps": steps, "window": (t_host0, t_host1), "status": status,
            "launches": 2 if paired else 3, "bytes_moved": moved}


def bench_fused(args, dist, w, dev):
    """The fused layer (SiLU on raw q, k, v; per-head RMSNorm, weight and sigmoid
    gate on the output; bf16 out) on the prefill workload's shapes, inputs
    resident on the device."""
    import torch
    from long_context_fwd_b200 import inputs as I
    from long_context_fwd_b200 import ops

    g = torch.Generator(device=dev)
    g.manual_seed(24680)
    q, k = (torch.randn((w.B, w.H, w.N, w.D), generator=g, device=dev).to(torch.bfloat16)
            for _ in range(2))
    v, gate = (torch.randn((w.B, w.H, w.N, w.E), generator=g, device=dev).to(torch.bfloat16)
               for _ in range(2))
    nw = torch.ones((w.H, w.E), dtype=torch.float32, device=dev)
    sl = torch.from_numpy(I.slopes_for(w)).to(dev)
    out = torch.empty((w.B, w.H, w.N, w.E), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(max(3, args.warmup)):
        ops.fwd_fused(q, k, v, gate, sl, nw, 1e-6, out)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0, "device-side wait timed out during warm-up"
    dist.barrier()
    steps = args.fused_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_host0 = time.time()
    e0.record(stream)
    for _ in range(steps):
        ops.fwd_fused(q, k, v, gate, sl, nw, 1e-6, out)
    e1.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.time()
    dist.barrier()
    ms = dist.max(e0.elapsed_time(e1)) / steps
    status = ops.device_status(reset=True)
    del q, k, v, gate, out
    torch.cuda.empty_cache()
    return {"ms": ms, "steps": steps, "status": status, "window": (t_host0, t_host1)}


def cpu_baseline(w, seconds: float):
    """The float64 oracle's recurrence on a bounded sample of the workload, all
    H heads of whole batch rows while ~`seconds` last (one row cut to its first
    n tokens when a single row would take longer)."""
    import numpy as np
    import oracle
    from long_context_fwd_b200 import inputs as I

    sl = I.slopes_for(w)

    def run(b, n, threads=0):
        arrs = [I.head_inputs(w, b, h, 0, n) for h in range(w.H)]
        q = np.stack([a[0] for a in arrs])[None]
        k = np.stack([a[1] for a in arrs])[None]
        v = np.stack([a[2] for a in arrs])[None]
        t0 = time.time()
        oracle.recurrent(q, k, v, sl, threads=threads)
        return time.time() - t0

    n = 128
    dt = run(0, n)
    n = int(min(w.N, max(n, n * seconds / max(dt, 1e-3) * 0.9)))
    total, rows = run(0, n), 1
    if n == w.N:  # whole rows fit: take as many as the budget allows
        while rows < w.B and total * (rows + 1) / rows < seconds:
            total += run(rows, n)
            rows += 1
    # one core on a shorter prefix of batch row 0 (about a fifth of the budget)
    n1 = int(min(w.N, max(16, n * (seconds / 5) / max(total / rows, 1e-3) / oracle.max_threads())))
    t1 = run(0, n1, threads=1)
    return {"value": rows * n / total, "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"float64 recurrence, batch rows 0..{rows - 1} of {w.B}, all {w.H} heads, "
                      f"first {n} of {w.N} tokens ({total:.1f} s)",
            "single_core": {"value": n1 / t1, "unit": "tokens/s",
                            "sample": f"batch row 0, all {w.H} heads, first {n1} tokens ({t1:.1f} s)"}}


def job_throughput(world: int, units_per_rank: int, ms_per_step_max: float) -> float:
    """Whole-job throughput: every rank processes its own units each step; the
    step takes as long as the slowest rank."""
    return world * units_per_rank / (ms_per_step_max / 1e3)


def prefill_flops(w) -> int:
    """Algorithmic flops of one prefill launch of the blocked form at the
    kernel's 128-token blocks: 4 D E + 2 BLK (D + E) per token-head."""
    return w.B * w.H * w.N * (4 * w.D * w.E + 2 * BLK * (w.D + w.E))


def prefill_bytes(w) -> int:
    """Algorithmic bytes of one prefill launch: q, k, v read once (bf16), out
    written once (fp32)."""
    return w.B * w.H * w.N * (2 * (w.D + w.D + w.E) + 4 * w.E)


def main_ours(args):
    import torch
    from long_context_fwd_b200 import inputs as I
    from long_context_fwd_b200 import ops

    dist = Dist()
    torch.cuda.set_device(dist.local)
    dev = torch.device("cuda", dist.local)
    dist.init("nccl")
    w = I.WORKLOADS[args.workload]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    hbm, bf16, bf16_sustained, peak_src = peaks()
    sampler = ClockSampler(dist.local)
    pre = bench_prefill(args, dist, w, dev)
    legs = {}
    for name in [x for x in args.extra_workloads.split(",") if x]:
        wx = I.WORKLOADS[name]
        steps = max(3, min(args.extra_max_steps, int(args.extra_seconds * 1e3 /
                                                    max(1e-3, prefill_bytes(wx) / hbm / 1e6))))
        legs[name] = (wx, bench_prefill_leg(dist, wx, dev, steps, args.warmup))
    states = {}
    for name in [x for x in args.state_workloads.split(",") if x]:
        wx = I.WORKLOADS[name]
        sbytes = wx.B * wx.H * wx.N * 2 * (wx.D + wx.E)
        steps = max(3, min(args.extra_max_steps, int(args.extra_seconds * 1e3 /
                                                    max(1e-3, sbytes / hbm / 1e6))))
        states[name] = (wx, bench_state_leg(dist, wx, dev, steps, args.warmup))
    dec = None if args.no_decode else bench_decode(args, dist, dev)
    decf = None if args.no_decode else bench_decode(args, dist, dev, fused=True)
    bwd = None if args.backward_steps <= 0 else bench_backward(args, dist, w, dev)
    fus = None if args.fused_steps <= 0 else bench_fused(args, dist, w, dev)
    sampler.stop()
    tokens_step = w.B * w.N
    ms_step = pre["total_ms"] / args.steps
    value = job_throughput(dist.world, tokens_step, ms_step)
    bytes_launch = prefill_bytes(w)

    def traffic_for(wx):
        # the committed captures are of head-major tensors
        return measured_traffic(wx, sms) if args.layout == "head-major" else None

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded torch generator on the device; q, k = SiLU(N(0,1)), v = N(0,1))",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "E": w.E,
                   "global_batch": w.B * dist.world, "seq_len": w.N, "chunk": args.chunk or "auto",
                   "layout": args.layout,
                   "parallelism": f"replicas x{dist.world} (independent (b,h) problems, no collective)",
                   "l2": f"no flush: each step streams {bytes_launch / 1e9:.2f} GB, larger than the "
                         "126 MB L2"},
        "roofline": dict(roofline(bytes_launch, prefill_flops(w), pre["launch_ms"], hbm, bf16,
                                  traffic_for(w), peak_src),
                         tensor_peak_tflops_sustained=bf16_sustained),
        "gpu_launches": args.steps,
        "device_status": pre["status"],
        "e2e": None if pre["e2e_ms"] is None else {
            "value": job_throughput(dist.world, tokens_step, pre["e2e_ms"]), "unit": "tokens/s",
            "h2d_bytes_per_step": pre["h2d"], "d2h_bytes_per_step": pre["d2h"],
            "ms_per_step": pre["e2e_ms"],
            "pipelining": f"{pre['e2e_groups']} groups of sequences: uploads on "
                          f"{args.e2e_upload_streams} stream(s), prefills and downloads on one "
                          "each, ordered per group by events"},
        "clocks": sampler.summary([pre["window"]]),
    }
    if "sustained" in pre:
        su = pre["sustained"]
        ck = sampler.summary([su["window"]])
        line["sustained"] = {
            "what": f"the headline launches again, {su['steps']} back to back",
            "value": job_throughput(dist.world, tokens_step, su["total_ms"] / su["steps"]),
            "unit": "tokens/s", "steps": su["steps"], "ms_per_step": su["total_ms"] / su["steps"],
            "device_status": su["status"], "clocks": ck,
            "roofline": roofline(bytes_launch, prefill_flops(w), su["launch_ms"], hbm,
                                 bf16_sustained, traffic_for(w), peak_src)}
        if ck and ck.get("sm_mhz"):
            # the same time at the maximum SM clock, if it scaled with the clock
            line["sustained"]["ms_per_step_x_mhz_over_max"] = (
                su["total_ms"] / su["steps"] * ck["sm_mhz"] / ck["sm_max_mhz"])
    for name, (wx, r) in legs.items():
        tok = wx.B * wx.N
        key = {8192: "prefill_8k", 1 << 20: "prefill_1m"}.get(wx.N, wx.name)
        line[key] = {
            "workload": wx.name, "value": job_throughput(dist.world, tok, r["total_ms"] / r["steps"]),
            "unit": "tokens/s", "steps": r["steps"], "ms_per_step": r["total_ms"] / r["steps"],
            "gpu_launches": r["steps"], "device_status": r["status"],
            "split": ["whole sequences / chunk scan", "hand-over", "split scan"][
                ops.fwd_plan(wx.B, wx.H, wx.N, 0, sms)[0]["mode"]],
            "clocks": sampler.summary([r["window"]]),
            "roofline": roofline(prefill_bytes(wx), prefill_flops(wx), r["launch_ms"], hbm, bf16,
                                 traffic_for(wx), peak_src)}
    for name, (wx, r) in states.items():
        # k and v read once (bf16), the state written once (fp32); flops: the
        # state product (K~^T V) per token-head
        sbytes = wx.B * wx.H * (wx.N * 2 * (wx.D + wx.E) + 4 * wx.D * wx.E)
        line["state_" + {8192: "8k", 1 << 20: "1m"}.get(wx.N, wx.name)] = {
            "workload": wx.name, "what": "lightning_attn_state: the state after the sequence, "
                                         "no outputs (prompt prefix / sequence-split step)",
            "value": job_throughput(dist.world, wx.B * wx.N, r["total_ms"] / r["steps"]),
            "unit": "tokens/s", "steps": r["steps"], "ms_per_step": r["total_ms"] / r["steps"],
            "gpu_launches": r["steps"], "device_status": r["status"],
            "clocks": sampler.summary([r["window"]]),
            "roofline": roofline(sbytes, wx.B * wx.H * wx.N * 2 * wx.D * wx.E, r["launch_ms"],
                                 hbm, bf16, None, peak_src)}
    if dec:
        # per head-step: the state read and written (fp32), q, k, v in (bf16),
        # out (fp32) and the slope; flops: decay, k^T v and q S, 5 D E
        line["decode"] = {"workload": dec["workload"],
                          "value": dist.world * dec["tokens"] / (dec["ms"] / 1e3),
                          "unit": "tokens/s", "ms_per_step": dec["ms"], "steps": dec["steps"],
                          "gpu_launches": dec["steps"], "state_finite": dec["finite"],
                          "clocks": sampler.summary([dec["window"]]),
                          "roofline": roofline(dec["bytes"], dec["flops"], dec["ms"], hbm, bf16,
                                               None, peak_src)}
    if decf:
        line["decode_layer"] = {"workload": decf["workload"],
                                "what": "lightning_attn_decode_fused: SiLU on raw q, k, v, the "
                                        "state step, RMSNorm, weight and sigmoid gate, bf16 out",
                                "value": dist.world * decf["tokens"] / (decf["ms"] / 1e3),
                                "unit": "tokens/s", "ms_per_step": decf["ms"],
                                "steps": decf["steps"], "gpu_launches": decf["steps"],
                                "state_finite": decf["finite"],
                                "clocks": sampler.summary([decf["window"]]),
                                "roofline": roofline(decf["bytes"], decf["flops"], decf["ms"], hbm,
                                                     bf16, None, peak_src)}
    if bwd:
        # minimal traffic of the operation: q, k, v, dout read once (bf16), dq,
        # dk, dv written once (fp32); flops: three operators in the blocked form
        # (dq, dk, dv, whether dk and dv share a launch or not)
        units = w.B * w.H * w.N
        bytes_min = units * (2 * (2 * w.D + 2 * w.E) + 4 * (2 * w.D + w.E))
        r = roofline(bytes_min, 3 * prefill_flops(w), bwd["ms"], hbm, bf16, None, peak_src)
        r["bytes_moved_by_the_launches"] = bwd["bytes_moved"]
        line["backward"] = {"value": job_throughput(dist.world, tokens_step, bwd["ms"]),
                            "unit": "tokens/s", "ms_per_step": bwd["ms"], "steps": bwd["steps"],
                            "gpu_launches": bwd["launches"] * bwd["steps"],
                            "device_status": bwd["status"],
                            "clocks": sampler.summary([bwd["window"]]), "roofline": r}
    if fus:
        # the layer's traffic: raw q, k, v and the gate in (bf16), y out (bf16)
        units = w.B * w.H * w.N
        bytes_layer = units * 2 * (2 * w.D + 3 * w.E)
        line["fused_layer"] = {"value": job_throughput(dist.world, tokens_step, fus["ms"]),
                               "unit": "tokens/s", "ms_per_step": fus["ms"],
                               "steps": fus["steps"], "gpu_launches": fus["steps"],
                               "device_status": fus["status"],
                               "clocks": sampler.summary([fus["window"]]),
                               "roofline": roofline(bytes_layer, prefill_flops(w), fus["ms"], hbm,
                                                    bf16, None, peak_src)}
    if dist.rank == 0 and dist.world == 1 and args.cpu_seconds > 0:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


# ----------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# ----------------------------------------------------------------------------
def main_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import numpy as np
    import oracle
    from long_context_fwd_b200 import inputs as I

    w = I.WORKLOADS[args.workload]
    sl = I.slopes_for(w)
    budget = 120.0  # seconds for the whole reference run
    per_step = budget / max(1, args.steps + args.warmup)

    def sample(n):
        arrs = [I.head_inputs(w, 0, h, 0, n) for h in range(w.H)]
        return (np.stack([a[i] for a in arrs])[None] for i in range(3))

    q, k, v = sample(64)
    t0 = time.time()
    oracle.recurrent(q, k, v, sl)
    rate = 64 / max(time.time() - t0, 1e-4)
    n = int(min(w.N, max(64, rate * per_step)))
    q, k, v = sample(n)
    for _ in range(args.warmup):
        oracle.recurrent(q, k, v, sl)
    times = []
    for _ in range(args.steps):
        t0 = time.time()
        oracle.recurrent(q, k, v, sl)
        times.append(time.time() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = n / (ms / 1e3)
    sample_desc = (f"float64 recurrence, batch row 0, all {w.H} heads, first {n} of {w.N} tokens "
                   f"per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy generator)",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "E": w.E},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.max_threads(),
                             "kind": "oracle", "sample": sample_desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        main_reference(a)
    else:
        main_ours(a)
