"""The multi-rank path of the benchmark on CPU: two gloo ranks, each running the
float64 oracle on its own replica of a small workload, with the slowest rank's
time reduced to every rank (no GPU, no collective on the data path)."""
import os
import socket
import time

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import oracle
    from long_context_fwd_b200 import inputs as I

    d = bench.Dist()
    d.init("gloo", timeout_s=60)
    w = I.Workload("mr", 1, 2, 96, 8, 8, "bf16", index=500)
    q, k, v = I.prefill_inputs(w)
    sl = I.alibi_slopes(w.H)
    d.barrier()
    t0 = time.time()
    res = oracle.recurrent(q, k, v, sl)
    time.sleep(0.05 * (rank + 1))  # ranks finish at different times
    ms = (time.time() - t0) * 1e3
    d.barrier()
    ms_max = d.max(ms)
    out.put((rank, ms, ms_max, float(np.abs(res).sum()),
             bench.job_throughput(d.world, w.B * w.N, ms_max)))
    d.close()


def test_two_gloo_ranks_report_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got.sort()
    (r0, ms0, max0, s0, thr0), (r1, ms1, max1, s1, thr1) = got
    assert max0 == max1 == max(ms0, ms1)
    assert s0 == s1  # identical replicas
    assert thr0 == thr1 == 2 * 96 / (max0 / 1e3)
