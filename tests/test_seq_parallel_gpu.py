"""GPU: the sequence-parallel prefill through NCCL and the library's kernels.

One rank on one GPU (the runs here have one GPU each): the NCCL process group,
the all-gathers of the chunk state and length, the state pass
(lightning_attn_state), the combination (lightning_attn_state_combine) and
the prefill from the entering state, compared with the float64 oracle's
recurrence over the same sequence and its state after it.  With one rank the
entering state is the caller's initial state and the final state is the
combination of that state with the rank's own chunk state, so both kernels'
results reach the outputs checked here.  The rank slicing for several ranks
is covered on CPU ranks (tests/test_seq_parallel_cpu.py).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from long_context_fwd_b200 import inputs as I
from parity import TOL_BF16, bf16_to_dev, f32_to_dev, rel

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("B,H,N", [(1, 8, 3000), (2, 64, 700)])
def test_one_rank_sequence_parallel_prefill_matches_oracle(B, H, N):
    import torch.distributed as dist
    from long_context_fwd_b200.seq_parallel import prefill_sequence_parallel

    w = I.Workload(f"seqpar_gpu{H}", B, H, N, 128, 128, "bf16", index=1700 + H)
    q, k, v = I.prefill_inputs(w)
    sl = I.alibi_slopes(H)
    sl[5::8] = 0.0
    s0 = 0.05 * np.random.default_rng(H).standard_normal((B, H, 128, 128))
    ref, sref = oracle.recurrent(q, k, v, sl, s0=s0, return_state=True)

    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True, timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=DEV)
    try:
        out, final = prefill_sequence_parallel(
            bf16_to_dev(q, DEV), bf16_to_dev(k, DEV), bf16_to_dev(v, DEV), f32_to_dev(sl, DEV),
            init_state=f32_to_dev(s0.astype(np.float32), DEV))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert rel(out.cpu().numpy(), ref) <= TOL_BF16
    assert rel(final.cpu().numpy(), sref) <= TOL_BF16
