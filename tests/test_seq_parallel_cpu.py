"""The sequence-parallel prefill's host logic on CPU ranks (gloo, no GPU).

long_context_fwd_b200.seq_parallel splits one sequence into consecutive
chunks, one per rank: each rank's chunk state, an all-gather of the states and
the chunk lengths, the combination of the states before its chunk, and the
prefill of its chunk from that state.  Here the compute steps are stated on
the float64 oracle (its recurrence for the state and the prefill, the
linearity of the recurrence in its initial state for the combination), so
that the ranks' chunk outputs, put together, must equal the oracle's
recurrence over the whole sequence -- checking the collective order, the rank
slicing and the uneven chunk lengths the module handles (with four ranks, one
chunk is empty).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


CUTS = {2: (0, 700, 1500), 3: (0, 128, 1000, 1501),
        4: (0, 300, 300, 1200, 1333)}  # rank 1's chunk is empty


def _oracle_steps():
    import oracle
    from long_context_fwd_b200.seq_parallel import Steps

    def state(k, v, sl):
        kk, vv = k.numpy(), v.numpy()
        _, s = oracle.recurrent(kk, kk, vv, sl.numpy(), return_state=True)
        return torch.from_numpy(s)

    def combine(states, counts, sl, init):
        lam = sl.numpy().astype(np.float64)[None, :, None, None]
        s = np.zeros(states.shape[1:]) if init is None else init.numpy().astype(np.float64)
        for j, n in enumerate(counts):
            s = np.exp(-lam * n) * s + states[j].numpy()
        return torch.from_numpy(s)

    def prefill(q, k, v, sl, init):
        return torch.from_numpy(oracle.recurrent(q.numpy(), k.numpy(), v.numpy(), sl.numpy(),
                                                 s0=init.numpy()))

    return Steps(state, combine, prefill, torch.float64)


def _rank(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from long_context_fwd_b200 import inputs as I
    from long_context_fwd_b200.seq_parallel import prefill_sequence_parallel

    dist.init_process_group("gloo", rank=rank, world_size=world)
    cuts = CUTS[world]
    w = I.Workload("seqpar", 1, 3, cuts[-1], 16, 8, "f32", index=600)
    q, k, v = I.prefill_inputs(w)
    sl = torch.from_numpy(I.alibi_slopes(w.H))
    s0 = torch.from_numpy(0.1 * np.random.default_rng(1).standard_normal((1, 3, 16, 8)))
    a, b = cuts[rank], cuts[rank + 1]
    chunk = [torch.from_numpy(np.ascontiguousarray(x[:, :, a:b])) for x in (q, k, v)]
    o, final = prefill_sequence_parallel(*chunk, sl, init_state=s0, steps=_oracle_steps())
    out.put((rank, o.numpy(), final.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
def test_ranks_chunks_equal_the_whole_sequence(world):
    import oracle
    from long_context_fwd_b200 import inputs as I

    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((out.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = I.Workload("seqpar", 1, 3, CUTS[world][-1], 16, 8, "f32", index=600)
    q, k, v = I.prefill_inputs(w)
    s0 = 0.1 * np.random.default_rng(1).standard_normal((1, 3, 16, 8))
    ref, sref = oracle.recurrent(q, k, v, I.alibi_slopes(w.H), s0=s0, return_state=True)
    whole = np.concatenate([g[1] for g in got], axis=2)
    assert np.linalg.norm(whole - ref) <= 1e-12 * np.linalg.norm(ref)
    for _, _, final in got:  # every rank has the state after the whole sequence
        assert np.linalg.norm(final - sref) <= 1e-12 * np.linalg.norm(sref)
