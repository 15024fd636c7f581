"""GPU parity of the state pass (lightning_attn_state) and of the chunk-state
combination (lightning_attn_state_combine) against the float64 oracle.

The state pass gives the recurrent state after N tokens without the outputs;
the combination joins consecutive chunks' states (the recurrence is linear in
its initial state).  Together with a prefill from an initial state they split
one sequence into chunks that can run at the same time (on several GPUs, see
long_context_fwd_b200/seq_parallel.py); here the chunks run one after the
other on one GPU and the joined result must equal the oracle's recurrence
over the whole sequence.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_fwd_b200 import inputs as I
from long_context_fwd_b200 import ops
from parity import TOL_BF16, bf16_to_dev, f32_to_dev, rel, worst_head

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _case(seed, B, H, N, D=128, E=128):
    w = I.Workload(f"state{seed}", B, H, N, D, E, "bf16", index=1500 + seed)
    q, k, v = I.prefill_inputs(w)
    sl = I.alibi_slopes(H)
    sl[3::4] = 0.0
    return q, k, v, sl


def _worst_state(got, ref):
    return max(rel(got[b, h], ref[b, h]) for b in range(ref.shape[0]) for h in range(ref.shape[1]))


@pytest.mark.parametrize("B,H,N,chunk,with_init", [
    (1, 3, 3000, 0, False),     # few sequences: chunked, ticketed scan
    (2, 80, 1100, 0, True),     # more sequences than SMs: whole sequences
    (1, 4, 20000, 2048, True),  # explicit chunks
    (1, 5, 100, 0, False),      # one ragged block
    (1, 1, 1, 0, True),         # one token
])
def test_state_pass_matches_oracle(B, H, N, chunk, with_init):
    q, k, v, sl = _case(N % 97 + B, B, H, N)
    s0 = (0.05 * np.random.default_rng(N).standard_normal((B, H, 128, 128))) if with_init else None
    st = ops.state(bf16_to_dev(k, DEV), bf16_to_dev(v, DEV), f32_to_dev(sl, DEV),
                   init_state=None if s0 is None else f32_to_dev(s0, DEV), chunk=chunk)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    _, ref = oracle.recurrent(q, k, v, sl, s0=s0, return_state=True)
    got = st.cpu().numpy()
    assert rel(got, ref) <= TOL_BF16
    assert _worst_state(got, ref) <= TOL_BF16


@pytest.mark.parametrize("D,E", [(64, 128), (128, 64), (64, 64)])
def test_state_pass_narrow_heads(D, E):
    q, k, v, sl = _case(D + E, 1, 6, 5000, D, E)
    st = ops.state(bf16_to_dev(k, DEV), bf16_to_dev(v, DEV), f32_to_dev(sl, DEV))
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    _, ref = oracle.recurrent(q, k, v, sl, return_state=True)
    assert rel(st.cpu().numpy(), ref) <= TOL_BF16


@pytest.mark.parametrize("cuts", [(0, 1000, 2500, 7000), (0, 128, 129, 4000, 4001)])
def test_chunked_sequence_through_states_matches_oracle(cuts):
    # chunks [cuts[i], cuts[i+1]): each chunk's state from zero, the entering
    # state of chunk r combined from chunks 0..r-1 and an initial state, the
    # chunk's prefill from it -- the outputs and the final state must equal
    # the recurrence over the whole sequence
    B, H, N = 2, 4, cuts[-1]
    q, k, v, sl = _case(len(cuts), B, H, N)
    s0 = 0.05 * np.random.default_rng(5).standard_normal((B, H, 128, 128))
    ts, t0 = f32_to_dev(sl, DEV), f32_to_dev(s0, DEV)
    part = lambda x, a, b: bf16_to_dev(np.ascontiguousarray(x[:, :, a:b]), DEV)
    spans = list(zip(cuts[:-1], cuts[1:]))
    states = torch.stack([ops.state(part(k, a, b), part(v, a, b), ts) for a, b in spans])
    counts = [b - a for a, b in spans]
    outs = []
    for r, (a, b) in enumerate(spans):
        enter = ops.state_combine(states[:r].contiguous(), counts[:r], ts, init_state=t0)
        outs.append(ops.fwd(part(q, a, b), part(k, a, b), part(v, a, b), ts,
                            init_state=enter).cpu().numpy())
    final = ops.state_combine(states, counts, ts, init_state=t0)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == 0
    ref, sref = oracle.recurrent(q, k, v, sl, s0=s0, return_state=True)
    got = np.concatenate(outs, axis=2)
    assert rel(got, ref) <= TOL_BF16
    assert worst_head(got, ref) <= TOL_BF16
    assert rel(final.cpu().numpy(), sref) <= TOL_BF16


def test_combine_of_no_chunks_is_the_initial_state():
    B, H = 1, 3
    sl = f32_to_dev(I.alibi_slopes(H), DEV)
    s0 = torch.randn((B, H, 128, 128), device=DEV)
    empty = torch.empty((0, B, H, 128, 128), device=DEV)
    assert torch.equal(ops.state_combine(empty, [], sl, init_state=s0), s0)
    assert torch.count_nonzero(ops.state_combine(empty, [], sl)) == 0
