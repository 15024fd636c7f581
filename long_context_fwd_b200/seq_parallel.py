"""One sequence split across the ranks of a process group (one GPU each).

The pages train with 1M-token contexts and infer with 4M ("MiniMax-01"
abstract); one head's state is only 64 KiB, so a sequence longer than one GPU
holds -- or one that should finish sooner -- can be cut into consecutive
chunks, one per rank, with a single exchange step.  The recurrence
S_t = gamma S_{t-1} + k_t^T v_t is linear in its initial state, so:

1. every rank computes its chunk's state from a zero initial state
   (``ops.state``: K and V only, 512 B per token-head);
2. the states and the chunk lengths are all-gathered (NCCL over NVLink;
   64 KiB per head per rank);
3. rank r combines the states of chunks 0 .. r-1 into its entering state
   (``ops.state_combine``);
4. rank r runs the prefill of its chunk from that state (``ops.fwd`` with
   ``init_state``).

Each rank moves 1280 + 512 B per token-head of its own chunk, and the ranks
work at the same time.  The state after the whole sequence (for a decode that
follows) is the combination of all R states, available on every rank.

The compute steps default to the CUDA library; ``steps`` lets a caller (or a
test on CPU ranks) supply its own ``state``, ``combine`` and ``prefill``
functions with the same signatures.
"""
from __future__ import annotations

from typing import Callable, NamedTuple, Optional

import torch
import torch.distributed as dist


class Steps(NamedTuple):
    """The three compute steps: state(k, v, slopes) -> [B,H,D,E];
    combine(states [R,B,H,D,E], counts, slopes, init_state) -> [B,H,D,E];
    prefill(q, k, v, slopes, init_state) -> out [B,H,N,E]; and the dtype of
    the states and outputs they return (an empty chunk's are made in it)."""

    state: Callable
    combine: Callable
    prefill: Callable
    dtype: torch.dtype = torch.float32


def cuda_steps() -> Steps:
    """The library's kernels (the only implementation the product path uses)."""
    from long_context_fwd_b200 import ops

    return Steps(
        state=lambda k, v, sl: ops.state(k, v, sl),
        combine=lambda st, counts, sl, init: ops.state_combine(st, counts, sl, init_state=init),
        prefill=lambda q, k, v, sl, init: ops.fwd(q, k, v, sl, init_state=init),
    )


def prefill_sequence_parallel(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                              slopes: torch.Tensor, *, init_state: Optional[torch.Tensor] = None,
                              group=None, steps: Optional[Steps] = None):
    """Prefill of this rank's chunk of every (b, h) sequence.

    q, k [B,H,n_r,D], v [B,H,n_r,E] hold tokens of chunk r = this rank's index
    in ``group`` (chunks in rank order; lengths may differ between ranks, and
    a rank's chunk may be empty).  init_state (optional, [B,H,D,E]) is the
    state before chunk 0, the same on every rank.  Returns (out [B,H,n_r,E] of
    this chunk, the state after the whole sequence [B,H,D,E]).  Every rank
    takes the same collective steps.
    """
    steps = steps or cuda_steps()
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    B, H, n_r, D = k.shape
    E = v.shape[-1]
    if n_r == 0:  # an empty chunk adds nothing to the state and has no outputs
        local = torch.zeros((B, H, D, E), dtype=steps.dtype, device=k.device)
    else:
        local = steps.state(k, v, slopes).contiguous()
    parts = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(parts, local, group=group)
    n_local = torch.tensor([q.shape[2]], dtype=torch.int64, device=local.device)
    counts_t = [torch.empty_like(n_local) for _ in range(world)]
    dist.all_gather(counts_t, n_local, group=group)
    counts = [int(c.item()) for c in counts_t]
    states = torch.stack(parts)
    entering = steps.combine(states[:rank].contiguous(), counts[:rank], slopes, init_state)
    if n_r == 0:
        out = torch.empty((B, H, 0, E), dtype=steps.dtype, device=k.device)
    else:
        out = steps.prefill(q, k, v, slopes, entering)
    final = steps.combine(states, counts, slopes, init_state)
    return out, final
