"""Time-axis split of one long sequence across ranks (context parallelism).

Rank r holds the r-th contiguous segment (in time order) of every (b, h) chain.
Each rank runs its segment from a zero state (rank 0 from the sequence's initial
state) and gets its segment's transfer P_r (the state map with zero values);
one all-gather exchanges the (P_r, local final state) pairs; rank r >= 1 folds
those of ranks 0..r-1 into its true starting state and adds that state's
contribution to its outputs.  The recurrence is linear in (values, starting
state), which is what makes the split exact ("KDA Technical Deep Dive",
§Systems and implementation tradeoffs, Training: the chunk-boundary state seeds
the next chunk; associative scan kernels parallelise the work).

Every step runs in libkda's kernels (kda_segment_local, kda_segment_start_state,
kda_segment_correct); this module only moves the (P, final) pairs between ranks
with torch.distributed.
"""
from __future__ import annotations

import types

import torch
import torch.distributed as dist

import gated_delta_rule_109_b200 as kda

# the per-segment steps; tests may pass stand-ins with the same signatures
KERNEL_OPS = types.SimpleNamespace(
    segment_local=lambda q, k, v, la, beta, s0, ws: kda.segment_local(q, k, v, la, beta, s0, workspace=ws),
    segment_start_state=kda.segment_start_state,
    segment_correct=lambda start, lf, out, ws: kda.segment_correct(start, lf, out, workspace=ws),
)


def forward_context_parallel(q, k, v, log_alpha, beta, initial_state=None, *, workspace, group=None,
                             ops=KERNEL_OPS):
    """This rank's segment of the prefill, exact for the whole sequence.

    q, k, v, log_alpha, beta: this rank's segment ``[B, T_r, H, ·]``;
    initial_state: the sequence's initial state (used on rank 0 only);
    workspace: ``kda.workspace_bytes(B, T_r, H, 128, 128, segment=True)`` bytes.
    Returns ``(out, final)``: this segment's outputs and the state after it (on
    the last rank: the sequence's final state).  Every rank takes the same
    collective steps (one all-gather).
    """
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    out, local_final, transfer = ops.segment_local(q, k, v, log_alpha, beta,
                                                   initial_state if rank == 0 else None, workspace)
    if transfer.shape != local_final.shape:
        raise ValueError("the time-axis split needs dk == dv")
    pair = torch.stack([transfer, local_final]).contiguous()
    gathered = [torch.empty_like(pair) for _ in range(world)]
    dist.all_gather(gathered, pair, group=group)
    if rank == 0:
        return out, local_final
    transfers = torch.stack([g[0] for g in gathered[:rank]]).contiguous()
    finals = torch.stack([g[1] for g in gathered[:rank]]).contiguous()
    start = ops.segment_start_state(transfers, finals)
    final = ops.segment_correct(start, local_final, out, workspace)
    return out, final
