"""One sequence cut across ranks under the additive (linear) memory rule.

With the additive update the memory before a token is the initial memory plus the sum of
the increments sigma(K)^T V of everything before it (AI Wiki "Infini-Attention", "How does
the compressive memory work?" and "What is linear attention and the delta rule?"), so a
sequence split into contiguous chunks, one per rank, needs a single exchange: every rank's
chunk increment (dM_r, dz_r), all-gathered, after which rank r starts its forward from
M0 + sum_{r' < r} dM_r'.  Each rank computes its increment with the state-only entry point
(the forward's memory kernels, no outputs), runs the ordinary forward on its chunk, and
ends with the memory after the whole sequence without a second collective.

The delta rule's update reads the memory it changes, so it has no such split: shard it over
(batch, key/value head) instead, which needs no collective at all.

Every chunk but the last must end on a segment boundary (a multiple of N tokens), so that
the chunks' segments are the sequence's segments.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding


def _library_state(k, v, N, rule):
    return binding.state(k, v, None, None, N=N, rule=rule)


def _library_forward(q, k, v, beta, M0, z0, N, rule):
    return binding.forward(q, k, v, beta, M0, z0, N=N, rule=rule)


def forward_sequence_parallel(q, k, v, beta, M0=None, z0=None, *, N: int, rule="linear",
                              group=None, state_fn=None, forward_fn=None):
    """This rank's chunk of one sequence: q [B,H,L_r,d], k/v [B,Hkv,L_r,d], the same beta and
    initial memory (M0 [B,Hkv,d,d], z0 [B,Hkv,d] or None) on every rank; ranks hold
    consecutive chunks in rank order.

    Returns (out_r, M_final, z_final): this rank's outputs and, on every rank, the memory
    after the whole sequence.  ``state_fn(k, v, N, rule) -> (dM, dz)`` and
    ``forward_fn(q, k, v, beta, M0, z0, N, rule) -> (out, M, z)`` default to the CUDA
    library; one all-gather on ``group`` (NCCL for CUDA tensors) carries the increments.
    """
    if rule not in ("linear", binding.LINEAR):
        raise ValueError("sequence sharding needs the additive rule; shard the delta rule "
                         "over (batch, key/value head)")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    L_r = q.shape[2]
    if rank < world - 1 and L_r % N != 0:
        raise ValueError(f"rank {rank}: a chunk before the last must hold whole segments "
                         f"(L_r = {L_r}, N = {N})")
    state_fn = state_fn or _library_state
    forward_fn = forward_fn or _library_forward

    dM, dz = state_fn(k, v, N, rule)
    packed = torch.cat([dM.reshape(-1), dz.reshape(-1)])
    parts = [torch.empty_like(packed) for _ in range(world)]
    dist.all_gather(parts, packed, group=group)
    nM = dM.numel()

    def unpack(x):
        return x[:nM].reshape(dM.shape), x[nM:].reshape(dz.shape)

    start_M = torch.zeros_like(dM) if M0 is None else M0.to(dM.dtype).clone()
    start_z = torch.zeros_like(dz) if z0 is None else z0.to(dz.dtype).clone()
    final_M, final_z = start_M.clone(), start_z.clone()
    for r, part in enumerate(parts):
        pm, pz = unpack(part)
        if r < rank:
            start_M += pm
            start_z += pz
        final_M += pm
        final_z += pz
    out, _, _ = forward_fn(q, k, v, beta, start_M, start_z, N, rule)
    return out, final_M, final_z
