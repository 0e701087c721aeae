"""Independent memory chains across ranks (head and batch sharding).

Every (batch b, key/value head kvh) pair owns its memory (M, z) and its G = H / Hkv query
heads, and nothing else reads that memory (AI Wiki "Infini-Attention", "How does the
compressive memory work?": the memory is kept per head), so ranks can take disjoint sets
of these chains and run the forward with no data-path collective at all.  An optional
all-gather brings every rank's outputs to every rank.

Chain c = b * Hkv + kvh.  In each tensor of the forward a chain's rows are contiguous and in
chain order: q / out [B, H, L, d] hold rows c*G .. c*G+G-1 of the flattened B*H axis, k / v
[B, Hkv, L, d] and M / z [B, Hkv, ...] row c of the flattened B*Hkv axis.  A contiguous
range of chains is therefore a view of every tensor, which the library runs as one problem
with B' = 1, Hkv' = the number of chains and H' = G times that; only beta, indexed by the
query head within a batch, is gathered for the range.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding


def chain_range(n_chains: int, world: int, rank: int):
    """The contiguous range [c0, c1) of chains rank ``rank`` of ``world`` takes: sizes differ
    by at most one, the larger ranges first."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    base, extra = divmod(n_chains, world)
    c0 = rank * base + min(rank, extra)
    return c0, c0 + base + (1 if rank < extra else 0)


def shard(q, k, v, beta, M0, z0, c0: int, c1: int):
    """Views of chains [c0, c1) of a forward's inputs, shaped as one problem with B' = 1:
    q [1, (c1-c0)*G, L, d], k / v [1, c1-c0, L, d], beta [(c1-c0)*G] (gathered), M0 / z0 the
    chains' initial memory or None."""
    B, H, L, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    n = c1 - c0
    qs = q.reshape(B * H, L, d)[c0 * G:c1 * G].reshape(1, n * G, L, d)
    ks = k.reshape(B * Hkv, L, d)[c0:c1].reshape(1, n, L, d)
    vs = v.reshape(B * Hkv, L, d)[c0:c1].reshape(1, n, L, d)
    kvh = torch.arange(c0, c1, device=beta.device) % Hkv
    bs = beta.reshape(Hkv, G)[kvh].reshape(n * G).contiguous()
    M0s = None if M0 is None else M0.reshape(B * Hkv, d, d)[c0:c1].reshape(1, n, d, d)
    z0s = None if z0 is None else z0.reshape(B * Hkv, d)[c0:c1].reshape(1, n, d)
    return qs, ks, vs, bs, M0s, z0s


def _library_forward(q, k, v, beta, M0, z0, N, rule):
    return binding.forward(q, k, v, beta, M0, z0, N=N, rule=rule)


def forward_head_sharded(q, k, v, beta, M0=None, z0=None, *, N: int, rule="linear",
                         group=None, gather: bool = True, forward_fn=None):
    """The forward of this rank's chains of one problem.

    q [B,H,L,d], k/v [B,Hkv,L,d], beta [H], M0 [B,Hkv,d,d] / z0 [B,Hkv,d] or None describe the
    whole problem; only this rank's chains (``chain_range`` over B*Hkv) are read, so the
    other chains' rows may hold anything.  Returns (out, M_out, z_out): with ``gather`` the
    whole problem's results on every rank (one all-gather per tensor on ``group``), else
    this rank's chains only, shaped [1, n*G, L, d], [1, n, d, d], [1, n, d].
    ``forward_fn(q, k, v, beta, M0, z0, N, rule) -> (out, M, z)`` defaults to the library.
    """
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    B, H, L, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    n_chains = B * Hkv
    c0, c1 = chain_range(n_chains, world, rank)
    forward_fn = forward_fn or _library_forward
    if c1 > c0:
        out, M, z = forward_fn(*shard(q, k, v, beta, M0, z0, c0, c1), N, rule)
    else:   # more ranks than chains
        out = q.new_empty((1, 0, L, d))
        M = q.new_empty((1, 0, d, d), dtype=torch.float32)
        z = q.new_empty((1, 0, d), dtype=torch.float32)
    if not gather:
        return out, M, z
    if world == 1:
        return out.reshape(B, H, L, d), M.reshape(B, Hkv, d, d), z.reshape(B, Hkv, d)
    # equal-size pieces for the all-gather: every rank pads its range to the largest one
    most = -(-n_chains // world)
    full = []
    for x, per in ((out, G * L * d), (M, d * d), (z, d)):
        flat = x.reshape(-1)
        buf = flat.new_zeros(most * per)
        buf[:flat.numel()] = flat
        parts = [torch.empty_like(buf) for _ in range(world)]
        dist.all_gather(parts, buf, group=group)
        pieces = []
        for r in range(world):
            a, b = chain_range(n_chains, world, r)
            pieces.append(parts[r][:(b - a) * per])
        full.append(torch.cat(pieces))
    return (full[0].reshape(B, H, L, d), full[1].reshape(B, Hkv, d, d),
            full[2].reshape(B, Hkv, d))
