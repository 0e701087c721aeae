"""Chains across ranks (compressive_memory_long_b200.headpar), on CPU with gloo ranks.

Each rank runs only its contiguous range of (batch, kv head) chains -- the fp64 oracle
stands in for the per-rank compute (test infrastructure; the product default is the CUDA
library) -- and one all-gather per tensor assembles the results.  The union must equal one
oracle run over the whole problem, for both rules, grouped heads, and ranges that cross a
batch boundary or are empty (more ranks than chains).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from compressive_memory_long_b200 import workloads as wl

W = wl.Workload("headpar", B=2, H=6, Hkv=3, d=16, N=8, S=3, tail=5, dtype="f32",
                rule="delta", seed=71, beta_dist=("normal", 0.0, 1.0),
                M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_forward(q, k, v, beta, M0, z0, N, rule):
    import oracle
    out, M, z = oracle.infini_attn_fwd(q.numpy(), k.numpy(), v.numpy(), beta.numpy(),
                                       None if M0 is None else M0.numpy(),
                                       None if z0 is None else z0.numpy(), N=N, rule=rule)
    return (torch.from_numpy(out.astype(np.float32)), torch.from_numpy(M.astype(np.float32)),
            torch.from_numpy(z.astype(np.float32)))


def _rank_main(rank, world, port, results, rule, with_state):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from compressive_memory_long_b200 import headpar
        w = W.replace(rule=rule)
        q, k, v, beta, M0, z0 = (torch.from_numpy(x) for x in wl.host_inputs(w))
        if not with_state:
            M0 = z0 = None
        c0, c1 = headpar.chain_range(w.B * w.Hkv, world, rank)
        # rows of other ranks' chains are never read: poison them
        for x, per in ((q, w.G), (k, 1), (v, 1)):
            flat = x.view(w.B * x.shape[1] // per, per, *x.shape[2:])
            flat[:c0] = float("nan")
            flat[c1:] = float("nan")
        out, M, z = headpar.forward_head_sharded(q, k, v, beta, M0, z0, N=w.N, rule=rule,
                                                 forward_fn=_oracle_forward)
        results[rank] = (out.numpy(), M.numpy(), z.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4, 7])
@pytest.mark.parametrize("rule,with_state", [("delta", True), ("linear", False)])
def test_union_of_ranks_equals_one_run(world, rule, with_state):
    import oracle
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results, rule, with_state))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    w = W.replace(rule=rule)
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    ro, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0 if with_state else None,
                                        z0 if with_state else None, N=w.N, rule=rule)
    for r in range(world):              # every rank holds the whole problem's results
        np.testing.assert_allclose(results[r][0], ro, rtol=1e-6, atol=1e-7)
        np.testing.assert_allclose(results[r][1], rM, rtol=1e-6, atol=1e-7)
        np.testing.assert_allclose(results[r][2], rz, rtol=1e-6, atol=1e-7)


def test_chain_ranges_cover_every_chain_once():
    from compressive_memory_long_b200 import headpar
    for n in (1, 5, 6, 16, 512):
        for world in (1, 2, 3, 8, 9):
            ranges = [headpar.chain_range(n, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        headpar.chain_range(4, 2, 2)


def test_shard_views_match_the_chains():
    """A range of chains is a view: rows of q / k / v / M0 / z0 and the gathered beta are the
    chains' own, including a range that crosses a batch boundary."""
    from compressive_memory_long_b200 import headpar
    q, k, v, beta, M0, z0 = (torch.from_numpy(x) for x in wl.host_inputs(W))
    c0, c1 = 2, 5                       # (b0, kvh2), (b1, kvh0), (b1, kvh1)
    qs, ks, vs, bs, Ms, zs = headpar.shard(q, k, v, beta, M0, z0, c0, c1)
    G = W.G
    chains = [(c // W.Hkv, c % W.Hkv) for c in range(c0, c1)]
    for j, (b, kvh) in enumerate(chains):
        assert torch.equal(ks[0, j], k[b, kvh]) and torch.equal(vs[0, j], v[b, kvh])
        assert torch.equal(Ms[0, j], M0[b, kvh]) and torch.equal(zs[0, j], z0[b, kvh])
        for g in range(G):
            assert torch.equal(qs[0, j * G + g], q[b, kvh * G + g])
            assert bs[j * G + g] == beta[kvh * G + g]
    assert qs.data_ptr() == q[0, 2 * G].data_ptr()       # no copy
