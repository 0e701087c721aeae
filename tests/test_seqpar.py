"""One sequence cut across ranks under the additive rule (compressive_memory_long_b200.seqpar).

On CPU: two gloo ranks run the sharded forward with the fp64 oracle standing in for the
per-rank compute (test infrastructure only; the product default is the CUDA library), and
their outputs and final memory must equal one oracle run over the whole sequence.  The
exchange, the prefix of earlier chunks and the chunk-boundary rule are what is tested here.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from compressive_memory_long_b200 import workloads as wl


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_fns():
    import oracle

    def state_fn(k, v, N, rule):
        B, Hkv, L, d = k.shape
        q = np.zeros((B, Hkv, L, d), np.float32)
        _, M, z = oracle.infini_attn_fwd(q, k.numpy(), v.numpy(), np.zeros(Hkv, np.float32),
                                         N=N, rule=rule)
        return torch.from_numpy(M), torch.from_numpy(z)

    def forward_fn(q, k, v, beta, M0, z0, N, rule):
        out, M, z = oracle.infini_attn_fwd(q.numpy(), k.numpy(), v.numpy(), beta.numpy(),
                                           M0.numpy().astype(np.float32),
                                           z0.numpy().astype(np.float32), N=N, rule=rule)
        return torch.from_numpy(out), torch.from_numpy(M), torch.from_numpy(z)

    return state_fn, forward_fn


W = wl.Workload("seqpar", B=2, H=4, Hkv=2, d=16, N=8, S=5, tail=3, dtype="f32", rule="linear",
                seed=51, beta_dist=("normal", 0.0, 1.0), M0_dist=("uniform", 0.0, 0.1),
                z0_dist=("uniform", 1.0, 2.0))
CUTS2 = [0, 16, 43]         # rank 0: tokens 0-15 (two segments), rank 1: 16-42 (ragged end)
CUTS3 = [0, 8, 32, 43]      # one, three and 1 3/8 segments


def _rank_main(rank, world, port, results, CUTS=CUTS2):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from compressive_memory_long_b200 import seqpar
        q, k, v, beta, M0, z0 = (torch.from_numpy(x) for x in wl.host_inputs(W))
        sl = slice(CUTS[rank], CUTS[rank + 1])
        state_fn, forward_fn = _oracle_fns()
        out, M, z = seqpar.forward_sequence_parallel(
            q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(), beta,
            M0.double(), z0.double(), N=W.N, rule="linear", state_fn=state_fn,
            forward_fn=forward_fn)
        results[rank] = (out.numpy(), M.numpy(), z.numpy())
        if rank == 0:       # a chunk before the last must end on a segment boundary
            try:
                seqpar.forward_sequence_parallel(q[:, :, :5], k[:, :, :5], v[:, :, :5], beta,
                                                 N=W.N, state_fn=state_fn, forward_fn=forward_fn)
                results["boundary"] = "accepted"
            except ValueError:
                results["boundary"] = "rejected"
        try:
            seqpar.forward_sequence_parallel(q, k, v, beta, N=W.N, rule="delta")
            results[f"delta{rank}"] = "accepted"
        except ValueError:
            results[f"delta{rank}"] = "rejected"
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [CUTS2, CUTS3], ids=["2ranks", "3ranks"])
def test_sequence_split_equals_one_run(cuts):
    import oracle
    world, port = len(cuts) - 1, _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results, cuts))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    q, k, v, beta, M0, z0 = wl.host_inputs(W)
    ro, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=W.N, rule="linear")
    # the oracle takes its initial memory in fp32, so rank 1's prefix is rounded to fp32 once
    got = np.concatenate([results[r][0] for r in range(world)], axis=2)
    np.testing.assert_allclose(got, ro, rtol=1e-6, atol=1e-9)
    for r in range(world):          # every rank ends with the memory after the whole sequence
        np.testing.assert_allclose(results[r][1], rM, rtol=1e-6, atol=1e-9)
        np.testing.assert_allclose(results[r][2], rz, rtol=1e-6, atol=1e-9)
    assert results["boundary"] == "rejected"
    assert all(results[f"delta{r}"] == "rejected" for r in range(world))
