"""The sharding helpers run through the CUDA library, on a one-rank NCCL group.

Head/batch sharding (headpar) with a single rank is the whole problem, reshaped as one
problem of B*Hkv chains: it must equal the plain forward bit for bit.  Sequence sharding of
the additive rule (seqpar) with a single rank runs its increment, its all-gather and its
forward: the outputs equal the plain forward exactly, and the final memory (M0 plus the
increment, not the forward's running memory) matches the oracle at the bf16 bound.
"""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from compressive_memory_long_b200 import binding, headpar, seqpar
from compressive_memory_long_b200 import workloads as wl

pytestmark = pytest.mark.gpu

_STATE = dict(M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0))
CASES = [
    wl.Workload("shard_tc_delta", B=2, H=4, Hkv=2, d=128, N=256, S=2, dtype="bf16",
                rule="delta", seed=81, beta_dist=("normal", 0.0, 1.0), **_STATE),
    wl.Workload("shard_tc_linear", B=2, H=6, Hkv=3, d=64, N=128, S=3, tail=50, dtype="bf16",
                rule="linear", seed=82, beta_dist=("normal", 0.0, 1.0), **_STATE),
    wl.Workload("shard_fused", B=2, H=4, Hkv=4, d=64, N=64, S=4, dtype="bf16", rule="linear",
                seed=83, beta_dist=("normal", 0.0, 1.0), **_STATE),
]


def rel_err(got, ref):
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    g = g.reshape(g.shape[0] * g.shape[1], -1)
    r = r.reshape(g.shape)
    return float((np.abs(g - r).max(axis=1) / np.maximum(np.abs(r).max(axis=1), 1e-30)).max())


@pytest.fixture(scope="module")
def one_rank_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_head_sharded_forward_on_one_rank(one_rank_group, w):
    t = {k: (None if x is None else x.cuda()) for k, x in wl.torch_inputs(w).items()}
    ref = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                          rule=w.rule)
    got = headpar.forward_head_sharded(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"],
                                       N=w.N, rule=w.rule)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert a.shape == b.shape and torch.equal(a, b)
    assert binding.infini_attn_device_status() == 0


@pytest.mark.parametrize("w", [c for c in CASES if c.rule == "linear"], ids=lambda w: w.name)
def test_sequence_parallel_forward_on_one_rank(one_rank_group, w):
    t = {k: (None if x is None else x.cuda()) for k, x in wl.torch_inputs(w).items()}
    ref_out, ref_M, ref_z = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"],
                                            t["z0"], N=w.N, rule="linear")
    out, M, z = seqpar.forward_sequence_parallel(t["q"], t["k"], t["v"], t["beta"], t["M0"],
                                                 t["z0"], N=w.N, rule="linear")
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)
    # the final memory is M0 plus the increment from the state call (its own kernels), the
    # forward's is its running memory: both must match the oracle at the bf16 bound
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    _, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=w.N, rule="linear")
    assert rel_err(M.cpu(), rM) <= 2e-2 and rel_err(ref_M.cpu(), rM) <= 2e-2
    assert rel_err(z.cpu()[:, :, None], rz[:, :, None]) <= 2e-2
    assert binding.infini_attn_device_status() == 0
