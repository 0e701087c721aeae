"""Failure paths, made to happen on purpose without a real failure and without faulting,
trapping or hanging the GPU: the workspace allocation fails (a host-side hook), and a
bounded device wait runs out (a test hook withholds one publish and shortens the wait
limit; the waiting kernel gives up, records the timeout and returns)."""
import numpy as np
import pytest
import torch

import oracle
from compressive_memory_long_b200 import binding
from compressive_memory_long_b200 import workloads as wl

pytestmark = pytest.mark.gpu

_STATE = dict(M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0))
ALLOCATING = [
    # tensor-core path (memory increments + recurrence + segment kernel)
    wl.Workload("oom_tc", B=1, H=4, Hkv=2, d=128, N=256, S=2, dtype="bf16", rule="delta",
                seed=61, beta_dist=("normal", 0.0, 1.0), **_STATE),
    # CUDA-core path
    wl.Workload("oom_simt", B=1, H=4, Hkv=2, d=32, N=64, S=3, dtype="bf16", rule="linear",
                seed=62, beta_dist=("normal", 0.0, 1.0), **_STATE),
    # fused 64-token kernel (its own small workspace)
    wl.Workload("oom_fused", B=1, H=2, Hkv=2, d=64, N=64, S=4, dtype="bf16", rule="linear",
                seed=63, beta_dist=("normal", 0.0, 1.0), **_STATE),
]


def inputs(w):
    return {k: (None if x is None else x.cuda()) for k, x in wl.torch_inputs(w).items()}


def rel_err(got, ref):
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    g = g.reshape(g.shape[0] * g.shape[1], -1)
    r = r.reshape(g.shape)
    return float((np.abs(g - r).max(axis=1) / np.maximum(np.abs(r).max(axis=1), 1e-30)).max())


@pytest.mark.parametrize("w", ALLOCATING, ids=lambda w: w.name)
def test_failed_workspace_allocation_writes_nothing(w):
    t = inputs(w)
    out = torch.full_like(t["q"], 7.0)
    M = torch.full((w.B, w.Hkv, w.d, w.d), 7.0, device="cuda")
    z = torch.full((w.B, w.Hkv, w.d), 7.0, device="cuda")
    assert binding.infini_attn_test_fail_allocations(1) == 0
    try:
        with pytest.raises(binding.InfiniError) as e:
            binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                            rule=w.rule, out=out, M_out=M, z_out=z)
    finally:
        binding.infini_attn_test_fail_allocations(0)
    assert e.value.status == 4                          # INFINI_ERR_OOM
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()) and bool((M == 7.0).all()) and bool((z == 7.0).all())
    # the hook is spent: the same call now runs
    got = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                          rule=w.rule, out=out, M_out=M, z_out=z)
    ref = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                          rule=w.rule)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    assert binding.infini_attn_device_status() == 0


def test_failed_allocation_in_the_state_call():
    w = ALLOCATING[0]
    t = inputs(w)
    M = torch.full((w.B, w.Hkv, w.d, w.d), 7.0, device="cuda")
    z = torch.full((w.B, w.Hkv, w.d), 7.0, device="cuda")
    binding.infini_attn_test_fail_allocations(1)
    try:
        with pytest.raises(binding.InfiniError) as e:
            binding.state(t["k"], t["v"], t["M0"], t["z0"], N=w.N, rule=w.rule, M_out=M, z_out=z)
    finally:
        binding.infini_attn_test_fail_allocations(0)
    assert e.value.status == 4
    torch.cuda.synchronize()
    assert bool((M == 7.0).all()) and bool((z == 7.0).all())


def test_allocation_free_call_leaves_the_allocation_hook_alone():
    """infini_attn_fwd_noalloc allocates nothing, so an armed allocation failure stays armed
    for the next allocating call."""
    w = ALLOCATING[0]
    t = inputs(w)
    out = torch.empty_like(t["q"])
    M = torch.empty((w.B, w.Hkv, w.d, w.d), device="cuda")
    z = torch.empty((w.B, w.Hkv, w.d), device="cuda")
    binding.infini_attn_test_fail_allocations(1)
    try:
        binding.infini_attn_fwd_noalloc(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], out,
                                        M, z, w.N, w.rule)
        with pytest.raises(binding.InfiniError) as e:
            binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                            rule=w.rule)
        assert e.value.status == 4
    finally:
        binding.infini_attn_test_fail_allocations(0)
    assert binding.infini_attn_device_status() == 0


def test_bounded_wait_runs_out_and_is_reported():
    """The first unit of every head withholds its publish; the later units wait for it, give
    up after the (shortened) limit, record INFINI_ERR_TIMEOUT and return.  The status is read
    once, then cleared, and the same call afterwards is correct."""
    w = ALLOCATING[2]          # 2 units of 128 tokens per head: the fused kernel, direct sums
    t = inputs(w)
    binding.infini_attn_trace_enable(True)
    assert binding.infini_attn_test_wait_limit(1 << 20) == 0      # about half a millisecond
    assert binding.infini_attn_test_withhold_publish(True) == 0
    try:
        binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N, rule=w.rule)
        status = binding.infini_attn_device_status()
    finally:
        binding.infini_attn_test_withhold_publish(False)
        binding.infini_attn_test_wait_limit(0)
        binding.infini_attn_trace_enable(False)
    assert list(binding.infini_attn_trace_report()) == ["small_fused"]
    assert status == 5                                  # INFINI_ERR_TIMEOUT
    assert binding.infini_attn_device_status() == 0     # read once, then cleared
    out, M, z = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                                rule=w.rule)
    torch.cuda.synchronize()
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    ro, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=w.N, rule=w.rule)
    errs = (rel_err(out.float().cpu(), ro), rel_err(M.cpu(), rM),
            rel_err(z.cpu()[:, :, None], rz[:, :, None]))
    assert max(errs) <= 2e-2, errs
    assert binding.infini_attn_device_status() == 0
