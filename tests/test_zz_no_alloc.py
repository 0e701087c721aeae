"""The allocation-free entry point, infini_attn_fwd_noalloc.

Some callers may not allocate device memory while they run (a serving loop whose memory is
planned up front by its own allocator, or a host that hands plugins buffers but no right to
allocate); this entry point serves them from a fixed device array inside the library.  Its
results must match infini_attn_fwd on the same inputs, call after call, although every call
reuses the same array.  This file is collected last so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from compressive_memory_long_b200 import binding
from compressive_memory_long_b200 import workloads as wl

TOL_BF16 = 2e-2        # the bf16 tolerance of the parity tests


def rel_err(got, ref):
    g = got.double().reshape(got.shape[0] * got.shape[1], -1)
    r = ref.double().reshape(g.shape)
    return float(((g - r).abs().amax(dim=1) / r.abs().amax(dim=1).clamp_min(1e-30)).max())


def run(entry, t, w):
    out = torch.empty_like(t["q"])
    M = torch.empty((w.B, w.Hkv, w.d, w.d), dtype=torch.float32, device="cuda")
    z = torch.empty((w.B, w.Hkv, w.d), dtype=torch.float32, device="cuda")
    entry(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], out, M, z, w.N, w.rule)
    torch.cuda.synchronize()
    return out, M, z


@pytest.mark.gpu
@pytest.mark.parametrize("w", [
    wl.WORKLOADS["hf_repro_n64"],
    wl.Workload("noalloc_tc", B=1, H=4, Hkv=2, d=128, N=256, S=3, dtype="bf16", rule="delta",
                seed=31, beta_dist=("normal", 0.0, 1.0), M0_dist=("uniform", 0.0, 0.1),
                z0_dist=("uniform", 1.0, 2.0)),
    # short last segments: one more tensor-core segment; the CUDA-core tail after fused units
    wl.Workload("noalloc_tc_tail", B=1, H=4, Hkv=2, d=128, N=256, S=2, tail=100,
                dtype="bf16", rule="delta", seed=32, beta_dist=("normal", 0.0, 1.0)),
    wl.Workload("noalloc_fused_tail", B=2, H=4, Hkv=4, d=64, N=64, S=6, tail=21,
                dtype="bf16", rule="linear", seed=33, beta_dist=("normal", 0.0, 1.0),
                M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0)),
], ids=lambda w: w.name)
def test_noalloc_matches_allocating_entry_point(w):
    assert binding.infini_attn_workspace_bytes(w.B, w.Hkv, w.L, w.N, w.d) <= \
        binding.NOALLOC_SCRATCH_BYTES
    t = {k: (None if x is None else x.cuda()) for k, x in wl.torch_inputs(w).items()}
    ref = run(binding.infini_attn_fwd, t, w)
    for _ in range(2):       # two calls in a row share (and overwrite) the fixed array
        got = run(binding.infini_attn_fwd_noalloc, t, w)
        for a, b in zip(got, ref):
            assert rel_err(a, b) <= TOL_BF16
    assert binding.infini_attn_device_status() == 0


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_its_array():
    """A workspace larger than the fixed array is refused before anything is launched."""
    w = wl.WORKLOADS["stream1m_n2048_delta"]
    assert binding.infini_attn_workspace_bytes(w.B, w.Hkv, w.L, w.N, w.d) > \
        binding.NOALLOC_SCRATCH_BYTES
    base, gap = 1 << 40, 1 << 36       # disjoint fake ranges: never dereferenced
    ptrs = [ctypes.c_void_p(base + i * gap) for i in range(9)]
    rc = binding.LIB.infini_attn_fwd_noalloc(*ptrs, w.B, w.H, w.Hkv, w.L, w.N, w.d, 1, None)
    assert rc == 2          # INFINI_ERR_UNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["hf_repro_n64"])
def test_noalloc_call_replays_as_cuda_graph(name):
    """The call captured once in a CUDA graph (as the benchmark times launch-bound
    workloads) and replayed gives the eager call's results, bit for bit."""
    w = wl.WORKLOADS[name]
    t = {k: (None if x is None else x.cuda()) for k, x in wl.torch_inputs(w).items()}
    ref = run(binding.infini_attn_fwd_noalloc, t, w)
    out = torch.empty_like(t["q"])
    M = torch.empty((w.B, w.Hkv, w.d, w.d), dtype=torch.float32, device="cuda")
    z = torch.empty((w.B, w.Hkv, w.d), dtype=torch.float32, device="cuda")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        binding.infini_attn_fwd_noalloc(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"],
                                        out, M, z, w.N, w.rule)
    for _ in range(3):
        out.zero_()
        M.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref[0]) and torch.equal(M, ref[1]) and torch.equal(z, ref[2])
    del g
    assert binding.infini_attn_device_status() == 0
