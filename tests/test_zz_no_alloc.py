"""The allocation-free entry point, infini_attn_fwd_noalloc.

Some callers may not allocate device memory while they run (a serving loop whose memory is
planned up front by its own allocator, or a host that hands plugins buffers but no right to
allocate); this entry point serves them from a fixed device array inside the library.  Its
results must equal infini_attn_fwd's on the same inputs, call after call, although every
call reuses the same array and finds there whatever the previous call left.  This file is
collected last so that a run stopping at the first failure has already run every other test.
"""
import ctypes

import pytest
import torch

from compressive_memory_long_b200 import binding
from compressive_memory_long_b200 import workloads as wl


def run(entry, t, w):
    out = torch.empty_like(t["q"])
    M = torch.empty((w.B, w.Hkv, w.d, w.d), dtype=torch.float32, device="cuda")
    z = torch.empty((w.B, w.Hkv, w.d), dtype=torch.float32, device="cuda")
    entry(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], out, M, z, w.N, w.rule)
    torch.cuda.synchronize()
    return out, M, z


def inputs(w):
    return {k: (None if x is None else x.cuda()) for k, x in wl.torch_inputs(w).items()}


def rel_err(got, ref):
    g = got.double().reshape(got.shape[0] * got.shape[1], -1)
    r = ref.double().reshape(g.shape)
    return float(((g - r).abs().amax(dim=1) / r.abs().amax(dim=1).clamp_min(1e-30)).max())


_STATE = dict(M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0))
# Every path below sums in a fixed order, so the two entry points agree bit for bit.
DETERMINISTIC = [
    # fused 64-token per-unit kernel (few units per head: direct sums of the aggregates)
    wl.WORKLOADS["hf_repro_n64"].replace(name="noalloc_fused", **_STATE),
    # tensor-core segment kernel + delta chain
    wl.Workload("noalloc_tc", B=1, H=4, Hkv=2, d=128, N=256, S=3, dtype="bf16", rule="delta",
                seed=31, beta_dist=("normal", 0.0, 1.0), **_STATE),
    # tensor-core path, additive rule, and a short last segment run as one more segment
    wl.Workload("noalloc_tc_tail", B=1, H=4, Hkv=2, d=64, N=256, S=2, tail=100,
                dtype="bf16", rule="linear", seed=32, beta_dist=("normal", 0.0, 1.0)),
    # the fused units followed by the CUDA-core tail
    wl.Workload("noalloc_fused_tail", B=2, H=4, Hkv=4, d=64, N=64, S=6, tail=21,
                dtype="bf16", rule="linear", seed=33, beta_dist=("normal", 0.0, 1.0), **_STATE),
    # CUDA-core kernels: grouped heads at N = 64, delta rule
    wl.Workload("noalloc_simt", B=1, H=4, Hkv=2, d=64, N=64, S=5, dtype="bf16", rule="delta",
                seed=34, beta_dist=("normal", 0.0, 1.0), **_STATE),
]


@pytest.mark.gpu
@pytest.mark.parametrize("w", DETERMINISTIC, ids=lambda w: w.name)
def test_noalloc_equals_allocating_entry_point(w):
    """Calls alternate between two input sets of the same shape (other seeds, other initial
    memories), with a call of another shape in between, so a workspace byte that a call
    reads without writing it first would carry the previous call's data into the results.
    Each call must equal infini_attn_fwd on its own inputs exactly."""
    set_a = inputs(w)
    set_b = inputs(w.replace(seed=w.seed + 100, M0_dist=("uniform", 0.0, 0.3),
                             z0_dist=("uniform", 0.5, 3.0)))
    other = DETERMINISTIC[(DETERMINISTIC.index(w) + 1) % len(DETERMINISTIC)]
    set_o = inputs(other)
    ref_a = run(binding.infini_attn_fwd, set_a, w)
    ref_b = run(binding.infini_attn_fwd, set_b, w)
    ref_o = run(binding.infini_attn_fwd, set_o, other)
    for t, ww, ref in ((set_a, w, ref_a), (set_b, w, ref_b), (set_o, other, ref_o),
                       (set_a, w, ref_a), (set_b, w, ref_b)):
        got = run(binding.infini_attn_fwd_noalloc, t, ww)
        for name, a, b in zip(("out", "M_out", "z_out"), got, ref):
            assert torch.equal(a, b), f"{ww.name}: {name} differs (rel {rel_err(a, b):.3e})"
    assert binding.infini_attn_device_status() == 0


@pytest.mark.gpu
def test_noalloc_piece_kernel_path():
    """Long heads of 64-token segments run on the persistent piece kernel, whose look-back
    may sum the earlier pieces' memories in a different order from call to call: the memory
    agrees to fp32 rounding and the output to one bf16 step, on alternating inputs."""
    w = wl.Workload("noalloc_pieces", B=1, H=2, Hkv=2, d=64, N=64, S=64, dtype="bf16",
                    rule="linear", seed=35, beta_dist=("normal", 0.0, 1.0), **_STATE)
    sets = [inputs(w), inputs(w.replace(seed=w.seed + 100))]
    refs = [run(binding.infini_attn_fwd, t, w) for t in sets]
    for i in (0, 1, 0, 1):
        got = run(binding.infini_attn_fwd_noalloc, sets[i], w)
        assert rel_err(got[1], refs[i][1]) <= 1e-5 and rel_err(got[2], refs[i][2]) <= 1e-5
        assert rel_err(got[0], refs[i][0]) <= 2 ** -7
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
    t = inputs(w)
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
