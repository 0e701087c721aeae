"""The state-only entry point (infini_attn_state) against the fp64 oracle, and a sequence cut
in two chunks run through the library the way sequence sharding runs it (increment of the
first chunk, then the forward of the second from M0 plus that increment)."""
import numpy as np
import pytest
import torch

import oracle
from compressive_memory_long_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    g = got.reshape(got.shape[0] * got.shape[1], -1)
    r = ref.reshape(g.shape)
    return float((np.abs(g - r).max(axis=1) / np.maximum(np.abs(r).max(axis=1), 1e-30)).max())


def make(name, *, B, H, Hkv, d, N, S, tail=0, dtype="bf16", rule="linear", state=False, seed=0):
    kw = dict(M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0)) if state else {}
    return wl.Workload(name, B=B, H=H, Hkv=Hkv, d=d, N=N, S=S, tail=tail, dtype=dtype,
                       rule=rule, seed=seed, beta_dist=("normal", 0.0, 1.0), **kw)


CASES = [
    make("lin_tc", B=2, H=2, Hkv=2, d=128, N=128, S=3, state=True, seed=61),
    make("delta_tc", B=1, H=2, Hkv=2, d=128, N=256, S=2, rule="delta", seed=62),
    make("lin_n64_mha", B=2, H=4, Hkv=4, d=64, N=64, S=6, seed=63),       # fused-eligible shape
    make("lin_tc_tail", B=1, H=2, Hkv=2, d=64, N=128, S=2, tail=77, state=True, seed=64),
    make("delta_simt_tail", B=1, H=2, Hkv=2, d=32, N=64, S=2, tail=9, rule="delta", seed=65),
    make("f32_delta", B=1, H=2, Hkv=2, d=64, N=64, S=3, dtype="f32", rule="delta", state=True,
         seed=66),
    make("only_tail", B=1, H=2, Hkv=2, d=128, N=512, S=0, tail=100, rule="delta", seed=67),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_state_equals_forward_memory(w):
    from compressive_memory_long_b200 import binding
    t = {k: (None if x is None else x.cuda()) for k, x in wl.torch_inputs(w).items()}
    binding.infini_attn_trace_enable(True)
    M, z = binding.state(t["k"], t["v"], t["M0"], t["z0"], N=w.N, rule=w.rule)
    torch.cuda.synchronize()
    binding.infini_attn_trace_enable(False)
    names = list(binding.infini_attn_trace_report())
    assert not any(n.startswith(("segment", "small", "tail_segment")) for n in names), names
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    st = wl.has_initial_state(w)
    _, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0 if st else None, z0 if st else None,
                                       N=w.N, rule=w.rule)
    errs = (rel_err(M.cpu(), rM), rel_err(z.cpu()[:, :, None], rz[:, :, None]))
    assert max(errs) <= TOL[w.dtype], f"{w.name}: M/z rel err {errs}"
    assert binding.infini_attn_device_status() == 0


@pytest.mark.parametrize("N,cut", [(64, 512), (128, 768)])
def test_two_chunk_split_through_the_library(N, cut):
    from compressive_memory_long_b200 import binding
    w = make("split", B=2, H=4, Hkv=4, d=64, N=N, S=1024 // N, tail=40, state=True, seed=68)
    t = {k: (None if x is None else x.cuda()) for k, x in wl.torch_inputs(w).items()}
    a, b = slice(0, cut), slice(cut, w.L)
    part = {n: (t[n][:, :, a].contiguous(), t[n][:, :, b].contiguous()) for n in ("q", "k", "v")}
    dM0, dz0 = binding.state(part["k"][0], part["v"][0], N=N, rule="linear")
    dM1, dz1 = binding.state(part["k"][1], part["v"][1], N=N, rule="linear")
    out0, _, _ = binding.forward(part["q"][0], part["k"][0], part["v"][0], t["beta"], t["M0"],
                                 t["z0"], N=N, rule="linear")
    out1, _, _ = binding.forward(part["q"][1], part["k"][1], part["v"][1], t["beta"],
                                 t["M0"] + dM0, t["z0"] + dz0, N=N, rule="linear")
    M_final, z_final = t["M0"] + dM0 + dM1, t["z0"] + dz0 + dz1
    torch.cuda.synchronize()
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    ro, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=N, rule="linear")
    got = torch.cat([out0, out1], dim=2).float().cpu()
    errs = (rel_err(got, ro), rel_err(M_final.cpu(), rM),
            rel_err(z_final.cpu()[:, :, None], rz[:, :, None]))
    assert max(errs) <= TOL["bf16"], errs


@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_memory_path_kernels_and_z_precision(rule):
    """The tensor-core memory path launches what its rule needs: the delta rule's increments
    need z_{s-1}, so the separate sigma(K) sum and the z scan run before them; the additive
    rule's increments kernel forms the segment sums itself (sigma(K)^T 1 from sigma's two bf16
    parts into an fp32 accumulator) and only the scan follows.  Either way z keeps about 16
    bits of sigma: its error is held to 5e-5, far inside the bf16 bound."""
    from compressive_memory_long_b200 import binding
    w = make(f"zpath_{rule}", B=2, H=4, Hkv=2, d=128, N=256, S=3, tail=90, rule=rule,
             state=True, seed=68)
    t = {k: (None if x is None else x.cuda()) for k, x in wl.torch_inputs(w).items()}
    binding.infini_attn_trace_enable(True)
    out, M, z = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                                rule=w.rule)
    torch.cuda.synchronize()
    binding.infini_attn_trace_enable(False)
    names = set(binding.infini_attn_trace_report())
    want = ({"z_sum", "z_scan", "mem_increments", "mem_chain"} if rule == "delta"
            else {"mem_increments", "z_scan", "mem_prefix"})
    assert want <= names, names
    assert ("z_sum" in names) == (rule == "delta"), names
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    ro, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=w.N, rule=w.rule)
    ez = rel_err(z.cpu()[:, :, None], rz[:, :, None])
    errs = (rel_err(out.float().cpu(), ro), rel_err(M.cpu(), rM), ez)
    print(f"PARITY {w.name}: out {errs[0]:.2e} M {errs[1]:.2e} z {ez:.2e}")
    assert max(errs) <= TOL["bf16"], f"{w.name}: out/M/z rel err {errs}"
    assert ez <= 5e-5, f"{w.name}: z rel err {ez}"
    assert binding.infini_attn_device_status() == 0
