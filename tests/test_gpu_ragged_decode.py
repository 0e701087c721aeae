"""A final segment shorter than N, and the token-by-token decode step, against the fp64
oracle through the C ABI.

The oracle processes a last segment of L mod N tokens like any other (its own reading of
fixed-size segments); the decode step must give the forward's output for every token and,
after the last fold, its memory.  Tolerances as in the other parity tests: 1e-4 (fp32
activations), 2e-2 (bf16), max relative error per (batch, head) slice.
"""
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
    num = np.abs(g - r).max(axis=1)
    den = np.maximum(np.abs(r).max(axis=1), 1e-30)
    return float((num / den).max())


def make(name, *, B, H, Hkv, d, N, S, tail, dtype="bf16", rule="linear", state=False, seed=0):
    kw = dict(M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0)) if state else {}
    return wl.Workload(name, B=B, H=H, Hkv=Hkv, d=d, N=N, S=S, tail=tail, dtype=dtype,
                       rule=rule, seed=seed, beta_dist=("normal", 0.0, 1.5), **kw)


def oracle_run(w):
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    st = wl.has_initial_state(w)
    return oracle.infini_attn_fwd(q, k, v, beta, M0 if st else None, z0 if st else None, N=w.N,
                                  rule=w.rule)


def dev_inputs(w):
    return {k: (None if x is None else x.cuda()) for k, x in wl.torch_inputs(w).items()}


# (workload, a kernel that must run, whether the CUDA-core tail runs).  On the tensor-core
# path (bf16, d in {64, 128}, N % 128 == 0 or N = 64) the short segment is one more segment
# of the tensor-core kernels; after the fused 64-token kernels (additive rule, d = 64, whole
# 128-token units) and elsewhere the CUDA-core tail follows the full segments.
RAGGED = [
    (make("fused64", B=2, H=4, Hkv=4, d=64, N=64, S=6, tail=37, seed=11), "small_fused", True),
    (make("pieces64", B=1, H=2, Hkv=2, d=64, N=64, S=40, tail=1, state=True, seed=12),
     "small_pieces", True),
    (make("fused64_gqa", B=1, H=4, Hkv=2, d=64, N=64, S=6, tail=37, state=True, seed=26),
     "small_fused", True),
    (make("pieces64_gqa", B=1, H=6, Hkv=3, d=64, N=64, S=34, tail=63, seed=27),
     "small_pieces", True),
    (make("odd_s64", B=1, H=2, Hkv=2, d=64, N=64, S=3, tail=50, seed=13), "segment_tc", False),
    (make("tc_delta_n64", B=1, H=4, Hkv=2, d=64, N=64, S=5, tail=20, rule="delta", state=True,
          seed=28), "mem_chain", False),
    (make("tc_n64_d128", B=2, H=2, Hkv=1, d=128, N=64, S=2, tail=63, seed=29), "segment_tc",
     False),
    (make("simt_d32", B=1, H=2, Hkv=2, d=32, N=64, S=2, tail=10, seed=17), "segment_simt", True),
    (make("f32_delta", B=1, H=2, Hkv=2, d=64, N=64, S=2, tail=33, dtype="f32", rule="delta",
          state=True, seed=18), "delta_chain", True),
    (make("only_tail_f32", B=2, H=2, Hkv=2, d=32, N=128, S=0, tail=5, dtype="f32", seed=20),
     "tail_segment", True),
    (make("one_token", B=1, H=1, Hkv=1, d=64, N=64, S=0, tail=1, state=True, seed=21),
     "tail_segment", True),
    (make("tc2_delta", B=1, H=4, Hkv=2, d=128, N=256, S=2, tail=100, rule="delta", seed=14),
     "mem_chain", False),
    (make("tc2_delta_long", B=1, H=2, Hkv=2, d=128, N=768, S=1, tail=520, rule="delta",
          seed=23), "segment_tc", False),
    (make("tc_linear", B=2, H=2, Hkv=2, d=128, N=128, S=3, tail=127, state=True, seed=15),
     "mem_prefix", False),
    (make("tc_linear64", B=1, H=3, Hkv=3, d=64, N=256, S=1, tail=129, state=True, seed=24),
     "mem_prefix", False),
    (make("tc_delta64", B=1, H=2, Hkv=1, d=64, N=128, S=2, tail=64, rule="delta", seed=16),
     "mem_chain", False),
    (make("only_tail", B=1, H=2, Hkv=1, d=128, N=256, S=0, tail=200, rule="delta", state=True,
          seed=19), "segment_tc", False),
    (make("only_tail_linear", B=1, H=2, Hkv=2, d=64, N=512, S=0, tail=3, seed=25),
     "mem_prefix", False),
]


@pytest.mark.parametrize("w,main,simt_tail", RAGGED, ids=[r[0].name for r in RAGGED])
def test_ragged_last_segment(w, main, simt_tail):
    from compressive_memory_long_b200 import binding
    t = dev_inputs(w)
    binding.infini_attn_trace_enable(True)
    out, M, z = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                                rule=w.rule)
    torch.cuda.synchronize()
    binding.infini_attn_trace_enable(False)
    names = list(binding.infini_attn_trace_report())
    assert main in names, names
    assert ("tail_segment" in names) == simt_tail, names
    ro, rM, rz = oracle_run(w)
    errs = (rel_err(out.float().cpu(), ro), rel_err(M.cpu(), rM),
            rel_err(z.cpu()[:, :, None], rz[:, :, None]))
    assert max(errs) <= TOL[w.dtype], f"{w.name}: out/M/z rel err {errs}"
    assert binding.infini_attn_device_status() == 0


@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_ragged_in_place_state(rule):
    """M_out / z_out aliasing M0 / z0 with a final short segment (the tail reads the state
    the full segments wrote into the same buffers)."""
    from compressive_memory_long_b200 import binding
    w = make("ragged_in_place", B=1, H=4, Hkv=2, d=128, N=128, S=2, tail=77, rule=rule,
             state=True, seed=22)
    t = dev_inputs(w)
    M, z = t["M0"].clone(), t["z0"].clone()
    out, _, _ = binding.forward(t["q"], t["k"], t["v"], t["beta"], M, z, N=w.N, rule=rule,
                                M_out=M, z_out=z)
    torch.cuda.synchronize()
    ro, rM, rz = oracle_run(w)
    errs = (rel_err(out.float().cpu(), ro), rel_err(M.cpu(), rM),
            rel_err(z.cpu()[:, :, None], rz[:, :, None]))
    assert max(errs) <= TOL[w.dtype], errs


DECODE = [
    make("dec_bf16_linear", B=2, H=4, Hkv=2, d=64, N=64, S=2, tail=22, state=True, seed=31),
    make("dec_bf16_delta", B=1, H=2, Hkv=2, d=128, N=64, S=1, tail=36, rule="delta", seed=32),
    make("dec_f32_delta", B=1, H=2, Hkv=1, d=32, N=16, S=2, tail=8, dtype="f32", rule="delta",
         state=True, seed=33),
    make("dec_f32_linear", B=1, H=3, Hkv=3, d=64, N=10, S=3, tail=5, dtype="f32", seed=34),
    make("dec_exact_segments", B=1, H=2, Hkv=2, d=64, N=32, S=3, tail=0, rule="delta", seed=35),
    # keys split over clusters of 8 CTAs, two tiles of keys per CTA near the segment's end
    make("dec_long_cluster", B=1, H=8, Hkv=2, d=128, N=2100, S=1, tail=70, rule="delta",
         state=True, seed=38),
    make("dec_f32_multitile", B=1, H=2, Hkv=1, d=64, N=1100, S=1, tail=3, dtype="f32",
         seed=41),
    # a group of 8 query heads (the widest one cluster CTA takes), odd N, clusters of 2
    make("dec_g8", B=2, H=16, Hkv=2, d=32, N=300, S=1, tail=50, seed=39),
    # a group of 16 query heads: one CTA per query head instead
    make("dec_g16", B=1, H=16, Hkv=1, d=64, N=64, S=1, tail=10, seed=40),
]


@pytest.mark.parametrize("w", DECODE, ids=[w.name for w in DECODE])
def test_decode_matches_forward(w):
    """Feed the sequence one token at a time; the outputs are the forward's, and after the
    fold of the rows still cached the memory is the forward's M_out / z_out."""
    from compressive_memory_long_b200 import binding
    t = dev_inputs(w)
    B, Hkv, d = w.B, w.Hkv, w.d
    dt = w.torch_dtype
    kc = torch.zeros((B, Hkv, w.N, d), dtype=dt, device="cuda")
    vc = torch.zeros_like(kc)
    M = (t["M0"].clone() if t["M0"] is not None
         else torch.zeros((B, Hkv, d, d), dtype=torch.float32, device="cuda"))
    z = (t["z0"].clone() if t["z0"] is not None
         else torch.zeros((B, Hkv, d), dtype=torch.float32, device="cuda"))
    outs = []
    for tok in range(w.L):
        pos = tok % w.N
        o = binding.decode_step(t["q"][:, :, tok].contiguous(), t["k"][:, :, tok].contiguous(),
                                t["v"][:, :, tok].contiguous(), t["beta"], kc, vc, pos, M, z,
                                rule=w.rule)
        outs.append(o)
    binding.fold(kc, vc, w.L % w.N, M, z, rule=w.rule)
    torch.cuda.synchronize()
    got = torch.stack(outs, dim=2).float().cpu()
    ro, rM, rz = oracle_run(w)
    errs = (rel_err(got, ro), rel_err(M.cpu(), rM), rel_err(z.cpu()[:, :, None], rz[:, :, None]))
    assert max(errs) <= TOL[w.dtype], f"{w.name}: out/M/z rel err {errs}"
    assert binding.infini_attn_device_status() == 0


def test_decode_continues_a_forward():
    """A forward over whole segments, then decode from its M_out / z_out: the same outputs
    as one forward over the whole sequence."""
    from compressive_memory_long_b200 import binding
    w = make("dec_after_fwd", B=1, H=4, Hkv=4, d=64, N=64, S=4, tail=40, seed=36)
    t = dev_inputs(w)
    pre = 3 * w.N
    _, M, z = binding.forward(t["q"][:, :, :pre].contiguous(), t["k"][:, :, :pre].contiguous(),
                              t["v"][:, :, :pre].contiguous(), t["beta"], N=w.N, rule=w.rule)
    kc = torch.zeros((w.B, w.Hkv, w.N, w.d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    outs = []
    for tok in range(pre, w.L):
        outs.append(binding.decode_step(t["q"][:, :, tok].contiguous(),
                                        t["k"][:, :, tok].contiguous(),
                                        t["v"][:, :, tok].contiguous(), t["beta"], kc, vc,
                                        tok % w.N, M, z, rule=w.rule))
    binding.fold(kc, vc, w.L % w.N, M, z, rule=w.rule)
    torch.cuda.synchronize()
    ro, rM, rz = oracle_run(w)
    got = torch.stack(outs, dim=2).float().cpu()
    errs = (rel_err(got, ro[:, :, pre:]), rel_err(M.cpu(), rM),
            rel_err(z.cpu()[:, :, None], rz[:, :, None]))
    assert max(errs) <= TOL["bf16"], errs


@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_decode_segment_in_cuda_graph(rule):
    """The calls of one segment (the fold included) allocate nothing, so they can be
    captured in a CUDA graph; a replay from the same starting state gives the eager
    results exactly."""
    from compressive_memory_long_b200 import binding
    w = make("dec_graph", B=2, H=4, Hkv=2, d=128, N=64, S=1, tail=0, rule=rule, state=True,
             seed=37)
    t = dev_inputs(w)
    q, k, v = (t[n].permute(2, 0, 1, 3).contiguous() for n in ("q", "k", "v"))
    kc = torch.zeros((w.B, w.Hkv, w.N, w.d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    M, z = t["M0"].clone(), t["z0"].clone()
    outs = torch.empty((w.N, w.B, w.H, w.d), dtype=torch.bfloat16, device="cuda")

    def calls():
        for p in range(w.N):
            binding.decode_step(q[p], k[p], v[p], t["beta"], kc, vc, p, M, z, rule=rule,
                                out=outs[p])

    calls()
    torch.cuda.synchronize()
    eager = (outs.clone(), M.clone(), z.clone())
    g = torch.cuda.CUDAGraph()
    M.copy_(t["M0"])
    z.copy_(t["z0"])
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        calls()
    M.copy_(t["M0"])
    z.copy_(t["z0"])
    outs.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(outs, eager[0]) and torch.equal(M, eager[1]) and torch.equal(z, eager[2])
    ro, rM, rz = oracle_run(w)
    got = outs.permute(1, 2, 0, 3).float().cpu()
    errs = (rel_err(got, ro), rel_err(M.cpu(), rM), rel_err(z.cpu()[:, :, None], rz[:, :, None]))
    assert max(errs) <= TOL["bf16"], errs
    del g
