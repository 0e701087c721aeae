"""GPU path vs the fp64 CPU oracle, element by element, through the C ABI.

Tolerances (max relative error per (batch, head) slice, max |x - r| / max |r|):
1e-4 for fp32 activations, 2e-2 for bf16 activations with fp32 accumulation; the same
bounds hold for out, M_out and z_out.  Full-size workloads are checked on sampled
(batch, kv head) chains: the oracle runs each sampled chain's memory over every segment
and computes outputs on sampled segments.
"""
import numpy as np
import pytest
import torch

import oracle
from compressive_memory_long_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref):
    """max over leading (batch, head) slices of max|x - r| / max|r|."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    g = got.reshape(got.shape[0] * got.shape[1], -1)
    r = ref.reshape(g.shape)
    num = np.abs(g - r).max(axis=1)
    den = np.maximum(np.abs(r).max(axis=1), 1e-30)
    return float((num / den).max())


def row_err(got, ref):
    """The same ratio per output row (one token of one head): max_j |x - r| / max_j |r|,
    the row's scale floored at 1e-6 of its slice's, so a row far smaller than the rest of
    its slice (a first segment with an empty memory under a large gate) is judged on its
    own scale."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    d = ref.shape[-1]
    g = got.reshape(got.shape[0] * got.shape[1], -1, d)
    r = ref.reshape(g.shape)
    slice_max = np.abs(r).max(axis=(1, 2), keepdims=True)[..., 0]
    scale = np.maximum(np.abs(r).max(axis=2), 1e-6 * slice_max)
    return float((np.abs(g - r).max(axis=2) / np.maximum(scale, 1e-30)).max())


def elem_err(got, ref):
    """Elementwise |x - r| / max(|r|, 1e-6 max|r| of the slice): reported, not bounded (an
    element near zero after cancellation carries the absolute error of its row)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    g = got.reshape(got.shape[0] * got.shape[1], -1)
    r = ref.reshape(g.shape)
    floor = 1e-6 * np.abs(r).max(axis=1, keepdims=True)
    return float((np.abs(g - r) / np.maximum(np.abs(r), np.maximum(floor, 1e-30))).max())


def report(name, **errs):
    """One line per check (pytest -s shows them): the achieved errors beside the bound."""
    print("PARITY " + name + " " + " ".join(f"{k}={v:.3e}" for k, v in errs.items()), flush=True)


def to_dev(t):
    return {k: (None if x is None else x.cuda()) for k, x in t.items()}


def run_gpu(w, t=None):
    from compressive_memory_long_b200 import binding
    t = to_dev(wl.torch_inputs(w) if t is None else t)
    out, M, z = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                                rule=w.rule)
    torch.cuda.synchronize()
    # a bounded wait that gave up anywhere in the launch fails here (and the sticky status is
    # read and cleared, so later tests start clean)
    assert binding.infini_attn_device_status() == 0, f"{w.name}: a device wait timed out"
    return out, M, z


def check_full(w):
    out, M, z = run_gpu(w)
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    ro, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0 if wl.has_initial_state(w) else None,
                                        z0 if wl.has_initial_state(w) else None, N=w.N,
                                        rule=w.rule)
    o = out.float().cpu()
    errs = (rel_err(o, ro), rel_err(M.cpu(), rM), rel_err(z.cpu()[:, :, None], rz[:, :, None]))
    er = row_err(o, ro)
    report(w.name, out=errs[0], M=errs[1], z=errs[2], out_row=er, out_elem=elem_err(o, ro))
    tol = TOL[w.dtype]
    assert max(errs) <= tol, f"{w.name}: out/M/z rel err {errs} > {tol}"
    assert er <= tol, f"{w.name}: per-row out rel err {er} > {tol}"
    return errs


def check_sampled(w, chains, segs):
    out, M, z = run_gpu(w)
    out_c, M_c, z_c = out.cpu(), M.cpu(), z.cpu()
    del out, M, z
    torch.cuda.empty_cache()
    tol = TOL[w.dtype]
    for (b, kvh) in chains:
        q, k, v, beta, M0, z0 = wl.host_slices(w, b, kvh)
        st = wl.has_initial_state(w)
        ro, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0 if st else None,
                                            z0 if st else None, N=w.N, rule=w.rule,
                                            seg_out=segs)
        heads = slice(kvh * w.G, (kvh + 1) * w.G)
        worst = [0.0, 0.0, 0.0]
        for s in segs:
            rows = slice(s * w.N, (s + 1) * w.N)
            o, r = out_c[b:b + 1, heads, rows].float(), ro[:, :, rows]
            e, er = rel_err(o, r), row_err(o, r)
            worst = [max(worst[0], e), max(worst[1], er), max(worst[2], elem_err(o, r))]
            assert e <= tol, f"{w.name} chain {(b, kvh)} segment {s}: out rel err {e}"
            assert er <= tol, f"{w.name} chain {(b, kvh)} segment {s}: per-row out rel err {er}"
        eM = rel_err(M_c[b:b + 1, kvh:kvh + 1], rM)
        ez = rel_err(z_c[b:b + 1, kvh:kvh + 1, None], rz[:, :, None])
        report(f"{w.name}[{b},{kvh}]", out=worst[0], M=eM, z=ez, out_row=worst[1],
               out_elem=worst[2])
        assert max(eM, ez) <= tol, f"{w.name} chain {(b, kvh)}: M/z rel err {eM}, {ez}"


@pytest.mark.parametrize("name", ["fp32_linear_small", "hf_repro_n64"])
def test_small_workloads_full(name):
    check_full(wl.WORKLOADS[name])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rule", ["linear", "delta"])
@pytest.mark.parametrize("d", [32, 64, 128])
def test_shapes_and_rules(dtype, rule, d):
    """Several q tiles per segment, several segments, GQA, a nonzero initial state."""
    w = wl.Workload("t", B=2, H=4, Hkv=2, d=d, N=192, S=3, dtype=dtype, rule=rule, seed=11,
                    beta_dist=("normal", 0.0, 1.5), M0_dist=("uniform", 0.0, 0.1),
                    z0_dist=("uniform", 1.0, 2.0))
    check_full(w)


@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_gqa8b_sampled(rule):
    w = wl.WORKLOADS["gqa8b_n2048_delta"].replace(rule=rule)
    check_sampled(w, chains=[(0, 3)], segs=[0, 1, 15])


def test_gqa8b_short_last_segment_sampled():
    """The 8B-class layout with a 1000-token seventeenth segment (run on the tensor-core
    kernels as one more segment): the first and the short segment of two chains."""
    w = wl.WORKLOADS["gqa8b_n2048_delta"].replace(name="gqa8b_tail1000", tail=1000)
    check_sampled(w, chains=[(0, 0), (0, 7)], segs=[0, 16])


def test_stream1m_sampled():
    w = wl.WORKLOADS["stream1m_n2048_delta"]
    check_sampled(w, chains=[(0, 7)], segs=[0, 1, 511])


def test_batched_sampled():
    w = wl.WORKLOADS["batched_n1024_linear"]
    check_sampled(w, chains=[(0, 0), (15, 31)], segs=[0, 3, 7])


# ---- properties of the boundary on the device ---------------------------------------

def test_null_state_equals_zero_state():
    from compressive_memory_long_b200 import binding
    w = wl.WORKLOADS["hf_repro_n64"].replace(rule="delta", S=3)
    t = to_dev(wl.torch_inputs(w))
    a = binding.forward(t["q"], t["k"], t["v"], t["beta"], None, None, N=w.N, rule=w.rule)
    Z = torch.zeros(w.B, w.Hkv, w.d, w.d, device="cuda")
    zz = torch.zeros(w.B, w.Hkv, w.d, device="cuda")
    b = binding.forward(t["q"], t["k"], t["v"], t["beta"], Z, zz, N=w.N, rule=w.rule)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_in_place_state_and_streaming_split(rule):
    """Running [0, L1) then [L1, L) with the state updated in place (M_out is M0) gives the
    single-call result; only (M, z) carries between calls."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("split", B=1, H=4, Hkv=2, d=64, N=128, S=4, dtype="bf16", rule=rule,
                    seed=12, beta_dist=("normal", 0.0, 1.0), M0_dist=("uniform", 0.0, 0.1),
                    z0_dist=("uniform", 1.0, 2.0))
    t = to_dev(wl.torch_inputs(w))
    full, Mf, zf = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                                   rule=rule)
    M, z = t["M0"].clone(), t["z0"].clone()
    L1 = 2 * w.N
    halves = []
    for sl in (slice(0, L1), slice(L1, w.L)):
        qs, ks, vs = (t[n][:, :, sl].contiguous() for n in ("q", "k", "v"))
        o, _, _ = binding.forward(qs, ks, vs, t["beta"], M, z, N=w.N, rule=rule, M_out=M,
                                  z_out=z)
        halves.append(o)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(halves, dim=2), full)
    assert torch.allclose(M, Mf, rtol=1e-6, atol=1e-6) and torch.allclose(z, zf, rtol=1e-6)


def test_device_argument_errors():
    from compressive_memory_long_b200 import binding
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 3, 128, 64, dtype=torch.bfloat16, device="cuda")
    beta = torch.zeros(2, device="cuda")
    with pytest.raises(binding.InfiniError) as e:      # H % Hkv != 0
        binding.forward(q, k, k, beta, N=64)
    assert e.value.status == 1
    q = torch.zeros(1, 2, 128, 48, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.InfiniError) as e:
        binding.forward(q, q, q, beta, N=64)
    assert e.value.status == 2


# ---- the tensor-core segment kernel (bf16, d in {64, 128}, N % 128 == 0) --------------

@pytest.mark.parametrize("rule", ["linear", "delta"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N,S", [(128, 3), (256, 2), (384, 2)])
def test_tensor_core_segment_kernel(rule, d, N, S):
    """Several 128-row q tiles (diagonal and off-diagonal key tiles), GQA, nonzero state;
    checks that the tensor-core kernel is the one that ran and that no wait gave up."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("tc", B=2, H=4, Hkv=2, d=d, N=N, S=S, dtype="bf16", rule=rule, seed=21,
                    beta_dist=("normal", 0.0, 1.5), M0_dist=("uniform", 0.0, 0.1),
                    z0_dist=("uniform", 1.0, 2.0))
    binding.infini_attn_trace_enable(True)
    check_full(w)
    binding.infini_attn_trace_enable(False)
    report = binding.infini_attn_trace_report()
    assert "segment_tc" in report and "mem_increments" in report
    assert ("mem_chain" if rule == "delta" else "mem_prefix") in report
    assert binding.infini_attn_device_status() == 0


@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_tensor_core_segment_kernel_many_items_per_cta(rule):
    """More work units than SMs (B*H*S*ceil(N/512) = 2*4*17*3 = 408), with N = 1280 (an odd
    number of 256-row pairs, so one unit per segment holds a single item) and a short 17th
    segment (300 rows: its items past row 300 are skipped): each CTA of the persistent
    kernel walks several items, heavy and light."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("tc_many", B=2, H=4, Hkv=2, d=64, N=1280, S=16, tail=300, dtype="bf16",
                    rule=rule, seed=23, beta_dist=("normal", 0.0, 1.5),
                    M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0))
    binding.infini_attn_trace_enable(True)
    check_full(w)
    binding.infini_attn_trace_enable(False)
    assert "segment_tc" in binding.infini_attn_trace_report()
    assert binding.infini_attn_device_status() == 0


def test_tensor_core_first_segment_empty_memory():
    """z0 = 0: the first segment's retrieval is exactly 0, so with beta -> +inf the first
    segment's output is exactly 0 and later segments are not."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("tc0", B=1, H=2, Hkv=2, d=128, N=256, S=2, dtype="bf16", rule="delta",
                    seed=22, beta_dist=("normal", 40.0, 0.0))
    out, _, _ = run_gpu(w)
    assert torch.count_nonzero(out[:, :, :256]) == 0
    assert torch.count_nonzero(out[:, :, 256:]) > 0
    assert binding.infini_attn_device_status() == 0


# ---- 64-token segments on the tensor cores: a pair of segments per 128-row tile ------

@pytest.mark.parametrize("rule", ["linear", "delta"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,Hkv,S", [(4, 4, 6), (8, 2, 5), (2, 1, 1)])
def test_tensor_core_64_token_segments(rule, d, H, Hkv, S):
    """N = 64 where the fused additive-rule kernels do not apply (the delta rule, d = 128, or
    a segment count that is not a whole number of 128-token units): one CTA per pair of
    segments (block-diagonal causal mask, each half retrieving from its own memory), an odd
    number of segments (a pair without its second), a single segment; the memory path and
    the segment kernel both on the tensor cores, no CUDA-core segment kernel."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("tc64", B=2, H=H, Hkv=Hkv, d=d, N=64, S=S, dtype="bf16", rule=rule, seed=31,
                    beta_dist=("normal", 0.0, 1.5), M0_dist=("uniform", 0.0, 0.1),
                    z0_dist=("uniform", 1.0, 2.0))
    fused = rule == "linear" and d == 64 and S % 2 == 0
    binding.infini_attn_trace_enable(True)
    check_full(w)
    binding.infini_attn_trace_enable(False)
    report = list(binding.infini_attn_trace_report())
    if fused:
        assert report in (["small_fused"], ["small_pieces"]), report
    else:
        assert "segment_tc" in report and "mem_increments" in report, report
        assert ("mem_chain" if rule == "delta" else "mem_prefix") in report, report
        assert not any(n in report for n in ("segment_simt", "delta_chain", "tail_segment")), report
    assert binding.infini_attn_device_status() == 0


def test_tensor_core_64_token_pair_halves_use_their_own_memory():
    """beta -> +inf (the output is the retrieval alone) and M0 = 0, z0 = 0: the first
    segment's rows are exactly 0 (empty memory), while the second segment of the same
    128-row tile retrieves from the memory after the first segment, so its rows are not."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("tc64_halves", B=1, H=2, Hkv=2, d=128, N=64, S=2, dtype="bf16",
                    rule="delta", seed=32, beta_dist=("normal", 40.0, 0.0))
    out, _, _ = run_gpu(w)
    assert torch.count_nonzero(out[:, :, :64]) == 0
    assert torch.count_nonzero(out[:, :, 64:]) > 0
    assert binding.infini_attn_device_status() == 0


# ---- the fused single-launch path (bf16, linear rule, N = 64, d = 64, MHA) -------------

@pytest.mark.parametrize("S", [2, 4, 6, 16])
def test_small_fused_shapes(S):
    """One launch with the decoupled look-back: several units per head, nonzero state."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("small", B=2, H=3, Hkv=3, d=64, N=64, S=S, dtype="bf16", rule="linear",
                    seed=23, beta_dist=("normal", 0.0, 1.5), M0_dist=("uniform", 0.0, 0.1),
                    z0_dist=("uniform", 1.0, 2.0))
    binding.infini_attn_trace_enable(True)
    check_full(w)
    binding.infini_attn_trace_enable(False)
    assert list(binding.infini_attn_trace_report()) == ["small_fused"]
    assert binding.infini_attn_device_status() == 0


def test_small_fused_in_place_split():
    from compressive_memory_long_b200 import binding
    w = wl.Workload("small_split", B=1, H=2, Hkv=2, d=64, N=64, S=8, dtype="bf16",
                    rule="linear", seed=24, beta_dist=("normal", 0.0, 1.0),
                    M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0))
    t = to_dev(wl.torch_inputs(w))
    full, Mf, zf = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], N=w.N,
                                   rule=w.rule)
    M, z = t["M0"].clone(), t["z0"].clone()
    outs = []
    for sl in (slice(0, 256), slice(256, 512)):
        qs, ks, vs = (t[n][:, :, sl].contiguous() for n in ("q", "k", "v"))
        o, _, _ = binding.forward(qs, ks, vs, t["beta"], M, z, N=w.N, rule=w.rule, M_out=M,
                                  z_out=z)
        outs.append(o)
    torch.cuda.synchronize()
    got = torch.cat(outs, dim=2).float()
    assert rel_err(got.cpu(), full.float().cpu()) <= 1e-2
    assert torch.allclose(M, Mf, rtol=1e-4, atol=1e-4) and torch.allclose(z, zf, rtol=1e-5)


# ---- the persistent piece kernel (same layouts, heads of 16 or more 128-token units) -----

@pytest.mark.parametrize("B,H,S", [(2, 3, 32), (1, 2, 66), (2, 8, 150), (1, 16, 600)])
def test_small_pieces_shapes(B, H, S):
    """Pieces of one or several units, a shorter last piece, look-back over many pieces."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("pieces", B=B, H=H, Hkv=H, d=64, N=64, S=S, dtype="bf16", rule="linear",
                    seed=31 + S, beta_dist=("normal", 0.0, 1.5), M0_dist=("uniform", 0.0, 0.1),
                    z0_dist=("uniform", 1.0, 2.0))
    binding.infini_attn_trace_enable(True)
    check_full(w)
    binding.infini_attn_trace_enable(False)
    assert list(binding.infini_attn_trace_report()) == ["small_pieces"]
    assert binding.infini_attn_device_status() == 0


def test_small_pieces_zero_state_and_split():
    """No initial state (the first segment has no memory term), then the same sequence in
    two calls with the memory carried in place."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("pieces_split", B=1, H=4, Hkv=4, d=64, N=64, S=96, dtype="bf16",
                    rule="linear", seed=41, beta_dist=("normal", 0.0, 1.0))
    check_full(w)
    t = to_dev(wl.torch_inputs(w))
    full, Mf, zf = binding.forward(t["q"], t["k"], t["v"], t["beta"], None, None, N=w.N,
                                   rule=w.rule)
    M = torch.zeros_like(Mf)
    z = torch.zeros_like(zf)
    outs = []
    for sl in (slice(0, 2048), slice(2048, 6144)):
        qs, ks, vs = (t[n][:, :, sl].contiguous() for n in ("q", "k", "v"))
        o, _, _ = binding.forward(qs, ks, vs, t["beta"], M, z, N=w.N, rule=w.rule, M_out=M,
                                  z_out=z)
        outs.append(o)
    torch.cuda.synchronize()
    got = torch.cat(outs, dim=2).float()
    assert rel_err(got.cpu(), full.float().cpu()) <= 1e-2
    assert torch.allclose(M, Mf, rtol=1e-4, atol=1e-3) and torch.allclose(z, zf, rtol=1e-5)


@pytest.mark.parametrize("B,H,Hkv,S,kernel", [(2, 4, 2, 4, "small_fused"),
                                              (1, 6, 2, 16, "small_fused"),
                                              (1, 8, 2, 66, "small_pieces"),
                                              (2, 4, 1, 40, "small_pieces")])
def test_small_fused_grouped_heads(B, H, Hkv, S, kernel):
    """Several query heads per key/value head on the fused 64-token kernels: each query head
    is a chain of its own over its group's keys, values and state; the memory is the
    group's (M_out and z_out match the oracle)."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("small_gqa", B=B, H=H, Hkv=Hkv, d=64, N=64, S=S, dtype="bf16",
                    rule="linear", seed=51 + S, beta_dist=("normal", 0.0, 1.5),
                    M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0))
    binding.infini_attn_trace_enable(True)
    check_full(w)
    binding.infini_attn_trace_enable(False)
    assert list(binding.infini_attn_trace_report()) == [kernel]
    assert binding.infini_attn_device_status() == 0


def test_small_grouped_heads_in_place_take_the_general_path():
    """Grouped heads with M_out = M0: a query head could still be reading M0 while its
    group's writer replaces it, so the call runs on the general kernels; the results match
    the oracle and the same call without aliasing."""
    from compressive_memory_long_b200 import binding
    w = wl.Workload("small_gqa_inplace", B=1, H=4, Hkv=2, d=64, N=64, S=8, dtype="bf16",
                    rule="linear", seed=57, beta_dist=("normal", 0.0, 1.0),
                    M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0))
    t = to_dev(wl.torch_inputs(w))
    ref_out, ref_M, ref_z = binding.forward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"],
                                            N=w.N, rule=w.rule)
    M, z = t["M0"].clone(), t["z0"].clone()
    binding.infini_attn_trace_enable(True)
    out, _, _ = binding.forward(t["q"], t["k"], t["v"], t["beta"], M, z, N=w.N, rule=w.rule,
                                M_out=M, z_out=z)
    torch.cuda.synchronize()
    binding.infini_attn_trace_enable(False)
    assert "small_fused" not in binding.infini_attn_trace_report()
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    ro, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=w.N, rule=w.rule)
    assert rel_err(out.float().cpu(), ro) <= TOL["bf16"]
    assert rel_err(M.cpu(), rM) <= TOL["bf16"] and rel_err(ref_M.cpu(), rM) <= TOL["bf16"]
    assert rel_err(z.cpu()[:, :, None], rz[:, :, None]) <= TOL["bf16"]
    assert binding.infini_attn_device_status() == 0


def test_n64_bandwidth_sampled():
    w = wl.WORKLOADS["n64_bandwidth"]
    check_sampled(w, chains=[(1, 5)], segs=[0, 1, 8191, 16383])
