"""The backward pass (infini_attn_bwd / _f32) against the fp64 reference gradients.

oracle/backward.py differentiates the restated forward (pinned to the C oracle and to
finite differences on CPU); here every gradient of  <dout, out> + <dM, M_out> + <dz, z_out>
must match it per (batch, head) slice: max |x - r| / max |r| <= 1e-4 for fp32 activations
and 2e-2 for bf16 ones (inputs and dq / dk / dv in bf16, arithmetic in fp32).
"""
import numpy as np
import pytest
import torch

from compressive_memory_long_b200 import binding
from compressive_memory_long_b200 import workloads as wl
from oracle import backward as bw

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref):
    g = np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    if g.ndim == 1:
        g, r = g[None], r[None]
    g = g.reshape(g.shape[0] * (g.shape[1] if g.ndim > 2 else 1), -1)
    r = r.reshape(g.shape)
    return float((np.abs(g - r).max(axis=1) / np.maximum(np.abs(r).max(axis=1), 1e-30)).max())


def make(name, *, B, H, Hkv, d, N, S, tail=0, dtype="f32", rule="linear", state=True, seed=0):
    kw = dict(M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0)) if state else {}
    return wl.Workload(name, B=B, H=H, Hkv=Hkv, d=d, N=N, S=S, tail=tail, dtype=dtype,
                       rule=rule, seed=seed, beta_dist=("normal", 0.0, 1.0), **kw)


CASES = [
    make("f32_lin_d32", B=1, H=2, Hkv=2, d=32, N=64, S=3, seed=91),
    make("f32_delta_d32", B=1, H=2, Hkv=2, d=32, N=64, S=3, rule="delta", seed=92),
    make("f32_delta_gqa_tail", B=2, H=4, Hkv=2, d=64, N=64, S=2, tail=37, rule="delta", seed=93),
    make("f32_lin_gqa_nostate", B=1, H=4, Hkv=2, d=64, N=128, S=2, tail=5, state=False, seed=94),
    make("f32_delta_nostate", B=1, H=2, Hkv=1, d=32, N=64, S=3, rule="delta", state=False, seed=95),
    make("bf16_delta_d128", B=1, H=4, Hkv=2, d=128, N=128, S=2, tail=64, dtype="bf16",
         rule="delta", seed=96),
    make("bf16_lin_d64", B=2, H=2, Hkv=2, d=64, N=64, S=4, dtype="bf16", seed=97),
    # tensor-core local attention (N % 128 == 0): several key / query tiles, grouped heads,
    # a short last segment
    make("bf16_delta_gqa_n256_tail", B=1, H=4, Hkv=2, d=64, N=256, S=2, tail=100, dtype="bf16",
         rule="delta", seed=98),
    make("bf16_lin_n384_d128", B=2, H=2, Hkv=1, d=128, N=384, S=2, dtype="bf16", seed=99),
    make("bf16_delta_g4_d128_tail", B=1, H=8, Hkv=2, d=128, N=256, S=3, tail=129, dtype="bf16",
         rule="delta", seed=100),
    # 64-token segments on the tensor cores (a pair of segments per 128-row tile, each half
    # retrieving from its own memory): grouped heads with a short last segment that leaves the
    # last pair without its second (3 segments), and an odd count of full segments
    make("bf16_delta_n64_gqa_tail", B=1, H=4, Hkv=2, d=128, N=64, S=2, tail=20, dtype="bf16",
         rule="delta", seed=101),
    make("bf16_lin_n64_d128_odd", B=2, H=2, Hkv=1, d=128, N=64, S=5, dtype="bf16", seed=102),
    make("bf16_delta_n64_d64_gqa_odd", B=2, H=4, Hkv=2, d=64, N=64, S=3, dtype="bf16", rule="delta",
         seed=103),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_gradients_match_the_reference(w):
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    st = wl.has_initial_state(w)
    rng = np.random.default_rng(w.seed + 1000)
    dout = rng.standard_normal(q.shape).astype(np.float32)
    dM = (0.1 * rng.standard_normal((w.B, w.Hkv, w.d, w.d))).astype(np.float32)
    dz = (0.01 * rng.standard_normal((w.B, w.Hkv, w.d))).astype(np.float32)
    dt = w.torch_dtype
    dout_t = torch.from_numpy(dout).to(dt)
    dout = dout_t.float().numpy()            # the values the device sees
    dev = {n: torch.from_numpy(x).to(dt).cuda() for n, x in (("q", q), ("k", k), ("v", v))}
    got = binding.backward(dev["q"], dev["k"], dev["v"], torch.from_numpy(beta).cuda(),
                           torch.from_numpy(M0).cuda() if st else None,
                           torch.from_numpy(z0).cuda() if st else None, dout_t.cuda(),
                           torch.from_numpy(dM).cuda(), torch.from_numpy(dz).cuda(), N=w.N,
                           rule=w.rule)
    torch.cuda.synchronize()
    ref = bw.gradients(q, k, v, beta, M0 if st else None, z0 if st else None, dout, dM, dz,
                       N=w.N, rule=w.rule)
    names = ("q", "k", "v", "beta", "M0", "z0")
    errs = {}
    for n, g in zip(names, got):
        gg = g.float().cpu().numpy()
        r = ref[n]
        errs[n] = rel_err(gg[None] if n == "beta" else gg, r[None] if n == "beta" else r)
    print("BWD " + w.name + " " + " ".join(f"d{n}={e:.3e}" for n, e in errs.items()), flush=True)
    tol = TOL[w.dtype]
    assert max(errs.values()) <= tol, errs
    assert binding.infini_attn_device_status() == 0


def test_gradients_without_memory_terms_and_optional_outputs():
    """dM = dz = NULL are zero gradients of the final memory; dbeta / dM0 / dz0 may be NULL."""
    import ctypes
    w = CASES[0]
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    rng = np.random.default_rng(7)
    dout = rng.standard_normal(q.shape).astype(np.float32)
    t = {n: torch.from_numpy(x).cuda() for n, x in
         (("q", q), ("k", k), ("v", v), ("beta", beta), ("M0", M0), ("z0", z0), ("dout", dout))}
    full = binding.backward(t["q"], t["k"], t["v"], t["beta"], t["M0"], t["z0"], t["dout"],
                            N=w.N, rule=w.rule)
    dq, dk, dv = (torch.empty_like(t[n]) for n in ("q", "k", "v"))
    P = ctypes.c_void_p
    rc = binding.LIB.infini_attn_bwd_f32(*(P(t[n].data_ptr()) for n in ("q", "k", "v", "beta", "M0", "z0", "dout")),
                                         None, None, P(dq.data_ptr()), P(dk.data_ptr()),
                                         P(dv.data_ptr()), None, None, None, w.B, w.H, w.Hkv,
                                         w.L, w.N, w.d, 0, None)
    torch.cuda.synchronize()
    assert rc == 0
    assert torch.equal(dq, full[0]) and torch.equal(dk, full[1]) and torch.equal(dv, full[2])
    ref = bw.gradients(q, k, v, beta, M0, z0, dout, np.zeros((1, w.Hkv, w.d, w.d)),
                       np.zeros((1, w.Hkv, w.d)), N=w.N, rule=w.rule)
    assert rel_err(full[4].cpu().numpy(), ref["M0"]) <= 1e-4
