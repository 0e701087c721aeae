"""Pins of the fp64 reference gradients (oracle/backward.py), all on CPU.

* its forward values equal the C oracle's (so the gradients are of the same function);
* central finite differences of  <dout, out> + <dM, M_out> + <dz, z_out>  along random
  directions of every input, both rules, grouped heads, a short last segment;
* the additive rule's memory gradients in closed form: M_out = M0 + sum_t sigma(k_t)^T v_t
  and z_out = z0 + sum_t sigma(k_t) ("How does the compressive memory work?") give
  dM0 = dM, dz0 = dz, dv_t = sigma(k_t) dM, dk_t = sigma'(k_t) * (dM v_t + dz) when only
  the final memory is in the loss -- a transposed M or a dropped term fails these.
"""
import numpy as np
import pytest

import oracle
from oracle import backward as bw


def _inputs(seed, B=1, H=4, Hkv=2, L=7, d=3, state=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, L, d)) * 0.8
    k = rng.standard_normal((B, Hkv, L, d)) * 0.8
    v = rng.standard_normal((B, Hkv, L, d))
    beta = rng.standard_normal(H)
    M0 = rng.uniform(0.0, 0.2, (B, Hkv, d, d)) if state else None
    z0 = rng.uniform(1.0, 2.0, (B, Hkv, d)) if state else None
    return q, k, v, beta, M0, z0


def _loss(x, dout, dM, dz, N, rule):
    out, M, z = bw.forward_values(*x, N=N, rule=rule)
    return float((out * dout).sum() + (M * dM).sum() + (z * dz).sum())


@pytest.mark.parametrize("rule", ["linear", "delta"])
@pytest.mark.parametrize("state", [True, False])
def test_forward_values_equal_the_c_oracle(rule, state):
    x = _inputs(3, state=state)
    q, k, v, beta, M0, z0 = x
    f32 = [None if a is None else a.astype(np.float32).astype(np.float64) for a in x]
    got = bw.forward_values(*f32, N=3, rule=rule)
    ref = oracle.infini_attn_fwd(*[None if a is None else a.astype(np.float32) for a in x],
                                 N=3, rule=rule)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("rule", ["linear", "delta"])
@pytest.mark.parametrize("seed", [1, 2])
def test_gradients_match_central_differences(rule, seed):
    x = list(_inputs(seed))
    N = 3                                     # L = 7: two segments of 3 and one of 1
    rng = np.random.default_rng(100 + seed)
    out, M, z = bw.forward_values(*x, N=N, rule=rule)
    dout, dM, dz = (rng.standard_normal(a.shape) for a in (out, M, z))
    grads = bw.gradients(*x, dout, dM, dz, N=N, rule=rule)
    names = ["q", "k", "v", "beta", "M0", "z0"]
    eps = 1e-6
    for i, name in enumerate(names):
        u = rng.standard_normal(np.shape(x[i]))
        xp = list(x)
        xm = list(x)
        xp[i] = x[i] + eps * u
        xm[i] = x[i] - eps * u
        fd = (_loss(xp, dout, dM, dz, N, rule) - _loss(xm, dout, dM, dz, N, rule)) / (2 * eps)
        an = float((grads[name] * u).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), f"{rule} d/d{name}: {fd} vs {an}"


def test_linear_memory_gradients_in_closed_form():
    q, k, v, beta, M0, z0 = _inputs(5, B=2, H=2, Hkv=2, L=9, d=4)
    rng = np.random.default_rng(9)
    dM = rng.standard_normal(M0.shape)
    dz = rng.standard_normal(z0.shape)
    dout = np.zeros(q.shape)
    g = bw.gradients(q, k, v, beta, M0, z0, dout, dM, dz, N=4, rule="linear")
    sk = np.where(k > 0, k + 1.0, np.exp(np.minimum(k, 0.0)))
    dsk = np.where(k > 0, 1.0, np.exp(np.minimum(k, 0.0)))
    # dv_t = sigma(k_t) dM ; dk_t = sigma'(k_t) * (dM v_t + dz)
    dv = np.einsum("bhtf,bhfc->bhtc", sk, dM)
    dk = dsk * (np.einsum("bhfc,bhtc->bhtf", dM, v) + dz[:, :, None, :])
    np.testing.assert_allclose(g["v"], dv, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["k"], dk, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["M0"], dM, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["z0"], dz, rtol=1e-12, atol=1e-12)
    assert not g["q"].any() and not g["beta"].any()
