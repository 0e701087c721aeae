"""Pins of the fp64 CPU oracle: checks against facts the pages and mathematics fix.

Each test states the passage or fact it rests on.  None re-types the oracle's loops;
each would fail on a plausible mistake (a dropped term, a wrong sign, a transposed M,
an off-by-one causal mask, a gate pointing the wrong way, a delta update applied token
by token instead of once per segment).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from compressive_memory_long_b200 import workloads as wl
from tests import _independent as ind

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_inputs(seed, B=1, H=2, Hkv=2, L=24, d=4, state=False, scale=0.7):
    r = np.random.default_rng(seed)
    q = (r.standard_normal((B, H, L, d)) * scale).astype(np.float32)
    k = (r.standard_normal((B, Hkv, L, d)) * scale).astype(np.float32)
    v = r.standard_normal((B, Hkv, L, d)).astype(np.float32)
    beta = r.standard_normal(H).astype(np.float32)
    M0 = z0 = None
    if state:
        M0 = r.uniform(-0.2, 0.5, (B, Hkv, d, d)).astype(np.float32)
        z0 = r.uniform(0.5, 2.0, (B, Hkv, d)).astype(np.float32)
    return q, k, v, beta, M0, z0


def _eval(expr):
    return eval(expr, {"__builtins__": {}}, {"e": math.e})


def _eval_tree(x):
    if isinstance(x, list):
        return np.array([_eval_tree(y) for y in x], dtype=np.float64)
    return np.float64(_eval(x))


# ---- hand-derived cases (tests/golden) ---------------------------------------------

@pytest.mark.parametrize("fname", ["hand_d1_two_segments.json", "hand_d2_orientation.json"])
@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_hand_cases(fname, rule):
    """Hand derivations from the block and memory equations (see each fixture)."""
    fx = json.load(open(os.path.join(GOLDEN, fname)))
    sh = fx["shape"]
    B, H, Hkv, L, N, d = (sh[x] for x in ("B", "H", "Hkv", "L", "N", "d"))
    q = np.array(fx["q"], np.float32).reshape(B, H, L, d)
    k = np.array(fx["k"], np.float32).reshape(B, Hkv, L, d)
    v = np.array(fx["v"], np.float32).reshape(B, Hkv, L, d)
    beta = np.array(fx["beta"], np.float32)
    out, M, z = oracle.infini_attn_fwd(q, k, v, beta, N=N, rule=rule)
    exp_out = _eval_tree(fx["expected"]["out"]).reshape(out.shape)
    exp_M = _eval_tree(fx["expected"][rule]["M_out"]).reshape(M.shape)
    exp_z = _eval_tree(fx["expected"][rule]["z_out"]).reshape(z.shape)
    np.testing.assert_allclose(out, exp_out, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(M, exp_M, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(z, exp_z, rtol=1e-14, atol=1e-14)


# ---- P1: the gate's two limits ("How does the gating mechanism choose ...") --------

@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_gate_limits(rule):
    """beta -> -inf leaves pure local attention; beta -> +inf pure memory retrieval.

    The local limit is checked against an independent causal-softmax (torch SDPA in
    float64) per segment; the memory limit against the empty-memory rule: segment 0 of a
    fresh memory returns exactly 0.  Together they fix the gate's direction.
    """
    q, k, v, _, _, _ = rand_inputs(1, L=24, d=4)
    N = 8
    lo, _, _ = oracle.infini_attn_fwd(q, k, v, np.full(2, -40, np.float32), N=N, rule=rule)
    hi, _, _ = oracle.infini_attn_fwd(q, k, v, np.full(2, 40, np.float32), N=N, rule=rule)
    for s in range(3):
        sl = slice(s * N, (s + 1) * N)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[:, :, sl].astype(np.float64)),
            torch.from_numpy(k[:, :, sl].astype(np.float64)),
            torch.from_numpy(v[:, :, sl].astype(np.float64)), is_causal=True,
            scale=1 / math.sqrt(4)).numpy()
        np.testing.assert_allclose(lo[:, :, sl], ref, rtol=1e-12, atol=1e-14)
    assert np.all(hi[:, :, :N] == 0.0)
    assert np.abs(hi[:, :, N:]).max() > 0.1
    # any beta: the stated convex combination of the two limits
    beta = np.array([0.3, -1.2], np.float32)
    mid, _, _ = oracle.infini_attn_fwd(q, k, v, beta, N=N, rule=rule)
    g = 1 / (1 + np.exp(-beta.astype(np.float64)))
    np.testing.assert_allclose(mid, g[None, :, None, None] * hi
                               + (1 - g)[None, :, None, None] * lo, rtol=1e-12, atol=1e-14)


# ---- P2: one segment on an empty memory is causal softmax attention -----------------

def test_one_segment_is_causal_attention():
    """With L = N and M0 = z0 = 0, out / (1 - g) equals textbook causal attention."""
    q, k, v, beta, _, _ = rand_inputs(2, B=2, H=3, Hkv=3, L=16, d=8)
    out, _, _ = oracle.infini_attn_fwd(q, k, v, beta, N=16, rule="delta")
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x.astype(np.float64)) for x in (q, k, v)), is_causal=True,
        scale=1 / math.sqrt(8)).numpy()
    g = 1 / (1 + np.exp(-beta.astype(np.float64)))
    np.testing.assert_allclose(out / (1 - g)[None, :, None, None], ref, rtol=1e-12, atol=1e-14)


# ---- P3: the additive memory is the running sum sigma(K)^T V ------------------------

@pytest.mark.parametrize("N", [1, 5, 8, 24])
def test_linear_state_closed_form(N):
    """Linear rule: M_out = M0 + sigma(K)^T V and z_out = z0 + sum sigma(K) over all tokens,
    whatever the segmentation ("What is linear attention and the delta rule?")."""
    q, k, v, beta, M0, z0 = rand_inputs(3, L=24, d=4, state=True)
    _, M, z = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=N, rule="linear")
    sK = ind.sigma(k)
    np.testing.assert_allclose(M, M0 + np.einsum("bhtc,bhte->bhce", sK, v.astype(np.float64)),
                               rtol=1e-12)
    np.testing.assert_allclose(z, z0 + sK.sum(axis=2), rtol=1e-12)


# ---- P4 / P11: an independent whole-sequence formulation ---------------------------

@pytest.mark.parametrize("rule", ["linear", "delta"])
@pytest.mark.parametrize("L,N", [(24, 8), (23, 8), (7, 3), (5, 5), (6, 1)])
@pytest.mark.parametrize("state", [False, True])
def test_matches_independent_formulation(rule, L, N, state):
    """Brute force on tiny inputs (ragged tails included): block-causal masked matrices
    for the additive rule, a matrix-form segment loop for the delta rule."""
    q, k, v, beta, M0, z0 = rand_inputs(4 + L + N, B=2, H=4, Hkv=2, L=L, d=3, state=state)
    got = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=N, rule=rule)
    ref = ind.forward(q, k, v, beta, M0, z0, N, rule)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


# ---- P5: the delta rule leaves an already-stored binding alone ---------------------

def test_delta_zero_residual():
    """A binding the memory already holds yields a zero residual, so the delta rule leaves
    M as it was ("How does the compressive memory work?").  With the rank-1
    memory M = z w^T, sigma(k) M / (sigma(k) z) = w for every key, so writing V = w
    leaves M unchanged while z still advances by sum sigma(K).  (One update only: after it
    z has grown, so M is no longer z w^T for the new z.)"""
    r = np.random.default_rng(5)
    d, L = 6, 12
    # z0 entries are powers of two, so M0 = z0 w^T is exactly rank-1 in float32
    z0 = (2.0 ** r.integers(-1, 2, (1, 1, d))).astype(np.float32)
    w = r.standard_normal(d).astype(np.float32)
    M0 = (z0[0, 0, :, None] * w[None, :]).astype(np.float32)[None, None]
    k = r.standard_normal((1, 1, L, d)).astype(np.float32)
    v = np.broadcast_to(w, (1, 1, L, d)).astype(np.float32)
    q = r.standard_normal((1, 1, L, d)).astype(np.float32)
    _, M, z = oracle.infini_attn_fwd(q, k, v, np.zeros(1, np.float32), M0, z0, N=L,
                                     rule="delta")
    np.testing.assert_allclose(M, M0, rtol=0, atol=1e-13 * np.abs(M0).max())
    np.testing.assert_allclose(z, z0 + ind.sigma(k).sum(axis=2), rtol=1e-13)
    # the additive rule on the same inputs does move M
    _, M_lin, _ = oracle.infini_attn_fwd(q, k, v, np.zeros(1, np.float32), M0, z0, N=L,
                                         rule="linear")
    assert np.abs(M_lin - M0).max() > 1.0


# ---- P6: from an empty memory the two rules agree on the first step ---------------

def test_rules_agree_on_first_segment():
    """While z = 0 the delta prediction is 0, so after segment 0 both rules hold the same
    M; outputs of segments 0 and 1 therefore agree; z never depends on the rule."""
    q, k, v, beta, _, _ = rand_inputs(6, L=24, d=4)
    N = 8
    a = oracle.infini_attn_fwd(q[:, :, :8], k[:, :, :8], v[:, :, :8], beta, N=N, rule="linear")
    b = oracle.infini_attn_fwd(q[:, :, :8], k[:, :, :8], v[:, :, :8], beta, N=N, rule="delta")
    np.testing.assert_array_equal(a[1], b[1])
    lo, Ml, zl = oracle.infini_attn_fwd(q, k, v, beta, N=N, rule="linear")
    de, Md, zd = oracle.infini_attn_fwd(q, k, v, beta, N=N, rule="delta")
    np.testing.assert_array_equal(lo[:, :, :16], de[:, :, :16])
    assert np.abs(lo[:, :, 16:] - de[:, :, 16:]).max() > 1e-6
    np.testing.assert_allclose(zl, zd, rtol=1e-15)
    assert np.abs(Ml - Md).max() > 1e-6


# ---- P7: the first token of a segment sees only itself locally ---------------------

def test_first_token_of_segment():
    """Softmax over a single key is that key's value: out_{sN} = (1-g) v_{sN} + g A_mem."""
    q, k, v, beta, M0, z0 = rand_inputs(7, L=24, d=4, state=True)
    N = 8
    out, _, _ = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=N, rule="linear")
    mem, _, _ = oracle.infini_attn_fwd(q, k, v, np.full(2, 40, np.float32), M0, z0, N=N,
                                       rule="linear")
    g = 1 / (1 + np.exp(-beta.astype(np.float64)))
    for s in range(3):
        t = s * N
        for h in range(2):
            np.testing.assert_allclose(out[0, h, t], (1 - g[h]) * v[0, h, t]
                                       + g[h] * mem[0, h, t], rtol=1e-12, atol=1e-14)


# ---- P9: GQA equals MHA with repeated key/value heads ------------------------------

@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_gqa_equals_repeated_mha(rule):
    q, k, v, beta, M0, z0 = rand_inputs(8, B=2, H=6, Hkv=2, L=12, d=3, state=True)
    a, Ma, za = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=4, rule=rule)
    rep = lambda x: np.repeat(x, 3, axis=1)
    b, Mb, zb = oracle.infini_attn_fwd(q, rep(k), rep(v), beta, rep(M0), rep(z0), N=4, rule=rule)
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(Mb[:, ::3], Ma, rtol=1e-14)
    np.testing.assert_allclose(zb[:, ::3], za, rtol=1e-14)


# ---- P10: the carried state is a resume point ------------------------------------

@pytest.mark.parametrize("rule", ["linear", "delta"])
def test_streaming_split(rule):
    """Only (M, z) passes between segments (reproduction analysis, step 6), so running
    [0, L1) and then [L1, L) from the carried state equals one run over [0, L)."""
    q, k, v, beta, M0, z0 = rand_inputs(9, L=32, d=4, state=True)
    N, L1 = 8, 16
    full, Mf, zf = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=N, rule=rule)
    a, M1, z1 = oracle.infini_attn_fwd(q[:, :, :L1], k[:, :, :L1], v[:, :, :L1], beta, M0, z0,
                                       N=N, rule=rule)
    b, M2, z2 = oracle.infini_attn_fwd(q[:, :, L1:], k[:, :, L1:], v[:, :, L1:], beta,
                                       M1.astype(np.float32), z1.astype(np.float32), N=N,
                                       rule=rule)
    # the resumed half starts from a float32-rounded state, hence the looser bound
    np.testing.assert_allclose(a, full[:, :, :L1], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(b, full[:, :, L1:], rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(M2, Mf, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(z2, zf, rtol=1e-6)


# ---- the segment-output mask changes nothing it does not skip --------------------

def test_segment_output_mask():
    q, k, v, beta, M0, z0 = rand_inputs(10, L=32, d=4, state=True)
    full, Mf, zf = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=8, rule="delta")
    part, Mp, zp = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=8, rule="delta",
                                          seg_out=[1, 3])
    np.testing.assert_array_equal(part[:, :, 8:16], full[:, :, 8:16])
    np.testing.assert_array_equal(part[:, :, 24:], full[:, :, 24:])
    assert np.all(part[:, :, :8] == 0) and np.all(part[:, :, 16:24] == 0)
    np.testing.assert_array_equal(Mp, Mf)
    np.testing.assert_array_equal(zp, zf)


# ---- sigma itself: both branches ------------------------------------------------

def test_feature_map_branches():
    """sigma = ELU + 1 ("What happens inside the Infini-attention block?"): with one key of
    value x and d = 1, the additive rule stores z_out = sigma(x)."""
    xs = np.array([-3.0, -0.5, 0.0, 1e-3, 0.75, 2.5], np.float32)
    for x in xs:
        k = np.full((1, 1, 1, 1), x, np.float32)
        _, _, z = oracle.infini_attn_fwd(k, k, k, np.zeros(1, np.float32), N=1, rule="linear")
        expect = float(x) + 1.0 if x > 0 else math.exp(float(x))
        assert z[0, 0, 0] == pytest.approx(expect, rel=1e-15)


def test_workload_slices_are_reproducible():
    """The input generator gives the same slice alone and inside a full draw."""
    w = wl.WORKLOADS["fp32_linear_small"]
    q, k, v, beta, M0, z0 = wl.host_inputs(w)
    np.testing.assert_array_equal(q[0, 1], wl.qkv_slice(w, "q", 0, 1))
    t = wl.torch_inputs(w)
    np.testing.assert_array_equal(t["k"].numpy(), k)
    w2 = wl.WORKLOADS["hf_repro_n64"]
    x = wl.qkv_slice(w2, "v", 1, 3)
    assert np.array_equal(x, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_workload_prefix_draw():
    """A bounded sample (the first rows of a slice) equals the full draw's prefix."""
    w = wl.WORKLOADS["hf_repro_n64"].replace(k_boost_frac=0.05, k_boost=4.0)
    for t in ("q", "k", "v"):
        full = wl.qkv_slice(w, t, 1, 2)
        np.testing.assert_array_equal(wl.qkv_slice(w, t, 1, 2, rows=192), full[:192])
