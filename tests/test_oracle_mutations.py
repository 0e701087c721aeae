"""Planted mistakes in the oracle are caught by its pins.

Each case edits one line of a temporary copy of the oracle's C source (on the CPU; the
oracle itself is untouched), compiles it, and checks that the pins of
test_oracle_pins.py -- hand-derived cases, the independent whole-sequence formulation and
the gate limits against torch SDPA -- reject the result.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests import _independent as ind
from tests.test_oracle_pins import GOLDEN, _eval_tree, rand_inputs

MUTATIONS = {
    "softmax scale dropped": ("logit[j] = a * scale;", "logit[j] = a;"),
    "gate reversed": ("oi[e] = g * amem + (1.0 - g) * ad;", "oi[e] = (1.0 - g) * amem + g * ad;"),
    "memory transposed in the read": ("num[e] += sq[c] * M[c * d + e];",
                                      "num[e] += sq[c] * M[e * d + c];"),
    "delta residual sign": ("rt[e] = (double)vt[e] - ((den == 0.0) ? 0.0 : num[e] / den);",
                            "rt[e] = (double)vt[e] + ((den == 0.0) ? 0.0 : num[e] / den);"),
    "z update dropped": ("z[c] += sk[t * d + c];", "z[c] += 0.0 * sk[t * d + c];"),
    "ELU without +1": ("return x > 0.0 ? x + 1.0 : exp(x);", "return x > 0.0 ? x : exp(x);"),
    # the two key loops of the local softmax (row maximum and weighted sum) change together
    "causal mask off by one": ("for (int64_t j = 0; j <= i; ++j)",
                               "for (int64_t j = 0; j <= i + 1 && j < n; ++j)", -1),
    "mask not causal": ("for (int64_t j = 0; j <= i; ++j)", "for (int64_t j = 0; j < n; ++j)", -1),
}


def pins_pass(lib_path) -> bool:
    """True when every pin below agrees with the library at lib_path."""
    run = lambda *a, **k: oracle.infini_attn_fwd(*a, lib_path=lib_path, **k)
    try:
        for fname in ("hand_d1_two_segments.json", "hand_d2_orientation.json"):
            fx = json.load(open(os.path.join(GOLDEN, fname)))
            sh = fx["shape"]
            B, H, Hkv, L, N, d = (sh[x] for x in ("B", "H", "Hkv", "L", "N", "d"))
            q = np.array(fx["q"], np.float32).reshape(B, H, L, d)
            k = np.array(fx["k"], np.float32).reshape(B, Hkv, L, d)
            v = np.array(fx["v"], np.float32).reshape(B, Hkv, L, d)
            for rule in ("linear", "delta"):
                out, M, z = run(q, k, v, np.array(fx["beta"], np.float32), N=N, rule=rule)
                np.testing.assert_allclose(out, _eval_tree(fx["expected"]["out"]).reshape(out.shape),
                                           rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(M, _eval_tree(fx["expected"][rule]["M_out"]).reshape(M.shape),
                                           rtol=1e-12, atol=1e-12)
                np.testing.assert_allclose(z, _eval_tree(fx["expected"][rule]["z_out"]).reshape(z.shape),
                                           rtol=1e-12, atol=1e-12)
        for rule in ("linear", "delta"):
            q, k, v, beta, M0, z0 = rand_inputs(40, B=1, H=4, Hkv=2, L=20, d=3, state=True)
            got = run(q, k, v, beta, M0, z0, N=6, rule=rule)
            ref = ind.forward(q, k, v, beta, M0, z0, 6, rule)
            for a, b in zip(got, ref):
                np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)
        q, k, v, _, _, _ = rand_inputs(41, L=16, d=4)
        lo, _, _ = run(q, k, v, np.full(2, -40, np.float32), N=8, rule="linear")
        ref = torch.nn.functional.scaled_dot_product_attention(
            *(torch.from_numpy(x[:, :, :8].astype(np.float64)) for x in (q, k, v)), is_causal=True,
            scale=1 / math.sqrt(4)).numpy()
        np.testing.assert_allclose(lo[:, :, :8], ref, rtol=1e-12, atol=1e-14)
    except AssertionError:
        return False
    return bool(np.all(np.isfinite(lo)))


def test_unmodified_source_passes(tmp_path):
    assert pins_pass(oracle.compile_variant(oracle.source(), str(tmp_path)))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new, *count = MUTATIONS[name] + ((1,) if len(MUTATIONS[name]) == 2 else ())
    src = oracle.source()
    assert src.count(old) >= 1, f"mutation site for {name!r} not found"
    mutated = src.replace(old, new, count[0])
    assert not pins_pass(oracle.compile_variant(mutated, str(tmp_path)))
