"""The decode reading, pinned on the CPU: feeding a sequence one token at a time -- each
token attends to the cached keys of its own segment up to itself, reads the memory from
before its segment, and a complete segment (or, at the end, the cached rest) is folded into
the memory -- gives the forward's outputs and final memory exactly (up to rounding order).

The token-by-token procedure is written here in plain numpy fp64, independently of both
the oracle and the CUDA decode kernel, and compared with the oracle's forward; so the
oracle is a valid reference for the GPU decode step.  Sources: AI Wiki "Infini-Attention",
"What happens inside the Infini-attention block?" and "How does the compressive memory
work?"; the Hugging Face reproduction analysis, "Infini-Attention Mechanism", steps 1-6.
"""
import numpy as np
import pytest

import oracle


def _sigma(x):
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def _fold(M, z, kc, vc, rule):
    """Fold cached rows (all reading the memory from before them) into (M, z)."""
    sk = _sigma(kc)                                    # [n, d]
    if rule == "linear":
        upd = vc
    else:
        den = sk @ z                                   # [n]
        pred = np.where(den[:, None] == 0, 0.0, (sk @ M) / np.where(den == 0, 1.0, den)[:, None])
        upd = vc - pred
    return M + sk.T @ upd, z + sk.sum(axis=0)


def decode_sequence(q, k, v, beta, M0, z0, N, rule):
    """q [H, L, d], k/v [Hkv, L, d] of one batch row; returns (out [H, L, d], M, z)."""
    H, L, d = q.shape
    Hkv = k.shape[0]
    G = H // Hkv
    out = np.zeros((H, L, d))
    M = [M0[h].copy() for h in range(Hkv)]
    z = [z0[h].copy() for h in range(Hkv)]
    for kvh in range(Hkv):
        cache_k, cache_v = [], []
        for t in range(L):
            cache_k.append(k[kvh, t])
            cache_v.append(v[kvh, t])
            K = np.stack(cache_k)
            V = np.stack(cache_v)
            for g in range(G):
                h = kvh * G + g
                s = K @ q[h, t] / np.sqrt(d)
                p = np.exp(s - s.max())
                a_dot = p @ V / p.sum()
                sq = _sigma(q[h, t])
                den = sq @ z[kvh]
                a_mem = np.zeros(d) if den == 0 else (sq @ M[kvh]) / den
                gate = 1.0 / (1.0 + np.exp(-beta[h]))
                out[h, t] = gate * a_mem + (1.0 - gate) * a_dot
            if len(cache_k) == N:                      # the segment is complete
                M[kvh], z[kvh] = _fold(M[kvh], z[kvh], K, V, rule)
                cache_k, cache_v = [], []
        if cache_k:                                    # the end of a shorter last segment
            M[kvh], z[kvh] = _fold(M[kvh], z[kvh], np.stack(cache_k), np.stack(cache_v), rule)
    return out, np.stack(M), np.stack(z)


@pytest.mark.parametrize("rule", ["linear", "delta"])
@pytest.mark.parametrize("H,Hkv,L,N,state", [(2, 2, 12, 4, False), (4, 2, 11, 4, True),
                                             (3, 1, 7, 8, True), (2, 1, 9, 3, False)])
def test_token_by_token_equals_forward(rule, H, Hkv, L, N, state):
    rng = np.random.default_rng(7 + L + N + H)
    d = 5
    q = (rng.standard_normal((1, H, L, d)) * 0.7).astype(np.float32)
    k = (rng.standard_normal((1, Hkv, L, d)) * 0.7).astype(np.float32)
    v = rng.standard_normal((1, Hkv, L, d)).astype(np.float32)
    beta = rng.standard_normal(H).astype(np.float32)
    M0 = rng.uniform(0.0, 0.2, (1, Hkv, d, d)).astype(np.float32) if state else None
    z0 = rng.uniform(1.0, 2.0, (1, Hkv, d)).astype(np.float32) if state else None
    ro, rM, rz = oracle.infini_attn_fwd(q, k, v, beta, M0, z0, N=N, rule=rule)
    m0 = M0[0].astype(np.float64) if state else np.zeros((Hkv, d, d))
    zz = z0[0].astype(np.float64) if state else np.zeros((Hkv, d))
    out, M, z = decode_sequence(q[0].astype(np.float64), k[0].astype(np.float64),
                                v[0].astype(np.float64), beta.astype(np.float64), m0, zz, N,
                                rule)
    np.testing.assert_allclose(out, ro[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(M, rM[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z, rz[0], rtol=1e-12, atol=1e-12)
