"""A second, independent fp64 statement of the Infini-attention forward, for pinning the oracle.

Written separately from the oracle and in a different form: whole-sequence masked
matrices instead of per-token loops.

* Local attention is one L x L softmax whose mask keeps key j for query i only when both
  sit in the same segment and j <= i (AI Wiki "Infini-Attention", "What happens inside
  the Infini-attention block?": causal softmax within the segment; the Hugging Face
  reproduction analysis, "Infini-Attention Mechanism", step 6: earlier segments' keys
  are discarded).
* For the additive rule the memory read of a query in segment s is the block-causal
  linear attention over every key of segments < s plus the initial state (the running
  sum of sigma(K)^T V of "What is linear attention and the delta rule?").
* For the delta rule (no closed form) the states are produced by a matrix-form segment
  loop, then read by the same masked formulation.

sigma is ``torch.nn.functional.elu(x) + 1`` (the library's ELU, alpha = 1).
"""
from __future__ import annotations

import numpy as np
import torch


def sigma(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.asarray(x, dtype=np.float64))
    return (torch.nn.functional.elu(t, alpha=1.0) + 1.0).numpy()


def _safe_div(num: np.ndarray, den: np.ndarray) -> np.ndarray:
    den_b = den[..., None]
    return np.where(den_b == 0.0, 0.0, num / np.where(den_b == 0.0, 1.0, den_b))


def forward(q, k, v, beta, M0, z0, N, rule):
    q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
    beta = np.asarray(beta, np.float64)
    B, H, L, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    if M0 is None:
        M0 = np.zeros((B, Hkv, d, d))
    if z0 is None:
        z0 = np.zeros((B, Hkv, d))
    M0 = np.asarray(M0, np.float64)
    z0 = np.asarray(z0, np.float64)
    seg = np.arange(L) // N
    S = int(seg[-1]) + 1
    same = seg[:, None] == seg[None, :]
    causal = np.arange(L)[None, :] <= np.arange(L)[:, None]
    local_mask = same & causal
    earlier = seg[None, :] < seg[:, None]          # key u lies in an earlier segment than t

    out = np.zeros((B, H, L, d))
    M_out = np.zeros((B, Hkv, d, d))
    z_out = np.zeros((B, Hkv, d))
    for b in range(B):
        for kvh in range(Hkv):
            K, V = k[b, kvh], v[b, kvh]
            sK = sigma(K)
            # states before each segment
            Ms = np.zeros((S, d, d))
            zs = np.zeros((S, d))
            M, z = M0[b, kvh].copy(), z0[b, kvh].copy()
            for s in range(S):
                Ms[s], zs[s] = M, z
                rows = seg == s
                Ks, Vs = sK[rows], V[rows]
                if rule == "linear":
                    W = Vs
                else:
                    W = Vs - _safe_div(Ks @ M, Ks @ z)
                M = M + Ks.T @ W
                z = z + Ks.sum(axis=0)
            M_out[b, kvh], z_out[b, kvh] = M, z

            for g in range(G):
                h = kvh * G + g
                Q = q[b, h]
                logits = (Q @ K.T) / np.sqrt(d)
                logits = np.where(local_mask, logits, -np.inf)
                logits -= logits.max(axis=1, keepdims=True)
                P = np.exp(logits)
                A_dot = (P / P.sum(axis=1, keepdims=True)) @ V
                sQ = sigma(Q)
                if rule == "linear":
                    Wt = (sQ @ sK.T) * earlier
                    num = Wt @ V + sQ @ M0[b, kvh]
                    den = Wt.sum(axis=1) + sQ @ z0[b, kvh]
                else:
                    num = np.einsum("tc,tce->te", sQ, Ms[seg])
                    den = np.einsum("tc,tc->t", sQ, zs[seg])
                A_mem = _safe_div(num, den)
                gate = 1.0 / (1.0 + np.exp(-beta[h]))
                out[b, h] = gate * A_mem + (1.0 - gate) * A_dot
    return out, M_out, z_out
