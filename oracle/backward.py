"""fp64 reference gradients of the Infini-attention forward (for a future backward pass).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: nothing in the CUDA library imports
it.  No GPU backward exists yet; this module is the reference such a kernel will be checked
against, committed and pinned first.

The forward is restated here in plain PyTorch fp64 tensor operations, segment by segment
in the order of AI Wiki "Infini-Attention", "What happens inside the Infini-attention
block?" (causal softmax within the segment, the sigma = ELU + 1 retrieval from the memory
before the segment, the sigmoid gate) and "How does the compressive memory work?" (the
additive and delta updates, the z update), with the same readings as the C oracle (a
quotient whose denominator is exactly 0 is 0; a last segment shorter than N is processed
the same way).  Its gradients are those of that definition, taken by automatic
differentiation (a library primitive standing for the chain rule).  Pins:
``tests/test_backward_oracle_pins.py`` (central finite differences, the additive rule's
closed-form memory gradients, and equality of the forward values with the C oracle).

Gradients are of  loss = <dout, out> + <dM, M_out> + <dz, z_out>  with respect to q, k,
v, beta, M0 and z0.
"""
from __future__ import annotations

import numpy as np
import torch


def _sigma(x):
    return torch.nn.functional.elu(x, alpha=1.0) + 1.0


def _quotient(num, den):
    """num / den with 0 where den == 0 (the gradient there is 0 as well)."""
    zero = den == 0
    safe = torch.where(zero, torch.ones_like(den), den)
    return torch.where(zero[..., None], torch.zeros_like(num), num / safe[..., None])


def forward(q, k, v, beta, M0, z0, N: int, rule: str):
    """q [B,H,L,d], k/v [B,Hkv,L,d], beta [H], M0 [B,Hkv,d,d], z0 [B,Hkv,d] (fp64 tensors).
    Returns (out [B,H,L,d], M_out [B,Hkv,d,d], z_out [B,Hkv,d])."""
    B, H, L, d = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    gate = torch.sigmoid(beta)
    outs = []
    Ms, zs = [], []
    for b in range(B):
        out_b = [None] * H
        M_b, z_b = [], []
        for kvh in range(Hkv):
            M, z = M0[b, kvh], z0[b, kvh]
            pieces = [[] for _ in range(G)]
            for s0 in range(0, L, N):
                s1 = min(s0 + N, L)
                K, V = k[b, kvh, s0:s1], v[b, kvh, s0:s1]
                n = s1 - s0
                mask = torch.ones(n, n, dtype=torch.bool).tril()
                for g in range(G):
                    h = kvh * G + g
                    Q = q[b, h, s0:s1]
                    scores = (Q @ K.T) / (d ** 0.5)
                    scores = scores.masked_fill(~mask, float("-inf"))
                    a_dot = torch.softmax(scores, dim=-1) @ V
                    sq = _sigma(Q)
                    a_mem = _quotient(sq @ M, sq @ z)
                    pieces[g].append(gate[h] * a_mem + (1.0 - gate[h]) * a_dot)
                sk = _sigma(K)
                if rule == "linear":
                    upd = V
                else:
                    upd = V - _quotient(sk @ M, sk @ z)
                M = M + sk.T @ upd
                z = z + sk.sum(dim=0)
            for g in range(G):
                out_b[kvh * G + g] = torch.cat(pieces[g], dim=0)
            M_b.append(M)
            z_b.append(z)
        outs.append(torch.stack(out_b))
        Ms.append(torch.stack(M_b))
        zs.append(torch.stack(z_b))
    return torch.stack(outs), torch.stack(Ms), torch.stack(zs)


def _t(x):
    return torch.tensor(np.asarray(x, dtype=np.float64), dtype=torch.float64)


def gradients(q, k, v, beta, M0, z0, dout, dM, dz, *, N: int, rule: str = "linear"):
    """Gradients of <dout, out> + <dM, M_out> + <dz, z_out>.  Inputs are numpy arrays (any
    float dtype; used in fp64); M0 / z0 may be None (zeros).  Returns a dict of fp64 numpy
    arrays: q, k, v, beta, M0, z0."""
    B, H, L, d = np.shape(q)
    Hkv = np.shape(k)[1]
    if M0 is None:
        M0 = np.zeros((B, Hkv, d, d))
    if z0 is None:
        z0 = np.zeros((B, Hkv, d))
    xs = {n: _t(x).requires_grad_(True) for n, x in
          (("q", q), ("k", k), ("v", v), ("beta", beta), ("M0", M0), ("z0", z0))}
    out, M, z = forward(xs["q"], xs["k"], xs["v"], xs["beta"], xs["M0"], xs["z0"], N, rule)
    loss = (out * _t(dout)).sum() + (M * _t(dM)).sum() + (z * _t(dz)).sum()
    grads = torch.autograd.grad(loss, list(xs.values()), allow_unused=True)
    return {n: (np.zeros(xs[n].shape) if g is None else g.detach().numpy())
            for n, g in zip(xs, grads)}


def forward_values(q, k, v, beta, M0, z0, *, N: int, rule: str = "linear"):
    """The restated forward's values (fp64 numpy), for pinning it to the C oracle."""
    B, H, L, d = np.shape(q)
    Hkv = np.shape(k)[1]
    if M0 is None:
        M0 = np.zeros((B, Hkv, d, d))
    if z0 is None:
        z0 = np.zeros((B, Hkv, d))
    with torch.no_grad():
        out, M, z = forward(_t(q), _t(k), _t(v), _t(beta), _t(M0), _t(z0), N, rule)
    return out.numpy(), M.numpy(), z.numpy()
