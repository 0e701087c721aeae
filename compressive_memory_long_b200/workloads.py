"""Seeded synthetic workloads for the Infini-attention forward pass.

This module holds input generation only -- none of the method's arithmetic -- so that
the CUDA path (tests, benchmark) and the CPU oracle draw exactly the same inputs.

Every tensor slice is drawn from its own numpy ``PCG64`` stream keyed by
``SeedSequence([seed, tensor_code, b, head])``.  A slice of one (batch, head) can
therefore be regenerated alone, which is how the oracle checks sampled heads of the
large workloads.  Values are drawn in float32, scaled in float32, then rounded to the
input dtype (bf16: round-to-nearest-even).  The oracle receives those rounded values
widened back to float32, which is exact.

Shapes follow the pages' workloads: 64-token segments with 16 rollouts (the Hugging
Face reproduction, "Infini-Attention Mechanism" / "Weight Decay and Rollouts"),
2048-token segments (AI Wiki "Infini-Attention", "Why is the memory footprint
bounded?"), a 1M-token stream for a 1B-class model and a GQA 8B-class head layout
("Can Infini-attention retrieve a passkey at one million tokens?", "What were the
results on 500K book summarization?").  No dataset is involved: the passkey, BookSum
and PG19 inputs are stood in for by their shapes only.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import math
from typing import Optional, Tuple

import numpy as np
import torch

_CODE = {"q": 1, "k": 2, "v": 3, "beta": 4, "M0": 5, "z0": 6, "kboost": 7}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Hkv: int
    d: int
    N: int
    S: int
    dtype: str            # "f32" or "bf16": dtype of q, k, v and out
    rule: str             # "linear" or "delta"
    seed: int
    beta_dist: Tuple      # ("normal", mean, std) or ("uniform", lo, hi)
    M0_dist: Optional[Tuple] = None   # None: zeros; ("uniform", lo, hi)
    z0_dist: Optional[Tuple] = None
    k_boost_frac: float = 0.0         # fraction of K rows (per (b, kv head)) scaled ...
    k_boost: float = 1.0              # ... by this factor before rounding
    description: str = ""
    tail: int = 0                     # tokens of a final segment shorter than N (0 <= tail < N)

    @property
    def L(self) -> int:
        return self.N * self.S + self.tail

    @property
    def G(self) -> int:
        return self.H // self.Hkv

    @property
    def tokens(self) -> int:
        return self.B * self.L

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    w.name: w for w in [
        Workload("fp32_linear_small", B=1, H=2, Hkv=2, d=32, N=64, S=4, dtype="f32",
                 rule="linear", seed=0, beta_dist=("normal", 0.0, 1.0),
                 description="fp32 linear-update correctness: B1 H2 d32, N64 x 4 segments"),
        Workload("hf_repro_n64", B=2, H=8, Hkv=8, d=64, N=64, S=16, dtype="bf16",
                 rule="linear", seed=1, beta_dist=("uniform", -3.0, 3.0),
                 description="HF-reproduction shape: B2 H8 d64, 64-token segments x 16 rollouts"),
        Workload("gqa8b_n2048_delta", B=1, H=32, Hkv=8, d=128, N=2048, S=16, dtype="bf16",
                 rule="delta", seed=2, beta_dist=("normal", 0.0, 1.0),
                 description="8B-class GQA: 32 q heads / 8 kv heads, d128, N2048 x 16"),
        Workload("stream1m_n2048_delta", B=1, H=16, Hkv=16, d=128, N=2048, S=512,
                 dtype="bf16", rule="delta", seed=3, beta_dist=("normal", 0.0, 2.0),
                 k_boost_frac=0.01, k_boost=4.0,
                 description="1B-class 1M-token stream: H16 d128, N2048 x 512, 1% of K rows x4"),
        Workload("batched_n1024_linear", B=16, H=32, Hkv=32, d=128, N=1024, S=8,
                 dtype="bf16", rule="linear", seed=4, beta_dist=("normal", 0.0, 1.0),
                 M0_dist=("uniform", 0.0, 0.1), z0_dist=("uniform", 1.0, 2.0),
                 description="batched throughput: B16 H32 d128, N1024 x 8, nonzero M0/z0"),
        Workload("n64_bandwidth", B=2, H=8, Hkv=8, d=64, N=64, S=16384, dtype="bf16",
                 rule="linear", seed=1, beta_dist=("uniform", -3.0, 3.0),
                 description="HF-reproduction head shape at N64 over a 1M-token stream"),
    ]
}


def _rng(w: Workload, tensor: str, b: int = 0, head: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(
        [w.seed, _CODE[tensor], b, head])))


def _round(x: np.ndarray, w: Workload) -> np.ndarray:
    """Round float32 values to the input dtype and widen back (exact) to float32."""
    if w.dtype == "f32":
        return x
    t = torch.from_numpy(x).to(torch.bfloat16)
    return t.to(torch.float32).numpy()


def qkv_slice(w: Workload, tensor: str, b: int, head: int, rows: Optional[int] = None) -> np.ndarray:
    """[L, d] float32 values (already rounded to the input dtype) of one head.

    ``rows``: draw only the first ``rows`` tokens (the same values as the full draw's
    prefix: the generator fills row by row)."""
    assert tensor in ("q", "k", "v")
    n_rows = w.L if rows is None else rows
    x = _rng(w, tensor, b, head).standard_normal((n_rows, w.d), dtype=np.float32)
    x = x / np.float32(math.sqrt(w.d))
    if tensor == "k" and w.k_boost_frac > 0.0:
        n = int(round(w.L * w.k_boost_frac))
        sel = _rng(w, "kboost", b, head).choice(w.L, size=n, replace=False)
        x[sel[sel < n_rows]] *= np.float32(w.k_boost)
    return _round(np.ascontiguousarray(x), w)


def _draw(rng: np.random.Generator, dist: Tuple, shape) -> np.ndarray:
    kind = dist[0]
    if kind == "normal":
        return (rng.standard_normal(shape, dtype=np.float32) * np.float32(dist[2])
                + np.float32(dist[1])).astype(np.float32)
    if kind == "uniform":
        return rng.uniform(dist[1], dist[2], size=shape).astype(np.float32)
    raise ValueError(kind)


def beta(w: Workload) -> np.ndarray:
    return _draw(_rng(w, "beta"), w.beta_dist, (w.H,))


def initial_state(w: Workload, b: int, kvh: int):
    """(M0 [d,d], z0 [d]) float32 for one (batch, kv head); zeros when not drawn."""
    M0 = (np.zeros((w.d, w.d), np.float32) if w.M0_dist is None
          else _draw(_rng(w, "M0", b, kvh), w.M0_dist, (w.d, w.d)))
    z0 = (np.zeros((w.d,), np.float32) if w.z0_dist is None
          else _draw(_rng(w, "z0", b, kvh), w.z0_dist, (w.d,)))
    return M0, z0


def has_initial_state(w: Workload) -> bool:
    return w.M0_dist is not None or w.z0_dist is not None


def host_slices(w: Workload, b: int, kvh: int, rows: Optional[int] = None):
    """float32 inputs of one (batch, kv head) and its G query heads, for the oracle.

    Returns q [1,G,L,d], k [1,1,L,d], v [1,1,L,d], beta [G], M0 [1,1,d,d], z0 [1,1,d]
    (L replaced by ``rows`` when given: the first ``rows`` tokens only).
    """
    q = np.stack([qkv_slice(w, "q", b, kvh * w.G + g, rows) for g in range(w.G)])[None]
    k = qkv_slice(w, "k", b, kvh, rows)[None, None]
    v = qkv_slice(w, "v", b, kvh, rows)[None, None]
    bt = beta(w)[kvh * w.G:(kvh + 1) * w.G]
    M0, z0 = initial_state(w, b, kvh)
    return q, k, v, bt, M0[None, None], z0[None, None]


def host_inputs(w: Workload):
    """All inputs as float32 numpy arrays (small workloads only)."""
    q = np.stack([np.stack([qkv_slice(w, "q", b, h) for h in range(w.H)]) for b in range(w.B)])
    k = np.stack([np.stack([qkv_slice(w, "k", b, h) for h in range(w.Hkv)]) for b in range(w.B)])
    v = np.stack([np.stack([qkv_slice(w, "v", b, h) for h in range(w.Hkv)]) for b in range(w.B)])
    st = [[initial_state(w, b, h) for h in range(w.Hkv)] for b in range(w.B)]
    M0 = np.stack([np.stack([s[0] for s in row]) for row in st])
    z0 = np.stack([np.stack([s[1] for s in row]) for row in st])
    return q, k, v, beta(w), M0, z0


def torch_inputs(w: Workload, device="cpu", pin_memory: bool = False, threads: int = 8):
    """All inputs as torch tensors in the input dtype (q, k, v) and float32 (the rest).

    Slices are drawn in parallel threads (numpy's generators release the GIL) and written
    straight into the destination tensors, so peak host memory stays near one copy.
    Returns dict(q, k, v, beta, M0, z0); M0/z0 are None when the workload starts from
    an empty memory.
    """
    dt = w.torch_dtype
    host = device == "cpu" or pin_memory

    def alloc(shape):
        if host:
            return torch.empty(shape, dtype=dt, pin_memory=pin_memory)
        return torch.empty(shape, dtype=dt, device=device)

    out = {"q": alloc((w.B, w.H, w.L, w.d)), "k": alloc((w.B, w.Hkv, w.L, w.d)),
           "v": alloc((w.B, w.Hkv, w.L, w.d))}
    jobs = [(t, b, h) for t, nh in (("q", w.H), ("k", w.Hkv), ("v", w.Hkv))
            for b in range(w.B) for h in range(nh)]

    def fill(job):
        t, b, h = job
        x = torch.from_numpy(qkv_slice(w, t, b, h)).to(dt)
        out[t][b, h].copy_(x)

    with _cf.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fill, jobs))
    out["beta"] = torch.from_numpy(beta(w))
    if has_initial_state(w):
        _, _, _, _, M0, z0 = host_inputs_state_only(w)
        out["M0"], out["z0"] = torch.from_numpy(M0), torch.from_numpy(z0)
    else:
        out["M0"], out["z0"] = None, None
    if not host or pin_memory:
        for key in ("beta", "M0", "z0"):
            if out[key] is not None:
                out[key] = out[key].pin_memory() if pin_memory else out[key].to(device)
    return out


def host_inputs_state_only(w: Workload):
    st = [[initial_state(w, b, h) for h in range(w.Hkv)] for b in range(w.B)]
    M0 = np.stack([np.stack([s[0] for s in row]) for row in st])
    z0 = np.stack([np.stack([s[1] for s in row]) for row in st])
    return None, None, None, None, M0, z0
