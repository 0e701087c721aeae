"""fp64 CPU oracle of the Infini-attention forward pass (ctypes loader).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg are the only callers.  The CUDA library never
imports, links or runs anything here, and nothing here imports the CUDA library.

The arithmetic lives in ``infini_oracle.c`` (plain loops, one thread, double
precision), written from AI Wiki "Infini-Attention", sections "What happens inside the
Infini-attention block?" and "How does the compressive memory work?".  Its pins (the
checks that tie it to the pages and to mathematics rather than to itself) are in
``tests/test_oracle_pins.py``.  ``backward.py`` holds fp64 reference gradients of the same
forward (for a backward pass not built yet), pinned in ``tests/test_backward_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "infini_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")

LINEAR = 0
DELTA = 1
_RULES = {"linear": LINEAR, "delta": DELTA, LINEAR: LINEAR, DELTA: DELTA}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math, so IEEE double semantics hold)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
                           "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _bind(path: str):
    lib = ctypes.CDLL(path)
    f = lib.oracle_infini_attn_fwd
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    f.argtypes = [P, P, P, P, P, P, P, P, P, I64, I64, I64, I64, I64, I64, ctypes.c_int, P]
    f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def source() -> str:
    with open(_SRC) as fh:
        return fh.read()


def compile_variant(src: str, out_dir: str) -> str:
    """Compile a modified copy of the oracle source (used by the tests that plant mistakes
    in the oracle to show its pins catch them).  Returns the shared-library path."""
    c_path = os.path.join(out_dir, "variant.c")
    so_path = os.path.join(out_dir, "libvariant.so")
    with open(c_path, "w") as fh:
        fh.write(src)
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
                           "-ffp-contract=off", "-o", so_path, c_path, "-lm"])
    return so_path


def _f32(a):
    if a is None:
        return None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def infini_attn_fwd(q, k, v, beta, M0=None, z0=None, *, N: int, rule="linear",
                    seg_out=None, out=None, lib_path=None):
    """Run the oracle.

    q [B,H,L,d], k/v [B,Hkv,L,d], beta [H], M0 [B,Hkv,d,d] or None, z0 [B,Hkv,d] or None.
    Inputs are converted to float32 (bf16 values widen exactly); results are float64.
    ``seg_out``: optional iterable of segment indices whose outputs are computed (all
    segments' memory updates always run).  ``out``: optional float64 array to fill
    (rows of segments not in ``seg_out`` keep its contents; default zeros).
    ``lib_path``: run a variant compiled by ``compile_variant`` instead of the oracle.
    Returns (out [B,H,L,d], M_out [B,Hkv,d,d], z_out [B,Hkv,d]).
    """
    q, k, v, beta, M0, z0 = (_f32(x) for x in (q, k, v, beta, M0, z0))
    B, H, L, d = q.shape
    Hkv = k.shape[1]
    assert k.shape == (B, Hkv, L, d) and v.shape == k.shape and beta.shape == (H,)
    if M0 is not None:
        assert M0.shape == (B, Hkv, d, d)
    if z0 is not None:
        assert z0.shape == (B, Hkv, d)
    S = -(-L // N)
    mask = None
    if seg_out is not None:
        mask = np.zeros(S, dtype=np.uint8)
        mask[list(seg_out)] = 1
    if out is None:
        out = np.zeros((B, H, L, d), dtype=np.float64)
    assert out.dtype == np.float64 and out.shape == (B, H, L, d) and out.flags.c_contiguous
    M_out = np.zeros((B, Hkv, d, d), dtype=np.float64)
    z_out = np.zeros((B, Hkv, d), dtype=np.float64)
    lib = _load() if lib_path is None else _bind(lib_path)
    rc = lib.oracle_infini_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M0),
                                        _ptr(z0), _ptr(out), _ptr(M_out), _ptr(z_out),
                                        B, H, Hkv, L, N, d, _RULES[rule], _ptr(mask))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (status {rc})")
    return out, M_out, z_out
