"""Thin ctypes binding of ``libinfini_attn.so`` (argument marshalling only).

Every step of the forward runs in the CUDA library; torch supplies device memory and the
current stream, nothing else.  There is no CPU fallback: if the library is missing or
fails to load, importing this module raises.

Names mirror the C ABI in ``include/infini_attn.h``:
``infini_attn_fwd`` (bf16), ``infini_attn_fwd_f32``, ``infini_attn_workspace_bytes``,
``infini_attn_status_string``, ``infini_attn_version``, ``infini_attn_decode_step`` (+
``_f32``), ``infini_attn_fold`` (+ ``_f32``), ``infini_attn_state`` (+ ``_f32``);
``forward``, ``decode_step``, ``fold`` and ``state`` allocate what is missing and pick the
entry point from the activation dtype.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

LINEAR = 0
DELTA = 1
RULES = {"linear": LINEAR, "delta": DELTA, LINEAR: LINEAR, DELTA: DELTA}

STATUS = {0: "INFINI_OK", 1: "INFINI_ERR_INVALID_ARG", 2: "INFINI_ERR_UNSUPPORTED",
          3: "INFINI_ERR_CUDA", 4: "INFINI_ERR_OOM", 5: "INFINI_ERR_TIMEOUT"}

#: C functions and their (argtypes, restype), exactly as include/infini_attn.h declares them
_P, _I64, _I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
_FWD_ARGS = [_P] * 9 + [_I64] * 6 + [_I, _P]
_DEC_ARGS = [_P] * 6 + [_I64] + [_P] * 3 + [_I64] * 5 + [_I, _P]
_FOLD_ARGS = [_P, _P, _I64, _P, _P] + [_I64] * 4 + [_I, _P]
_STATE_ARGS = [_P] * 6 + [_I64] * 5 + [_I, _P]
_BWD_ARGS = [_P] * 15 + [_I64] * 6 + [_I, _P]
SIGNATURES = {
    "infini_attn_fwd": (_FWD_ARGS, _I),
    "infini_attn_fwd_f32": (_FWD_ARGS, _I),
    "infini_attn_fwd_noalloc": (_FWD_ARGS, _I),
    "infini_attn_decode_step": (_DEC_ARGS, _I),
    "infini_attn_decode_step_f32": (_DEC_ARGS, _I),
    "infini_attn_fold": (_FOLD_ARGS, _I),
    "infini_attn_fold_f32": (_FOLD_ARGS, _I),
    "infini_attn_state": (_STATE_ARGS, _I),
    "infini_attn_bwd": (_BWD_ARGS, _I),
    "infini_attn_bwd_f32": (_BWD_ARGS, _I),
    "infini_attn_state_f32": (_STATE_ARGS, _I),
    "infini_attn_workspace_bytes": ([_I64] * 5, _I64),
    "infini_attn_status_string": ([_I], ctypes.c_char_p),
    "infini_attn_version": ([], _I),
    "infini_attn_device_status": ([_P], _I),
    "infini_attn_trace_enable": ([_I], _I),
    "infini_attn_test_fail_allocations": ([_I], _I),
    "infini_attn_test_wait_limit": ([_I64], _I),
    "infini_attn_test_withhold_publish": ([_I], _I),
    "infini_attn_trace_report": ([ctypes.c_char_p, _I64], _I64),
}


class InfiniError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


def _load():
    path = _build.LIB
    if not os.path.exists(path) and os.environ.get("INFINI_NO_AUTOBUILD") != "1":
        _build.build()
    lib = ctypes.CDLL(path)
    for name, (args, res) in SIGNATURES.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


LIB = _load()


def infini_attn_status_string(status: int) -> str:
    return LIB.infini_attn_status_string(status).decode()


def infini_attn_version() -> int:
    return LIB.infini_attn_version()


def infini_attn_workspace_bytes(B, Hkv, L, N, d) -> int:
    return LIB.infini_attn_workspace_bytes(B, Hkv, L, N, d)


def infini_attn_device_status(stream=None) -> int:
    """Synchronise the stream; INFINI_ERR_TIMEOUT (5) if a bounded device wait gave up."""
    return LIB.infini_attn_device_status(_stream_handle(stream))


def infini_attn_test_fail_allocations(n: int) -> int:
    """Test hook: the next ``n`` workspace allocations fail (INFINI_ERR_OOM)."""
    return LIB.infini_attn_test_fail_allocations(int(n))


def infini_attn_test_wait_limit(cycles: int) -> int:
    """Test hook: bound of every device wait in SM cycles (<= 0 restores the default)."""
    return LIB.infini_attn_test_wait_limit(int(cycles))


def infini_attn_test_withhold_publish(on: bool) -> int:
    """Test hook: the fused 64-token kernel's first unit per head skips its publish."""
    return LIB.infini_attn_test_withhold_publish(1 if on else 0)


def infini_attn_trace_enable(on: bool) -> bool:
    return bool(LIB.infini_attn_trace_enable(1 if on else 0))


def infini_attn_trace_report() -> dict:
    """Per-kernel launches and total device milliseconds since the last report."""
    import json
    n = LIB.infini_attn_trace_report(None, 0)
    buf = ctypes.create_string_buffer(int(n) + 64)
    LIB.infini_attn_trace_report(buf, len(buf))
    return json.loads(buf.value.decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _call(fn, q, k, v, beta, M0, z0, out, M_out, z_out, N, rule, stream):
    B, H, L, d = q.shape
    Hkv = k.shape[1]
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M0), _ptr(z0), _ptr(out), _ptr(M_out),
            _ptr(z_out), B, H, Hkv, L, int(N), d, RULES[rule], _stream_handle(stream))
    if rc != 0:
        raise InfiniError(rc, infini_attn_status_string(rc))


def infini_attn_fwd(q, k, v, beta, M0, z0, out, M_out, z_out, N, rule, stream=None):
    """bf16 entry point; all tensors preallocated, contiguous, on one CUDA device."""
    _call(LIB.infini_attn_fwd, q, k, v, beta, M0, z0, out, M_out, z_out, N, rule, stream)


def infini_attn_fwd_f32(q, k, v, beta, M0, z0, out, M_out, z_out, N, rule, stream=None):
    """fp32 entry point; all tensors preallocated, contiguous, on one CUDA device."""
    _call(LIB.infini_attn_fwd_f32, q, k, v, beta, M0, z0, out, M_out, z_out, N, rule, stream)


def infini_attn_fwd_noalloc(q, k, v, beta, M0, z0, out, M_out, z_out, N, rule, stream=None):
    """bf16 entry point that allocates nothing (workspace: the library's fixed device array
    of NOALLOC_SCRATCH_BYTES); all tensors preallocated, contiguous, on one CUDA device."""
    _call(LIB.infini_attn_fwd_noalloc, q, k, v, beta, M0, z0, out, M_out, z_out, N, rule, stream)


#: size of the fixed device array infini_attn_fwd_noalloc uses as its workspace
NOALLOC_SCRATCH_BYTES = 16 << 20


def _check(t, name, dtype, shape, device):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or t.device != device or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)}")


def forward(q, k, v, beta, M0=None, z0=None, *, N: int, rule="linear", out=None,
            M_out=None, z_out=None, stream=None):
    """Allocate outputs (unless given) and run the forward on q's device and dtype.

    q [B,H,L,d], k/v [B,Hkv,L,d] (bf16 or fp32), beta [H] fp32, M0 [B,Hkv,d,d] / z0
    [B,Hkv,d] fp32 or None.  Returns (out, M_out, z_out).
    """
    B, H, L, d = q.shape
    Hkv = k.shape[1]
    dev = q.device
    _check(q, "q", q.dtype, (B, H, L, d), dev)
    _check(k, "k", q.dtype, (B, Hkv, L, d), dev)
    _check(v, "v", q.dtype, (B, Hkv, L, d), dev)
    _check(beta, "beta", torch.float32, (H,), dev)
    _check(M0, "M0", torch.float32, (B, Hkv, d, d), dev)
    _check(z0, "z0", torch.float32, (B, Hkv, d), dev)
    if out is None:
        out = torch.empty_like(q)
    if M_out is None:
        M_out = torch.empty((B, Hkv, d, d), dtype=torch.float32, device=dev)
    if z_out is None:
        z_out = torch.empty((B, Hkv, d), dtype=torch.float32, device=dev)
    if q.dtype == torch.bfloat16:
        infini_attn_fwd(q, k, v, beta, M0, z0, out, M_out, z_out, N, rule, stream)
    elif q.dtype == torch.float32:
        infini_attn_fwd_f32(q, k, v, beta, M0, z0, out, M_out, z_out, N, rule, stream)
    else:
        raise ValueError(f"unsupported activation dtype {q.dtype}")
    return out, M_out, z_out


def decode_step(q, k, v, beta, k_cache, v_cache, pos: int, M, z, *, rule="linear", out=None,
                stream=None):
    """One token of every (batch, head) at offset ``pos`` of its current segment.

    q [B,H,d], k/v [B,Hkv,d] (bf16 or fp32), beta [H] fp32, k_cache/v_cache [B,Hkv,N,d]
    (the activation dtype; row ``pos`` is written), M [B,Hkv,d,d] / z [B,Hkv,d] fp32 (folded
    in place when pos == N - 1).  Returns out [B,H,d].
    """
    B, H, d = q.shape
    Hkv, N = k_cache.shape[1], k_cache.shape[2]
    dev = q.device
    _check(q, "q", q.dtype, (B, H, d), dev)
    _check(k, "k", q.dtype, (B, Hkv, d), dev)
    _check(v, "v", q.dtype, (B, Hkv, d), dev)
    _check(beta, "beta", torch.float32, (H,), dev)
    _check(k_cache, "k_cache", q.dtype, (B, Hkv, N, d), dev)
    _check(v_cache, "v_cache", q.dtype, (B, Hkv, N, d), dev)
    _check(M, "M", torch.float32, (B, Hkv, d, d), dev)
    _check(z, "z", torch.float32, (B, Hkv, d), dev)
    if out is None:
        out = torch.empty_like(q)
    if q.dtype == torch.bfloat16:
        fn = LIB.infini_attn_decode_step
    elif q.dtype == torch.float32:
        fn = LIB.infini_attn_decode_step_f32
    else:
        raise ValueError(f"unsupported activation dtype {q.dtype}")
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(k_cache), _ptr(v_cache), int(pos),
            _ptr(M), _ptr(z), _ptr(out), B, H, Hkv, N, d, RULES[rule], _stream_handle(stream))
    if rc != 0:
        raise InfiniError(rc, infini_attn_status_string(rc))
    return out


def fold(k_cache, v_cache, n: int, M, z, *, rule="linear", stream=None):
    """Fold the first ``n`` cached rows of every chain into (M, z), in place."""
    B, Hkv, N, d = k_cache.shape
    dev = k_cache.device
    _check(v_cache, "v_cache", k_cache.dtype, (B, Hkv, N, d), dev)
    _check(M, "M", torch.float32, (B, Hkv, d, d), dev)
    _check(z, "z", torch.float32, (B, Hkv, d), dev)
    if k_cache.dtype == torch.bfloat16:
        fn = LIB.infini_attn_fold
    elif k_cache.dtype == torch.float32:
        fn = LIB.infini_attn_fold_f32
    else:
        raise ValueError(f"unsupported activation dtype {k_cache.dtype}")
    rc = fn(_ptr(k_cache), _ptr(v_cache), int(n), _ptr(M), _ptr(z), B, Hkv, N, d, RULES[rule],
            _stream_handle(stream))
    if rc != 0:
        raise InfiniError(rc, infini_attn_status_string(rc))


def state(k, v, M0=None, z0=None, *, N: int, rule="linear", M_out=None, z_out=None,
          stream=None):
    """The memory after the whole sequence without the outputs: k/v [B,Hkv,L,d] (bf16 or
    fp32), M0 [B,Hkv,d,d] / z0 [B,Hkv,d] fp32 or None.  Returns (M_out, z_out)."""
    B, Hkv, L, d = k.shape
    dev = k.device
    _check(k, "k", k.dtype, (B, Hkv, L, d), dev)
    _check(v, "v", k.dtype, (B, Hkv, L, d), dev)
    _check(M0, "M0", torch.float32, (B, Hkv, d, d), dev)
    _check(z0, "z0", torch.float32, (B, Hkv, d), dev)
    if M_out is None:
        M_out = torch.empty((B, Hkv, d, d), dtype=torch.float32, device=dev)
    if z_out is None:
        z_out = torch.empty((B, Hkv, d), dtype=torch.float32, device=dev)
    if k.dtype == torch.bfloat16:
        fn = LIB.infini_attn_state
    elif k.dtype == torch.float32:
        fn = LIB.infini_attn_state_f32
    else:
        raise ValueError(f"unsupported activation dtype {k.dtype}")
    rc = fn(_ptr(k), _ptr(v), _ptr(M0), _ptr(z0), _ptr(M_out), _ptr(z_out), B, Hkv, L, int(N),
            d, RULES[rule], _stream_handle(stream))
    if rc != 0:
        raise InfiniError(rc, infini_attn_status_string(rc))
    return M_out, z_out


def backward(q, k, v, beta, M0, z0, dout, dM=None, dz=None, *, N: int, rule="linear",
             stream=None):
    """Gradients of <dout, out> + <dM, M_out> + <dz, z_out> of the forward with these inputs.

    q [B,H,L,d], k/v [B,Hkv,L,d] and dout [B,H,L,d] (bf16 or fp32), beta [H], M0/z0 and dM/dz
    fp32 or None.  Returns (dq, dk, dv, dbeta, dM0, dz0).
    """
    B, H, L, d = q.shape
    Hkv = k.shape[1]
    dev = q.device
    _check(q, "q", q.dtype, (B, H, L, d), dev)
    _check(k, "k", q.dtype, (B, Hkv, L, d), dev)
    _check(v, "v", q.dtype, (B, Hkv, L, d), dev)
    _check(dout, "dout", q.dtype, (B, H, L, d), dev)
    _check(beta, "beta", torch.float32, (H,), dev)
    _check(M0, "M0", torch.float32, (B, Hkv, d, d), dev)
    _check(z0, "z0", torch.float32, (B, Hkv, d), dev)
    _check(dM, "dM", torch.float32, (B, Hkv, d, d), dev)
    _check(dz, "dz", torch.float32, (B, Hkv, d), dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dbeta = torch.empty((H,), dtype=torch.float32, device=dev)
    dM0 = torch.empty((B, Hkv, d, d), dtype=torch.float32, device=dev)
    dz0 = torch.empty((B, Hkv, d), dtype=torch.float32, device=dev)
    if q.dtype == torch.bfloat16:
        fn = LIB.infini_attn_bwd
    elif q.dtype == torch.float32:
        fn = LIB.infini_attn_bwd_f32
    else:
        raise ValueError(f"unsupported activation dtype {q.dtype}")
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M0), _ptr(z0), _ptr(dout), _ptr(dM),
            _ptr(dz), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbeta), _ptr(dM0), _ptr(dz0), B, H, Hkv,
            L, int(N), d, RULES[rule], _stream_handle(stream))
    if rc != 0:
        raise InfiniError(rc, infini_attn_status_string(rc))
    return dq, dk, dv, dbeta, dM0, dz0
