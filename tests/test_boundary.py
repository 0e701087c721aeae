"""The C-ABI boundary on the host: the library loads, exports every symbol the header
declares with the declared signature, and rejects bad arguments before any CUDA call
(these calls pass fake device addresses that argument checking never dereferences)."""
import ctypes
import os
import re

import pytest

from compressive_memory_long_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"INFINI_API\s+[\w\s\*]+?\b(infini_\w+)\s*\(", src)
    return names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert "infini_attn_fwd" in names and "infini_attn_fwd_f32" in names
    lib = ctypes.CDLL(build.LIB)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
        assert n in binding.SIGNATURES, f"{n} has no binding"


def test_status_strings_and_version():
    for s in range(6):
        assert binding.infini_attn_status_string(s)
    assert "unknown" in binding.infini_attn_status_string(99)
    assert binding.infini_attn_version() >= 100


def tc_bytes(units, d, delta=True):
    """z_{s-1} and dz_s (fp32), bf16 M_{s-1}, fp32 B_s, bf16 hi / lo A_s, per segment."""
    return units * (2 * d * 4 + d * d * 2 + d * d * 4 + (2 * d * d * 2 if delta else 0)) + 256


def test_workspace_bytes():
    """An upper bound over every path: the tensor-core memory path's per-segment state is
    the larger one (the CUDA-core path keeps fp32 snapshots only)."""
    units = 2 * 8 * 16
    assert binding.infini_attn_workspace_bytes(2, 8, 1024, 64, 64) == tc_bytes(units, 64)
    assert tc_bytes(units, 64) >= units * (64 * 64 + 64) * 4 + 256
    # a final short segment counts as a segment
    assert binding.infini_attn_workspace_bytes(1, 1, 100, 64, 64) == tc_bytes(2, 64)
    assert binding.infini_attn_workspace_bytes(1, 1, 40, 64, 64) == tc_bytes(1, 64)
    assert binding.infini_attn_workspace_bytes(1, 4, 8192, 2048, 128) == tc_bytes(16, 128)
    assert binding.infini_attn_workspace_bytes(0, 1, 64, 64, 64) == 0


def test_allocation_failure_hook_arguments():
    """The host-side hook only counts: a negative count is refused, 0 disarms it."""
    assert binding.infini_attn_test_fail_allocations(-1) == 1
    assert binding.infini_attn_test_fail_allocations(0) == 0


BASE = 1 << 40      # fake, 16-byte aligned, never dereferenced


def call(entry="infini_attn_fwd", B=1, H=2, Hkv=2, L=128, N=64, d=64, rule=0, **ptr):
    """Call an entry point with disjoint fake device ranges; override any pointer."""
    gap = 1 << 32
    p = {name: BASE + i * gap for i, name in enumerate(
        ["q", "k", "v", "beta", "M0", "z0", "out", "M_out", "z_out"])}
    p.update(ptr)
    f = getattr(binding.LIB, entry)
    args = [None if p[n] is None else ctypes.c_void_p(p[n]) for n in
            ["q", "k", "v", "beta", "M0", "z0", "out", "M_out", "z_out"]]
    return f(*args, B, H, Hkv, L, N, d, rule, None)


INVALID, UNSUPPORTED = 1, 2


@pytest.mark.parametrize("entry", ["infini_attn_fwd", "infini_attn_fwd_f32"])
@pytest.mark.parametrize("kw,status", [
    (dict(q=None), INVALID), (dict(k=None), INVALID), (dict(v=None), INVALID),
    (dict(beta=None), INVALID), (dict(out=None), INVALID), (dict(M_out=None), INVALID),
    (dict(z_out=None), INVALID),
    (dict(B=0), INVALID), (dict(H=0), INVALID), (dict(L=-64), INVALID), (dict(N=0), INVALID),
    (dict(d=0), INVALID), (dict(H=3, Hkv=2), INVALID),
    (dict(rule=2), INVALID), (dict(rule=-1), INVALID),
    (dict(q=BASE + 8), INVALID), (dict(M_out=BASE + (7 << 32) + 4), INVALID),
    (dict(M_out=(1 << 40) + (4 << 32) + 64), INVALID),     # partial overlap with M0
    (dict(z_out=(1 << 40) + (5 << 32) + 16), INVALID),     # partial overlap with z0
    (dict(out=BASE), INVALID),                             # out on top of q
    (dict(d=48), UNSUPPORTED), (dict(d=256), UNSUPPORTED), (dict(L=96, N=32), UNSUPPORTED),
])
def test_argument_errors(entry, kw, status):
    assert call(entry, **kw) == status


def test_python_binding_checks_shapes():
    import torch
    q = torch.zeros(1, 2, 64, 32)
    with pytest.raises(ValueError):
        binding.forward(q, q, q, torch.zeros(2), N=64)     # CPU tensors are refused


DEC_PTRS = ["q", "k", "v", "beta", "k_cache", "v_cache", "M", "z", "out"]


def call_decode(entry="infini_attn_decode_step", B=1, H=2, Hkv=2, N=64, d=64, pos=0, rule=0,
                **ptr):
    gap = 1 << 32
    p = {name: BASE + i * gap for i, name in enumerate(DEC_PTRS)}
    p.update(ptr)
    a = [None if p[n] is None else ctypes.c_void_p(p[n]) for n in DEC_PTRS]
    f = getattr(binding.LIB, entry)
    return f(a[0], a[1], a[2], a[3], a[4], a[5], pos, a[6], a[7], a[8], B, H, Hkv, N, d, rule,
             None)


@pytest.mark.parametrize("entry", ["infini_attn_decode_step", "infini_attn_decode_step_f32"])
@pytest.mark.parametrize("kw,status", [
    *[(dict({n: None}), INVALID) for n in DEC_PTRS],
    (dict(pos=-1), INVALID), (dict(pos=64), INVALID), (dict(N=0), INVALID),
    (dict(H=3, Hkv=2), INVALID), (dict(Hkv=0), INVALID), (dict(rule=2), INVALID),
    (dict(q=BASE + 8), INVALID), (dict(k_cache=BASE + (4 << 32) + 4), INVALID),
    (dict(v_cache=BASE + (4 << 32)), INVALID),                 # both caches at one address
    (dict(out=BASE + (6 << 32)), INVALID),                     # out on top of M
    (dict(z=BASE + (6 << 32) + 64), INVALID),                  # z inside M
    (dict(d=48), UNSUPPORTED), (dict(d=256), UNSUPPORTED),
])
def test_decode_argument_errors(entry, kw, status):
    assert call_decode(entry, **kw) == status


FOLD_PTRS = ["k_cache", "v_cache", "M", "z"]


def call_fold(entry="infini_attn_fold", n=1, B=1, Hkv=2, N=64, d=64, rule=0, **ptr):
    gap = 1 << 32
    p = {name: BASE + i * gap for i, name in enumerate(FOLD_PTRS)}
    p.update(ptr)
    a = [None if p[x] is None else ctypes.c_void_p(p[x]) for x in FOLD_PTRS]
    return getattr(binding.LIB, entry)(a[0], a[1], n, a[2], a[3], B, Hkv, N, d, rule, None)


@pytest.mark.parametrize("entry", ["infini_attn_fold", "infini_attn_fold_f32"])
@pytest.mark.parametrize("kw,status", [
    *[(dict({n: None}), INVALID) for n in FOLD_PTRS],
    (dict(n=-1), INVALID), (dict(n=65), INVALID), (dict(B=0), INVALID), (dict(rule=-1), INVALID),
    (dict(M=BASE + (2 << 32) + 4), INVALID), (dict(z=BASE + (2 << 32)), INVALID),
    (dict(d=16), UNSUPPORTED),
    (dict(n=0), 0),                     # nothing to fold: returns before any CUDA call
])
def test_fold_argument_errors(entry, kw, status):
    assert call_fold(entry, **kw) == status


STATE_PTRS = ["k", "v", "M0", "z0", "M_out", "z_out"]


def call_state(entry="infini_attn_state", B=1, Hkv=2, L=128, N=64, d=64, rule=0, **ptr):
    gap = 1 << 32
    p = {name: BASE + i * gap for i, name in enumerate(STATE_PTRS)}
    p.update(ptr)
    a = [None if p[x] is None else ctypes.c_void_p(p[x]) for x in STATE_PTRS]
    return getattr(binding.LIB, entry)(*a, B, Hkv, L, N, d, rule, None)


@pytest.mark.parametrize("entry", ["infini_attn_state", "infini_attn_state_f32"])
@pytest.mark.parametrize("kw,status", [
    (dict(k=None), INVALID), (dict(v=None), INVALID), (dict(M_out=None), INVALID),
    (dict(z_out=None), INVALID), (dict(B=0), INVALID), (dict(L=0), INVALID),
    (dict(rule=5), INVALID), (dict(k=BASE + 4), INVALID),
    (dict(M_out=BASE + (2 << 32) + 64), INVALID),            # partial overlap with M0
    (dict(M_out=BASE), INVALID),                             # on top of k
    (dict(z_out=BASE + (1 << 32) + 16), INVALID),            # inside v
    (dict(d=48), UNSUPPORTED), (dict(N=100), UNSUPPORTED),
])
def test_state_argument_errors(entry, kw, status):
    assert call_state(entry, **kw) == status


BWD_PTRS = ["q", "k", "v", "beta", "M0", "z0", "dout", "dM", "dz", "dq", "dk", "dv", "dbeta",
            "dM0", "dz0"]


def call_bwd(entry="infini_attn_bwd", B=1, H=2, Hkv=2, L=128, N=64, d=64, rule=0, **ptr):
    gap = 1 << 32
    p = {name: BASE + i * gap for i, name in enumerate(BWD_PTRS)}
    p.update(ptr)
    a = [None if p[x] is None else ctypes.c_void_p(p[x]) for x in BWD_PTRS]
    return getattr(binding.LIB, entry)(*a, B, H, Hkv, L, N, d, rule, None)


@pytest.mark.parametrize("entry", ["infini_attn_bwd", "infini_attn_bwd_f32"])
@pytest.mark.parametrize("kw,status", [
    *[(dict({n: None}), INVALID) for n in ("q", "k", "v", "beta", "dout", "dq", "dk", "dv")],
    (dict(B=0), INVALID), (dict(H=3, Hkv=2), INVALID), (dict(rule=2), INVALID),
    (dict(q=BASE + 8), INVALID),
    (dict(dq=BASE), INVALID),                                # dq on top of q
    (dict(dk=BASE + (9 << 32) + 64), INVALID),               # dk inside dq
    (dict(dM0=BASE + (4 << 32)), INVALID),                   # dM0 on top of M0
    (dict(d=48), UNSUPPORTED), (dict(N=100), UNSUPPORTED),
])
def test_backward_argument_errors(entry, kw, status):
    assert call_bwd(entry, **kw) == status
