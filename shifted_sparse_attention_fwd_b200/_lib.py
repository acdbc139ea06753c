"""ctypes binding of libs2attn.so (the C ABI declared in include/s2attn.h).

Argument marshalling only: every step of S²-Attn runs in the library's CUDA kernels.
Functions carry the C names; tensors are torch CUDA tensors (device memory and streams are
torch's), passed as raw pointers. There is no CPU fallback: if the library cannot be
loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libs2attn.so")

S2ATTN_OK = 0
S2ATTN_ERR_INVALID_ARG = 1
S2ATTN_ERR_UNSUPPORTED = 2
S2ATTN_ERR_CUDA = 3
S2ATTN_ERR_TIMEOUT = 4

# option flags of the _general entry points (include/s2attn.h)
S2ATTN_FLAG_WRAP_OWN_GROUP = 1
S2ATTN_FLAG_WRAP_FRONT_FIRST = 2
S2ATTN_FLAG_PARTIAL_LAST_GROUP = 4

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/s2attn.h
SIGNATURES = {
    "s2attn_abi_version": (_I, []),
    "s2attn_status_string": (ctypes.c_char_p, [_I]),
    "s2attn_last_error": (ctypes.c_char_p, []),
    "s2attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "s2attn_fwd_ex": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "s2attn_bwd_workspace_size": (_Z, [_I, _I, _I]),
    "s2attn_bwd": (_I, [_P] * 9 + [_I] * 6 + [_F, _P, _Z, _P]),
    "s2attn_bwd_ex": (_I, [_P] * 9 + [_I] * 6 + [_F, _I, _I, _P, _Z, _P]),
    "s2attn_bwd_preprocess": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _Z, _P]),
    "s2attn_bwd_dkdv": (_I, [_P] * 6 + [_I] * 6 + [_F, _I, _I, _P, _Z, _P]),
    "s2attn_bwd_dq": (_I, [_P] * 5 + [_I] * 6 + [_F, _I, _I, _P, _Z, _P]),
    "s2attn_bwd_noalloc": (_I, [_P] * 9 + [_I] * 6 + [_F, _P]),
    "s2attn_bwd_workspace_size_ex": (_Z, [_I] * 8 + [_Z]),
    "s2attn_fwd_general": (_I, [_P] * 5 + [_I] * 6 + [_F, _I, _I, _I, _P, _P]),
    "s2attn_fwd_rope_q": (_I, [_P] * 6 + [_I] * 6 + [_F, _I, _I, _I, _F, _F, _P]),
    "s2attn_bwd_general": (_I, [_P] * 9 + [_I] * 6 + [_F, _I, _I, _I, _P, _P, _Z, _P]),
    "s2attn_bwd_workspace_size_general": (_Z, [_I] * 9 + [_Z]),
    "s2attn_rope_pi": (_I, [_P, _P, _I, _I, _I, _I, _F, _F, _I, _P, _P]),
    "s2attn_bwd_dkdv_ds": (_I, [_P] * 6 + [_I] * 6 + [_F, _I, _I, _P, _Z, _P]),
    "s2attn_bwd_dq_ds": (_I, [_P] * 2 + [_I] * 6 + [_F, _I, _I, _P, _Z, _P]),
    "s2attn_bwd_dkdv_ds_general": (_I, [_P] * 6 + [_I] * 6 + [_F, _I, _I, _I, _P, _P, _Z, _P]),
    "s2attn_bwd_dq_ds_general": (_I, [_P] * 2 + [_I] * 6 + [_F, _I, _I, _I, _P, _P, _Z, _P]),
    "s2attn_get_device_error": (_I, [_P, ctypes.POINTER(ctypes.c_uint)]),
    "s2attn_set_wait_timeout_ns": (None, [ctypes.c_ulonglong]),
    "s2attn_selftest_wait_timeout": (_I, [ctypes.c_ulonglong, _P]),
}

_lib = None


class S2AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)}"
        if status == S2ATTN_ERR_CUDA:
            msg += f" ({lib().s2attn_last_error().decode()})"
        super().__init__(msg)


def lib():
    """Load libs2attn.so once; raise if it is missing (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m shifted_sparse_attention_fwd_b200.build` (nvcc, sm_100a)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().s2attn_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != S2ATTN_OK:
        raise S2AttnError(status, where)


def _ptr(t, strided=False):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        return t  # raw integer address
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not strided and not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _bn_strides(t):
    """(batch, token) element strides of a [B, N, H, d] tensor whose (H, d) block is contiguous."""
    if t.dim() != 4 or t.stride(3) != 1 or t.stride(2) != t.shape[3]:
        raise ValueError("expected a [B, N, H, d] tensor with contiguous (H, d) blocks")
    return [t.stride(0), t.stride(1)]


def _strides_array(*ts):
    vals = []
    for t in ts:
        vals += _bn_strides(t)
    return (ctypes.c_longlong * len(vals))(*vals)


def _all_contiguous(*ts):
    return all(t.is_contiguous() for t in ts if isinstance(t, torch.Tensor))


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dims(q, k, G):
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    return B, Hq, Hkv, N, d, G


def _check_bf16(*ts):
    for t in ts:
        if t is not None and isinstance(t, torch.Tensor) and t.dtype != torch.bfloat16:
            raise ValueError(f"expected bf16, got {t.dtype}")


def s2attn_fwd(q, k, v, o, lse, G, scale=None, shift_head_begin=None, shift=None, stream=None,
               flags=0):
    """O and LSE of S²-Attn. q [B,N,Hq,d], k/v [B,N,Hkv,d] bf16; o like q; lse fp32 [B,Hq,N]."""
    _check_bf16(q, k, v, o)
    B, Hq, Hkv, N, d, G = _dims(q, k, G)
    scale = d ** -0.5 if scale is None else scale
    if flags or not _all_contiguous(q, k, v, o):
        # option flags, or views (e.g. of a packed qkv buffer): the general entry point
        shb = Hq // 2 if shift_head_begin is None else shift_head_begin
        sh = G // 2 if shift is None else shift
        strides = None if _all_contiguous(q, k, v, o) else _strides_array(q, k, v, o)
        _check(lib().s2attn_fwd_general(_ptr(q, True), _ptr(k, True), _ptr(v, True), _ptr(o, True),
                                        _ptr(lse), B, Hq, Hkv, N, d, G, scale, shb, sh,
                                        int(flags), strides, _stream(stream)),
               "s2attn_fwd_general")
        return
    if shift_head_begin is None and shift is None:
        _check(lib().s2attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                                G, scale, _stream(stream)), "s2attn_fwd")
        return
    shb = Hq // 2 if shift_head_begin is None else shift_head_begin
    sh = G // 2 if shift is None else shift
    _check(lib().s2attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                               G, scale, shb, sh, _stream(stream)), "s2attn_fwd_ex")


def s2attn_fwd_rope_q(q, k, v, o, lse, q_rot, G, scale=None, shift_head_begin=None, shift=None,
                      flags=0, base=10000.0, pi_scale=1.0, stream=None):
    """Forward with the RoPE-PI rotation of the queries fused in: q un-rotated, k already rotated
    (s2attn_rope_pi); also writes the rotated queries to q_rot (may be q itself)."""
    _check_bf16(q, k, v, o, q_rot)
    B, Hq, Hkv, N, d, G = _dims(q, k, G)
    scale = d ** -0.5 if scale is None else scale
    shb = Hq // 2 if shift_head_begin is None else shift_head_begin
    sh = G // 2 if shift is None else shift
    _check(lib().s2attn_fwd_rope_q(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(q_rot), B,
                                   Hq, Hkv, N, d, G, scale, shb, sh, int(flags), float(base),
                                   float(pi_scale), _stream(stream)), "s2attn_fwd_rope_q")


def s2attn_bwd_workspace_size(B, Hq, N) -> int:
    return int(lib().s2attn_bwd_workspace_size(B, Hq, N))


# Default cap on the workspace the allocating paths request for the dS hand-off.
DEFAULT_WORKSPACE_CAP = 8 << 30


def s2attn_bwd_workspace_size_ex(B, Hq, Hkv, N, d, G, shift_head_begin=None, shift=None,
                                 cap_bytes=0, flags=0) -> int:
    """Workspace for the backward without dQ recomputation (see include/s2attn.h)."""
    shb = Hq // 2 if shift_head_begin is None else shift_head_begin
    sh = G // 2 if shift is None else shift
    n = int(lib().s2attn_bwd_workspace_size_general(B, Hq, Hkv, N, d, G, shb, sh, int(flags),
                                                    int(cap_bytes)))
    if n == 0:
        raise S2AttnError(S2ATTN_ERR_INVALID_ARG, "s2attn_bwd_workspace_size_ex")
    return n


def s2attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, G, scale=None, shift_head_begin=None,
               shift=None, workspace=None, stream=None, flags=0):
    """dQ, dK, dV of S²-Attn (overwritten). workspace: a uint8 CUDA tensor, or None to let
    torch allocate s2attn_bwd_workspace_size_ex(..., DEFAULT_WORKSPACE_CAP) bytes."""
    _check_bf16(q, k, v, o, dO, dq, dk, dv)
    B, Hq, Hkv, N, d, G = _dims(q, k, G)
    scale = d ** -0.5 if scale is None else scale
    if workspace is None:
        ws_bytes = s2attn_bwd_workspace_size_ex(B, Hq, Hkv, N, d, G, shift_head_begin, shift,
                                                DEFAULT_WORKSPACE_CAP, flags)
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    if flags or not _all_contiguous(q, k, v, o, dO, dq, dk, dv):
        shb = Hq // 2 if shift_head_begin is None else shift_head_begin
        sh = G // 2 if shift is None else shift
        ts = (q, k, v, o, dO, dq, dk, dv)
        strides = None if _all_contiguous(*ts) else _strides_array(*ts)
        _check(lib().s2attn_bwd_general(
            _ptr(q, True), _ptr(k, True), _ptr(v, True), _ptr(o, True), _ptr(lse),
            _ptr(dO, True), _ptr(dq, True), _ptr(dk, True), _ptr(dv, True), B, Hq, Hkv, N, d, G,
            scale, shb, sh, int(flags), strides, _ptr(workspace), workspace.numel(),
            _stream(stream)), "s2attn_bwd_general")
        return
    if shift_head_begin is None and shift is None:
        _check(lib().s2attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO),
                                _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, G, scale,
                                _ptr(workspace), workspace.numel(), _stream(stream)),
               "s2attn_bwd")
        return
    shb = Hq // 2 if shift_head_begin is None else shift_head_begin
    sh = G // 2 if shift is None else shift
    _check(lib().s2attn_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO),
                               _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, G, scale, shb, sh,
                               _ptr(workspace), workspace.numel(), _stream(stream)),
           "s2attn_bwd_ex")


def s2attn_bwd_preprocess(o, lse, dO, workspace, stream=None):
    B, N, Hq, d = o.shape
    _check(lib().s2attn_bwd_preprocess(_ptr(o), _ptr(lse), _ptr(dO), B, Hq, N, d,
                                       _ptr(workspace), workspace.numel(), _stream(stream)),
           "s2attn_bwd_preprocess")


def s2attn_bwd_dkdv(q, k, v, dO, dk, dv, G, workspace, scale=None, shift_head_begin=None,
                    shift=None, stream=None):
    B, Hq, Hkv, N, d, G = _dims(q, k, G)
    scale = d ** -0.5 if scale is None else scale
    shb = Hq // 2 if shift_head_begin is None else shift_head_begin
    sh = G // 2 if shift is None else shift
    _check(lib().s2attn_bwd_dkdv(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dk), _ptr(dv), B, Hq,
                                 Hkv, N, d, G, scale, shb, sh, _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "s2attn_bwd_dkdv")


def s2attn_bwd_dq(q, k, v, dO, dq, G, workspace, scale=None, shift_head_begin=None, shift=None,
                  stream=None):
    B, Hq, Hkv, N, d, G = _dims(q, k, G)
    scale = d ** -0.5 if scale is None else scale
    shb = Hq // 2 if shift_head_begin is None else shift_head_begin
    sh = G // 2 if shift is None else shift
    _check(lib().s2attn_bwd_dq(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dq), B, Hq, Hkv, N, d,
                               G, scale, shb, sh, _ptr(workspace), workspace.numel(),
                               _stream(stream)), "s2attn_bwd_dq")


def s2attn_bwd_dkdv_ds(q, k, v, dO, dk, dv, G, workspace, scale=None, shift_head_begin=None,
                       shift=None, stream=None, flags=0, dq=None):
    """dK, dV and the dS tiles (first of the two dS hand-off stages). With option flags, or views
    with contiguous (H, d) blocks, the _general entry is used (`dq` then supplies dQ's strides;
    it is not written here)."""
    B, Hq, Hkv, N, d, G = _dims(q, k, G)
    scale = d ** -0.5 if scale is None else scale
    shb = Hq // 2 if shift_head_begin is None else shift_head_begin
    sh = G // 2 if shift is None else shift
    if flags or not _all_contiguous(q, k, v, dO, dk, dv, dq):
        ts = (q, k, v, dO, dO, dq if dq is not None else q, dk, dv)
        strides = None if _all_contiguous(*ts) else _strides_array(*ts)
        _check(lib().s2attn_bwd_dkdv_ds_general(
            _ptr(q, True), _ptr(k, True), _ptr(v, True), _ptr(dO, True), _ptr(dk, True),
            _ptr(dv, True), B, Hq, Hkv, N, d, G, scale, shb, sh, int(flags), strides,
            _ptr(workspace), workspace.numel(), _stream(stream)), "s2attn_bwd_dkdv_ds_general")
        return
    _check(lib().s2attn_bwd_dkdv_ds(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(dk), _ptr(dv), B,
                                    Hq, Hkv, N, d, G, scale, shb, sh, _ptr(workspace),
                                    workspace.numel(), _stream(stream)), "s2attn_bwd_dkdv_ds")


def s2attn_bwd_dq_ds(k, dq, G, workspace, scale=None, shift_head_begin=None, shift=None,
                     stream=None, flags=0):
    """dQ from the dS tiles (second of the two dS hand-off stages); flags or a strided k / dq
    go through the _general entry."""
    B, N, Hq, d = dq.shape
    Hkv = k.shape[2]
    scale = d ** -0.5 if scale is None else scale
    shb = Hq // 2 if shift_head_begin is None else shift_head_begin
    sh = G // 2 if shift is None else shift
    if flags or not _all_contiguous(k, dq):
        ts = (dq, k, k, dq, dq, dq, k, k)
        strides = None if _all_contiguous(k, dq) else _strides_array(*ts)
        _check(lib().s2attn_bwd_dq_ds_general(
            _ptr(k, True), _ptr(dq, True), B, Hq, Hkv, N, d, G, scale, shb, sh, int(flags),
            strides, _ptr(workspace), workspace.numel(), _stream(stream)),
            "s2attn_bwd_dq_ds_general")
        return
    _check(lib().s2attn_bwd_dq_ds(_ptr(k), _ptr(dq), B, Hq, Hkv, N, d, G, scale, shb, sh,
                                  _ptr(workspace), workspace.numel(), _stream(stream)),
           "s2attn_bwd_dq_ds")


def s2attn_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, G, scale=None, stream=None):
    """s2attn_bwd without a workspace argument: the library's own static scratch is used
    (for callers that cannot allocate; see include/s2attn.h for the size limit and the rule
    that calls must not overlap on the GPU)."""
    _check_bf16(q, k, v, o, dO, dq, dk, dv)
    B, Hq, Hkv, N, d, G = _dims(q, k, G)
    scale = d ** -0.5 if scale is None else scale
    _check(lib().s2attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO),
                                    _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, G, scale,
                                    _stream(stream)), "s2attn_bwd_noalloc")


def s2attn_get_device_error(stream=None):
    """(status, code): S2ATTN_ERR_TIMEOUT with a nonzero code if a kernel gave up a wait."""
    code = ctypes.c_uint(0)
    st = lib().s2attn_get_device_error(_stream(stream), ctypes.byref(code))
    return int(st), int(code.value)


def s2attn_set_wait_timeout_ns(ns: int):
    lib().s2attn_set_wait_timeout_ns(int(ns))


def s2attn_selftest_wait_timeout(timeout_ns: int, stream=None):
    _check(lib().s2attn_selftest_wait_timeout(int(timeout_ns), _stream(stream)),
           "s2attn_selftest_wait_timeout")


# ------------------------------------------------------------------------------------------
# Allocating conveniences (torch provides the memory; the library does the work).
# ------------------------------------------------------------------------------------------
def s2attn_rope_pi(x, y, base=10000.0, pi_scale=1.0, inverse=False, stream=None):
    """Rotary position embedding with Position Interpolation of x [B,N,H,d] bf16 into y (y may
    be x). Views with contiguous (H, d) blocks, e.g. q or k of a packed qkv, are accepted."""
    _check_bf16(x, y)
    B, N, H, d = x.shape
    if tuple(y.shape) != tuple(x.shape):
        raise ValueError("x and y must have the same shape")
    strides = None if _all_contiguous(x, y) else _strides_array(x, y)
    _check(lib().s2attn_rope_pi(_ptr(x, True), _ptr(y, True), B, N, H, d, float(base),
                                float(pi_scale), 1 if inverse else 0, strides, _stream(stream)),
           "s2attn_rope_pi")


def rope_pi(x, base=10000.0, pi_scale=1.0, inverse=False, stream=None, out=None):
    """Convenience form of s2attn_rope_pi: returns the rotated tensor (a new one unless `out`)."""
    y = torch.empty_like(x) if out is None else out
    s2attn_rope_pi(x, y, base, pi_scale, inverse, stream)
    return y


def fwd(q, k, v, G, scale=None, shift_head_begin=None, shift=None, stream=None, flags=0):
    o = torch.empty_like(q)
    lse = torch.empty((q.shape[0], q.shape[2], q.shape[1]), dtype=torch.float32, device=q.device)
    s2attn_fwd(q, k, v, o, lse, G, scale, shift_head_begin, shift, stream, flags)
    return o, lse


def bwd(q, k, v, o, lse, dO, G, scale=None, shift_head_begin=None, shift=None, stream=None,
        flags=0):
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    s2attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, G, scale, shift_head_begin, shift, None, stream,
               flags)
    return dq, dk, dv
