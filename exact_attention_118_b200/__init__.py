"""Python binding of libfa.so: exact, IO-aware fused attention for B200 (sm_100a).

The functions ``fa_fwd``, ``fa_bwd``, ``fa_bwd_workspace_size``,
``fa_get_device_error``, ``fa_set_bwd_main_events``, ``fa_last_cuda_error``,
``fa_selftest_wait_timeout``, ``fa_strerror`` and ``fa_version`` have the names and
arguments of the C ABI in ``include/fa.h`` (pointers and the stream are plain
integers) and only marshal arguments. ``attention_forward`` and
``attention_backward`` are conveniences that take torch CUDA tensors, allocate
the outputs with torch (device memory and streams are all torch supplies) and
call the C ABI on the current stream. Every step of the computation runs in the
library's CUDA kernels; there is no other path. If the library is missing the
import of this package raises.
"""

from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "fa.h")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(5)
FA_BF16, FA_F32 = 0, 1
FA_DEVERR_TIMEOUT, FA_DEVERR_SMEM_ALIGN, FA_DEVERR_SEQLENS = 1, 2, 4
FA_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

_SIGNATURES = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I, _P]),
    "fa_bwd_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_gqa_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _F, _F, _F, _I, _I, _I, _P]),
    "fa_fwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _P]),
    "fa_bwd_varlen_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "fa_bwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, _I, _I, _F,
                           _I, _I, _P]),
    "fa_fwd_window": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _I, _P]),
    "fa_bwd_window": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, _I, _F, _I, _I,
                           _P]),
    "fa_fwd_gqa": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "fa_bwd_gqa": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "fa_get_device_error": (_I, [_P]),
    "fa_decode_device_error": (_I, [ctypes.c_uint]),
    "fa_set_bwd_main_events": (_I, [_P, _P]),
    "fa_last_cuda_error": (_I, []),
    "fa_selftest_wait_timeout": (_I, [_P]),
    "fa_selftest_exp2_fma": (_I, [_P, _P, ctypes.c_longlong, _P]),
    "fa_strerror": (ctypes.c_char_p, [_I]),
    "fa_version": (_I, []),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python exact_attention_118_b200/build.py` "
            "(nvcc, sm_100a). There is no fallback path."
        )
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def header_symbols():
    """Names of the functions declared in include/fa.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:fa_status|size_t|const char\*|int)\s+(fa_\w+)\(", text, re.M)))


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        extra = f", cuda error {fa_last_cuda_error()}" if status == FA_ERR_CUDA else ""
        super().__init__(f"{what}: {fa_strerror(status)} (status {status}{extra})")
        self.status = status


# ----------------------------------------------------------- C ABI, same names

def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, o_dtype, stream) -> int:
    return _lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, o_dtype, stream)


def fa_bwd_workspace_size(B, H, N, d) -> int:
    return _lib.fa_bwd_workspace_size(B, H, N, d)


def fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, B, H, N, d, scale, causal, stream) -> int:
    return _lib.fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, B, H, N, d, scale, causal, stream)


def fa_bwd_gqa_workspace_size(B, H, Hkv, N, d) -> int:
    return _lib.fa_bwd_gqa_workspace_size(B, H, Hkv, N, d)


def fa_fwd_fp8(q8, k8, v8, o, lse, B, H, Hkv, N, d, scale, q_scale, k_scale, v_scale, window_left, window_right,
               o_dtype, stream) -> int:
    return _lib.fa_fwd_fp8(q8, k8, v8, o, lse, B, H, Hkv, N, d, scale, q_scale, k_scale, v_scale, window_left,
                           window_right, o_dtype, stream)


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, B, max_seqlen, T, H, Hkv, d, scale, window_left, window_right,
                  o_dtype, stream) -> int:
    return _lib.fa_fwd_varlen(q, k, v, o, lse, cu_seqlens, B, max_seqlen, T, H, Hkv, d, scale, window_left,
                              window_right, o_dtype, stream)


def fa_bwd_varlen_workspace_size(B, T, H, Hkv, d) -> int:
    return _lib.fa_bwd_varlen_workspace_size(B, T, H, Hkv, d)


def fa_bwd_varlen(q, k, v, o, lse, dO, dq, dk, dv, cu_seqlens, workspace, ws_bytes, B, max_seqlen, T, H, Hkv, d,
                  scale, window_left, window_right, stream) -> int:
    return _lib.fa_bwd_varlen(q, k, v, o, lse, dO, dq, dk, dv, cu_seqlens, workspace, ws_bytes, B, max_seqlen, T,
                              H, Hkv, d, scale, window_left, window_right, stream)


def fa_fwd_window(q, k, v, o, lse, B, H, Hkv, N, d, scale, window_left, window_right, o_dtype, stream) -> int:
    return _lib.fa_fwd_window(q, k, v, o, lse, B, H, Hkv, N, d, scale, window_left, window_right, o_dtype, stream)


def fa_bwd_window(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, B, H, Hkv, N, d, scale, window_left,
                  window_right, stream) -> int:
    return _lib.fa_bwd_window(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, B, H, Hkv, N, d, scale,
                              window_left, window_right, stream)


def fa_fwd_gqa(q, k, v, o, lse, B, H, Hkv, N, d, scale, causal, o_dtype, stream) -> int:
    return _lib.fa_fwd_gqa(q, k, v, o, lse, B, H, Hkv, N, d, scale, causal, o_dtype, stream)


def fa_bwd_gqa(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, B, H, Hkv, N, d, scale, causal, stream) -> int:
    return _lib.fa_bwd_gqa(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, B, H, Hkv, N, d, scale, causal,
                           stream)


def fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, stream) -> int:
    """fa_bwd with its scratch in a fixed device array inside the library; for
    callers that may not allocate device memory (see include/fa.h)."""
    return _lib.fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, stream)


def fa_get_device_error(stream) -> int:
    return _lib.fa_get_device_error(stream)


def fa_decode_device_error(word) -> int:
    return _lib.fa_decode_device_error(word)


def fa_set_bwd_main_events(before, after) -> int:
    return _lib.fa_set_bwd_main_events(before, after)


def fa_last_cuda_error() -> int:
    return _lib.fa_last_cuda_error()


def fa_selftest_wait_timeout(stream) -> int:
    return _lib.fa_selftest_wait_timeout(stream)


def fa_selftest_exp2_fma(x, y, n, stream) -> int:
    return _lib.fa_selftest_exp2_fma(x, y, n, stream)


def fa_strerror(status: int) -> str:
    return _lib.fa_strerror(status).decode()


def fa_version() -> int:
    return _lib.fa_version()


# ------------------------------------------------------ torch conveniences

def _check(status: int, what: str):
    if status != FA_OK:
        raise FAError(status, what)


def _stream_ptr(torch, device):
    return torch.cuda.current_stream(device).cuda_stream


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def _window(causal, window):
    if window is None:
        return -1, (0 if causal else -1)
    wl, wr = (int(x) for x in window)
    if causal:
        wr = 0
    return wl, wr


def attention_forward(q, k, v, scale=None, causal=False, out_fp32=False, out=None, lse=None, window=None):
    """O, lse = attention(q, k, v) on the GPU. q: contiguous bf16 CUDA tensor
    [B, H, N, d]; k, v: [B, Hkv, N, d] with H % Hkv == 0 (Hkv = H for
    multi-head attention). window: None or (wl, wr), key j visible to query i
    iff i - wl <= j <= i + wr (negative: unbounded), intersected with the
    causal mask when causal is set. Returns (O [B,H,N,d] bf16 or fp32, lse
    [B,H,N] fp32)."""
    import torch

    B, H, N, d = _shape(q)
    Hkv = int(k.shape[1]) if k.dim() == 4 else -1
    if scale is None:
        scale = d ** -0.5
    for t, heads in ((q, H), (k, Hkv), (v, Hkv)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, heads, N, d):
            raise ValueError("q [B,H,N,d] and k, v [B,Hkv,N,d] must be contiguous bf16 CUDA tensors")
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    wl, wr = _window(causal, window)
    st = fa_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, Hkv, N, d,
                       float(scale), wl, wr, FA_F32 if out.dtype == torch.float32 else FA_BF16,
                       _stream_ptr(torch, q.device))
    _check(st, "fa_fwd")
    return out, lse


def attention_backward(q, k, v, o, lse, do, scale=None, causal=False, workspace=None, window=None):
    """dQ [B,H,N,d], dK and dV [B,Hkv,N,d] of attention on the GPU, all bf16
    (masks as in attention_forward)."""
    import torch

    B, H, N, d = _shape(q)
    Hkv = int(k.shape[1]) if k.dim() == 4 else -1
    if scale is None:
        scale = d ** -0.5
    for t, shape in ((q, (B, H, N, d)), (k, (B, Hkv, N, d)), (v, (B, Hkv, N, d)), (o, (B, H, N, d)),
                     (do, (B, H, N, d))):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shape:
            raise ValueError("q, o, dO [B,H,N,d] and k, v [B,Hkv,N,d] must be contiguous bf16 CUDA tensors")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, H, N):
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, N]")
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    ws_bytes = fa_bwd_gqa_workspace_size(B, H, Hkv, N, d)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    wl, wr = _window(causal, window)
    st = fa_bwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                       dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                       B, H, Hkv, N, d, float(scale), wl, wr, _stream_ptr(torch, q.device))
    _check(st, "fa_bwd")
    return dq, dk, dv


def attention_forward_varlen(q, k, v, cu_seqlens, max_seqlen, scale=None, causal=False, window=None,
                             out_fp32=False):
    """Packed variable-length attention. q [T, H, d], k, v [T, Hkv, d] bf16
    CUDA tensors; cu_seqlens int32 CUDA tensor [B + 1]. Returns (O [T, H, d],
    lse [H, T] fp32)."""
    import torch

    if q.dim() != 3 or k.dim() != 3 or v.dim() != 3:
        raise ValueError("expected packed [T, heads, d] tensors")
    T, H, d = (int(x) for x in q.shape)
    Hkv = int(k.shape[1])
    for t, heads in ((q, H), (k, Hkv), (v, Hkv)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (T, heads, d):
            raise ValueError("q [T,H,d] and k, v [T,Hkv,d] must be contiguous bf16 CUDA tensors")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be an int32 CUDA tensor [B + 1]")
    B = int(cu_seqlens.numel()) - 1
    if scale is None:
        scale = d ** -0.5
    out = torch.empty((T, H, d), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=q.device)
    lse = torch.empty((H, T), dtype=torch.float32, device=q.device)
    wl, wr = _window(causal, window)
    st = fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                       cu_seqlens.data_ptr(), B, int(max_seqlen), T, H, Hkv, d, float(scale), wl, wr,
                       FA_F32 if out_fp32 else FA_BF16, _stream_ptr(torch, q.device))
    _check(st, "fa_fwd_varlen")
    return out, lse


def attention_backward_varlen(q, k, v, o, lse, do, cu_seqlens, max_seqlen, scale=None, causal=False, window=None,
                              workspace=None):
    """dQ [T, H, d], dK and dV [T, Hkv, d] of packed variable-length attention."""
    import torch

    T, H, d = (int(x) for x in q.shape)
    Hkv = int(k.shape[1])
    for t, shape in ((q, (T, H, d)), (k, (T, Hkv, d)), (v, (T, Hkv, d)), (o, (T, H, d)), (do, (T, H, d))):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shape:
            raise ValueError("q, o, dO [T,H,d] and k, v [T,Hkv,d] must be contiguous bf16 CUDA tensors")
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (H, T):
        raise ValueError("lse must be a contiguous fp32 tensor [H, T]")
    B = int(cu_seqlens.numel()) - 1
    if scale is None:
        scale = d ** -0.5
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = fa_bwd_varlen_workspace_size(B, T, H, Hkv, d)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    wl, wr = _window(causal, window)
    st = fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                       dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), cu_seqlens.data_ptr(), workspace.data_ptr(),
                       workspace.numel(), B, int(max_seqlen), T, H, Hkv, d, float(scale), wl, wr,
                       _stream_ptr(torch, q.device))
    _check(st, "fa_bwd_varlen")
    return dq, dk, dv


def check_device_error(stream=None):
    """Synchronise and raise FAError if a bounded device wait gave up."""
    import torch

    ptr = _stream_ptr(torch, None) if stream is None else stream
    _check(fa_get_device_error(ptr), "device")
