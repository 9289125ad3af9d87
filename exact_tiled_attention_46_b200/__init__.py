"""Exact tiled attention for B200 (sm_100a): thin Python binding of libfa46.so.

Every function here only checks and marshals arguments (device pointers, sizes
and the current CUDA stream) and calls the C ABI declared in include/fa.h; all
arithmetic runs in the library's CUDA kernels.  There is no CPU path: a call
without a CUDA tensor or without the built library raises.

    o, lse = fwd(q, k, v, causal=True)            # prefill forward
    dq, dk, dv = bwd(q, k, v, o, do, lse, causal=True)
    o, lse = decode(q, k_cache, v_cache, seqlens)  # split-KV decode
    o, lse = decode_append(q, k_new, v_new, k_cache, v_cache, seqlens)   # + KV append
    o, lse = decode_paged(q, k_pages, v_pages, page_table, seqlens)     # paged cache
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

__all__ = ["fwd", "bwd", "decode", "decode_combine", "device_status", "set_wait_limit_ns",
           "selftest_wait_timeout", "lib", "LIB_PATH", "FA_OK", "FA_ERR_INVALID_ARG",
           "FA_ERR_UNSUPPORTED", "FA_ERR_CUDA", "FA_ERR_TIMEOUT", "FaError",
           "bwd_workspace_size", "decode_workspace_size", "decode_chunk", "launch_guard", "decode_append",
           "decode_paged", "fwd_fp8", "attn_merge"]

# FA46_LIBRARY may name another build of the same library (the debug build,
# libfa46_debug.so); there is no fallback when it is missing.
LIB_PATH = os.environ.get("FA46_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa46.so")
FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = 0, 1, 2, 3, 4
FA_ERR_DEVICE_INDEX = 5
FA_BF16, FA_FP32 = 0, 1

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGNATURES = {
    "fa_abi_version": ([], _i),
    "fa_debug_build": ([], _i),
    "fa_status_string": ([_i], ctypes.c_char_p),
    "fa_fwd": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp], _i),
    "fa_fwd_ex": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp], _i),
    "fa_fwd_fp8": ([_vp, _vp, _vp, _f, _f, _f, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp], _i),
    "fa_bwd_workspace_size": ([_i, _i, _i, _i], _sz),
    "fa_bwd": ([_vp] * 9 + [_i] * 6 + [_f, _i, _i, _vp, _sz, _vp], _i),
    "fa_decode_chunk": ([], _i),
    "fa_decode_workspace_size": ([_i, _i, _i, _i], _sz),
    "fa_decode_splitkv": ([_vp] * 6 + [_i] * 5 + [_f, _i, _vp, _sz, _vp], _i),
    "fa_decode_combine": ([_vp] * 5 + [_i] * 5 + [_vp], _i),
    "fa_attn_merge": ([_vp] * 6 + [_i] * 5 + [_vp], _i),
    "fa_decode_append_splitkv": ([_vp] * 8 + [_i] * 5 + [_f, _i, _vp, _sz, _vp], _i),
    "fa_decode_paged_splitkv": ([_vp] * 9 + [_i] * 7 + [_f, _i, _vp, _sz, _vp], _i),
    "fa_decode_splitkv_static": ([_vp] * 6 + [_i] * 5 + [_f, _i, _vp], _i),
    "fa_device_status": ([ctypes.POINTER(_i), ctypes.POINTER(_i), _i, _vp], _i),
    "fa_set_wait_limit_ns": ([ctypes.c_ulonglong], None),
    "fa_selftest_wait_timeout": ([ctypes.c_ulonglong, _vp], _i),
    "fa_selftest_exp2_poly": ([_vp, _vp, _i, _vp], _i),
    "fa_launch_guard": ([_i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i)], _i),
}

_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().fa_status_string(status).decode()} (status {status})")


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library missing: {LIB_PATH} (run python -m exact_tiled_attention_46_b200.build)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def _check(status: int, what: str):
    if status != FA_OK:
        raise FaError(status, what)


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _need(t: torch.Tensor, name: str, dtype=torch.bfloat16, ndim: Optional[int] = None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def _odt(dtype) -> int:
    if dtype == torch.bfloat16:
        return FA_BF16
    if dtype == torch.float32:
        return FA_FP32
    raise TypeError("output dtype must be torch.bfloat16 or torch.float32")


def fwd(q, k, v, scale: Optional[float] = None, causal: bool = False, o_dtype=torch.bfloat16,
        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
    """Forward attention.  q [B,Lq,Hq,D], k/v [B,Lk,Hkv,D] bf16 -> (o, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, ndim=4)
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, _ = k.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Lq, Hq, D), dtype=o_dtype, device=q.device)
    _need(out, "out", dtype=None, ndim=4)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    _need(lse, "lse", dtype=torch.float32, ndim=3)
    _check(lib().fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                           B, Hq, Hkv, Lq, Lk, D, scale, int(bool(causal)), _odt(out.dtype), _stream(q)),
           "fa_fwd")
    return out, lse


def fwd_fp8(q, k, v, q_scale: float, k_scale: float, v_scale: float, scale: Optional[float] = None,
            causal: bool = False, o_dtype=torch.bfloat16, out: Optional[torch.Tensor] = None,
            lse: Optional[torch.Tensor] = None):
    """Forward attention on e4m3 inputs (torch.float8_e4m3fn, values = e4m3 * their scale) -> (o, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dtype=torch.float8_e4m3fn, ndim=4)
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, _ = k.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Lq, Hq, D), dtype=o_dtype, device=q.device)
    _need(out, "out", dtype=None, ndim=4)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    _need(lse, "lse", dtype=torch.float32, ndim=3)
    _check(lib().fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), float(q_scale), float(k_scale), float(v_scale),
                            out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lq, Lk, D, scale, int(bool(causal)),
                            _odt(out.dtype), _stream(q)),
           "fa_fwd_fp8")
    return out, lse


def bwd_workspace_size(B, Hq, Lq, D) -> int:
    return int(lib().fa_bwd_workspace_size(B, Hq, Lq, D))


def bwd(q, k, v, o, do, lse, scale: Optional[float] = None, causal: bool = False, grad_dtype=torch.bfloat16,
        workspace: Optional[torch.Tensor] = None):
    """Backward attention from the saved lse -> (dq, dk, dv)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _need(t, n, ndim=4)
    _need(lse, "lse", dtype=torch.float32, ndim=3)
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, _ = k.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq = torch.empty((B, Lq, Hq, D), dtype=grad_dtype, device=q.device)
    dk = torch.empty((B, Lk, Hkv, D), dtype=grad_dtype, device=q.device)
    dv = torch.empty((B, Lk, Hkv, D), dtype=grad_dtype, device=q.device)
    need = bwd_workspace_size(B, Hq, Lq, D)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(lib().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Lq, Lk, D, scale,
                        int(bool(causal)), _odt(grad_dtype), workspace.data_ptr(), workspace.numel(), _stream(q)),
           "fa_bwd")
    return dq, dk, dv


def decode_chunk() -> int:
    return int(lib().fa_decode_chunk())


def decode_workspace_size(B, Hq, Lmax, D) -> int:
    return int(lib().fa_decode_workspace_size(B, Hq, Lmax, D))


def decode(q, k_cache, v_cache, seqlens, scale: Optional[float] = None, o_dtype=torch.bfloat16,
           workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
           lse: Optional[torch.Tensor] = None):
    """Split-KV decode.  q [B,Hq,D], caches [B,Lmax,Hkv,D] bf16, seqlens int32 [B] -> (o, lse)."""
    _need(q, "q", ndim=3)
    _need(k_cache, "k_cache", ndim=4)
    _need(v_cache, "v_cache", ndim=4)
    _need(seqlens, "seqlens", dtype=torch.int32, ndim=1)
    B, Hq, D = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    need = decode_workspace_size(B, Hq, Lmax, D)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=o_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check(lib().fa_decode_splitkv(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), seqlens.data_ptr(),
                                   out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lmax, D, scale, _odt(out.dtype),
                                   workspace.data_ptr(), workspace.numel(), _stream(q)),
           "fa_decode_splitkv")
    return out, lse


def decode_append(q, k_new, v_new, k_cache, v_cache, seqlens, scale: Optional[float] = None,
                  o_dtype=torch.bfloat16, workspace: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
    """Decode with the new token appended: q [B,Hq,D], k_new/v_new [B,Hkv,D], caches [B,Lmax,Hkv,D].

    Attends over seqlens[b] cached rows plus the new row and writes the new rows
    into the caches at row seqlens[b]; ``seqlens`` is not advanced (add 1 after).
    """
    _need(q, "q", ndim=3)
    _need(k_new, "k_new", ndim=3)
    _need(v_new, "v_new", ndim=3)
    _need(k_cache, "k_cache", ndim=4)
    _need(v_cache, "v_cache", ndim=4)
    _need(seqlens, "seqlens", dtype=torch.int32, ndim=1)
    B, Hq, D = q.shape
    _, Lmax, Hkv, _ = k_cache.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    need = decode_workspace_size(B, Hq, Lmax + 1, D)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=o_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check(lib().fa_decode_append_splitkv(q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), k_cache.data_ptr(),
                                          v_cache.data_ptr(), seqlens.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                          B, Hq, Hkv, Lmax, D, scale, _odt(out.dtype), workspace.data_ptr(),
                                          workspace.numel(), _stream(q)),
           "fa_decode_append_splitkv")
    return out, lse


def decode_paged(q, k_pages, v_pages, page_table, seqlens, k_new=None, v_new=None, scale: Optional[float] = None,
                 o_dtype=torch.bfloat16, workspace: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
    """Decode from a paged cache: pages [num_pages,page_size,Hkv,D], page_table int32 [B,pages_per_seq].

    With k_new/v_new [B,Hkv,D] the new token is attended and appended at row
    seqlens[b] (its page must be in the table); ``seqlens`` is not advanced.
    """
    _need(q, "q", ndim=3)
    _need(k_pages, "k_pages", ndim=4)
    _need(v_pages, "v_pages", ndim=4)
    _need(page_table, "page_table", dtype=torch.int32, ndim=2)
    _need(seqlens, "seqlens", dtype=torch.int32, ndim=1)
    append = k_new is not None
    if append:
        _need(k_new, "k_new", ndim=3)
        _need(v_new, "v_new", ndim=3)
    B, Hq, D = q.shape
    num_pages, page_size, Hkv, _ = k_pages.shape
    pages_per_seq = page_table.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    need = decode_workspace_size(B, Hq, pages_per_seq * page_size + int(append), D)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=o_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _check(lib().fa_decode_paged_splitkv(q.data_ptr(), k_new.data_ptr() if append else None,
                                         v_new.data_ptr() if append else None, k_pages.data_ptr(),
                                         v_pages.data_ptr(), page_table.data_ptr(), seqlens.data_ptr(),
                                         out.data_ptr(), lse.data_ptr(), B, Hq, Hkv, num_pages, page_size,
                                         pages_per_seq, D, scale, _odt(out.dtype), workspace.data_ptr(),
                                         workspace.numel(), _stream(q)),
           "fa_decode_paged_splitkv")
    return out, lse


def decode_combine(o_part, lse_part, num_splits=None, o_dtype=torch.bfloat16):
    """Merge partial results: o_part [B,Hq,S,D], lse_part [B,Hq,S] fp32 -> (o [B,Hq,D], lse [B,Hq])."""
    _need(o_part, "o_part", dtype=torch.float32, ndim=4)
    _need(lse_part, "lse_part", dtype=torch.float32, ndim=3)
    B, Hq, S, D = o_part.shape
    ns_ptr = None
    if num_splits is not None:
        _need(num_splits, "num_splits", dtype=torch.int32, ndim=1)
        ns_ptr = num_splits.data_ptr()
    out = torch.empty((B, Hq, D), dtype=o_dtype, device=o_part.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=o_part.device)
    _check(lib().fa_decode_combine(o_part.data_ptr(), lse_part.data_ptr(), ns_ptr, out.data_ptr(), lse.data_ptr(),
                                   B, Hq, D, S, _odt(o_dtype), _stream(o_part)), "fa_decode_combine")
    return out, lse


def attn_merge(o_a, lse_a, o_b, lse_b, out=None, lse_out=None, o_dtype=torch.float32):
    """Merge two results over disjoint key sets: o_* [B,L,H,D] fp32, lse_* [B,H,L] -> (o, lse).

    ``out`` / ``lse_out`` may be ``o_a`` / ``lse_a`` (in-place accumulation).
    """
    _need(o_a, "o_a", dtype=torch.float32, ndim=4)
    _need(o_b, "o_b", dtype=torch.float32, ndim=4)
    _need(lse_a, "lse_a", dtype=torch.float32, ndim=3)
    _need(lse_b, "lse_b", dtype=torch.float32, ndim=3)
    B, L, H, D = o_a.shape
    if out is None:
        out = torch.empty((B, L, H, D), dtype=o_dtype, device=o_a.device)
    _need(out, "out", dtype=None, ndim=4)
    if lse_out is None:
        lse_out = torch.empty((B, H, L), dtype=torch.float32, device=o_a.device)
    _check(lib().fa_attn_merge(o_a.data_ptr(), lse_a.data_ptr(), o_b.data_ptr(), lse_b.data_ptr(), out.data_ptr(),
                               lse_out.data_ptr(), B, H, L, D, _odt(out.dtype), _stream(o_a)), "fa_attn_merge")
    return out, lse_out


def device_status(reset: bool = False, device=None):
    """(code, where) of the library's device status word (synchronises)."""
    code, where = ctypes.c_int(0), ctypes.c_int(0)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = torch.cuda.current_stream(dev).cuda_stream
    _check(lib().fa_device_status(ctypes.byref(code), ctypes.byref(where), int(reset), st), "fa_device_status")
    return code.value, where.value


def set_wait_limit_ns(ns: int):
    lib().fa_set_wait_limit_ns(int(ns))


def selftest_wait_timeout(wait_ns: int, device=None):
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _check(lib().fa_selftest_wait_timeout(int(wait_ns), torch.cuda.current_stream(dev).cuda_stream),
           "fa_selftest_wait_timeout")


def launch_guard(bwd: bool, D: int, causal: bool, query_regs: bool = True):
    """(compiled registers or None, registers the split assumes, cached check result) of one kernel instantiation."""
    regs, exp, state = ctypes.c_int(-1), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().fa_launch_guard(int(bool(bwd)), int(D), int(bool(causal)),
                                 ctypes.byref(regs) if query_regs else None, ctypes.byref(exp), ctypes.byref(state)),
           "fa_launch_guard")
    return (regs.value if query_regs else None), exp.value, state.value
