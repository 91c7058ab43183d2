"""ctypes binding of libfa.so (C ABI in include/fa.h) -- argument marshalling only.

Every function here checks that the tensors live on a CUDA device with the expected
dtype and contiguity, passes their device pointers and the current CUDA stream to the
library, and raises ``FAError`` with the library's status and message on failure.  No
attention arithmetic happens in Python; if ``libfa.so`` has not been built, every call
raises instead of falling back to anything else.
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# FA_LIBRARY selects another build of the library, e.g. the debug build libfa_debug.so
LIB_PATH = os.environ.get("FA_LIBRARY") or os.path.join(_HERE, "libfa.so")

FA_OK = 0
FA_ERR_INVALID = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_WORKSPACE = 3
FA_ERR_CUDA = 4
FA_ERR_TIMEOUT = 5
FA_ERR_DEVICE_ARG = 6
FA_ERR_DEBUG_CHECK = 7
FA_BF16 = 0
FA_F32 = 1

# Every symbol include/fa.h declares, with its ctypes signature.
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_fwd_ex": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "fa_fwd_window": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P]),
    "fa_fwd_bshd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _P]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _P]),
    "fa_decode_workspace_size": (_Z, [_I, _I, _I, _I]),
    "fa_decode": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "fa_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "fa_decode_paged": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "fa_decode_ex": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _Z, _P]),
    "fa_merge_lse": (_I, [_P, _P, _I, _I, _I, _P, _P, _I, _P]),
    "fa_decode_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "fa_decode_paged_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F,
                                 _P, _Z, _P]),
    "fa_get_error": (_I, [_P]),
    "fa_set_wait_limit_ns": (None, [ctypes.c_ulonglong]),
    "fa_fwd_selftest_timeout": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_decode_selftest_timeout": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "fa_build_flags": (_I, []),
    "fa_debug_selftest_bounds": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _P]),
    "fa_status_str": (ctypes.c_char_p, [_I]),
    "fa_last_error_message": (ctypes.c_char_p, []),
    "fa_version": (_I, []),
}

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{status_str(status)}: {message}")


def load(path: str = LIB_PATH):
    """Load libfa.so (once) and declare its signatures.  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise FAError(FA_ERR_UNSUPPORTED,
                          f"{path} is not built (run: python -m exact_io_aware_81_b200.build)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_str(status: int) -> str:
    try:
        return load().fa_status_str(int(status)).decode()
    except Exception:
        return str(status)


def _check(rc: int):
    if rc != FA_OK:
        raise FAError(rc, load().fa_last_error_message().decode())


def _stream_handle(stream, device=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream)


@contextlib.contextmanager
def _on_device(*tensors):
    """Run a library call on the device of its tensors (the C ABI launches on the current
    device); every tensor passed must be on that one device."""
    dev = tensors[0].device
    for t in tensors[1:]:
        if t is not None and t.device != dev:
            raise ValueError(f"all tensors must be on {dev}; found one on {t.device}")
    with torch.cuda.device(dev):
        yield dev


def _require(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {t.dim()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _output(t: Optional[torch.Tensor], name: str, dtype: torch.dtype, shape, device) -> torch.Tensor:
    """A caller-provided output checked against its dtype and exact shape, or a new one."""
    shape = tuple(shape)
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    _require(t, name, dtype, len(shape))
    if tuple(t.shape) != shape:
        raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
    return t


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
        scale: Optional[float] = None, out_dtype: torch.dtype = torch.bfloat16,
        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
        stream=None, window: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention forward: q (B,Hq,Nq,d), k/v (B,Hkv,Nk,d) bf16 -> (o, lse).

    scale defaults to 1/sqrt(d) (as flash_attn_func's softmax_scale=None does on the
    toolsku.com page).  causal uses bottom-right alignment (row i sees keys up to
    i + Nk - Nq).  window = W >= 1 (causal only) restricts row i to its W most recent
    keys (fa_fwd_window); 0 means no window.  o has out_dtype (bf16 or fp32); lse is
    fp32 (B,Hq,Nq), natural log.
    """
    _require(q, "q", torch.bfloat16, 4)
    _require(k, "k", torch.bfloat16, 4)
    _require(v, "v", torch.bfloat16, 4)
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, dk) != (B, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} k {tuple(k.shape)} v {tuple(v.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    out, lse = _fwd_outputs(q, (B, Hq, Nq, d), (B, Hq, Nq), out_dtype, out, lse)
    odt = FA_F32 if out_dtype == torch.float32 else FA_BF16
    if window:
        if not causal:
            raise ValueError("a sliding window needs causal=True")
        with _on_device(q, k, v, out, lse) as dev:
            rc = load().fa_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale), int(window),
                                      odt, _stream_handle(stream, dev))
    else:
        with _on_device(q, k, v, out, lse) as dev:
            rc = load().fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)),
                                  odt, _stream_handle(stream, dev))
    _check(rc)
    return out, lse


def _fwd_outputs(q, o_shape, lse_shape, out_dtype, out, lse):
    return (_output(out, "out", out_dtype, o_shape, q.device),
            _output(lse, "lse", torch.float32, lse_shape, q.device))


def fwd_bshd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
             scale: Optional[float] = None, out_dtype: torch.dtype = torch.bfloat16,
             out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
             stream=None, window: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention forward on (batch, sequence, heads, dim) tensors (fa_fwd_bshd), the layout
    flash_attn_func takes: q (B,Nq,Hq,d), k/v (B,Nk,Hkv,d) bf16 -> o (B,Nq,Hq,d) and lse
    fp32 (B,Hq,Nq).  causal, scale, window and out_dtype as fwd."""
    _require(q, "q", torch.bfloat16, 4)
    _require(k, "k", torch.bfloat16, 4)
    _require(v, "v", torch.bfloat16, 4)
    B, Nq, Hq, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    if (Bk, dk) != (B, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} k {tuple(k.shape)} v {tuple(v.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    if window and not causal:
        raise ValueError("a sliding window needs causal=True")
    out, lse = _fwd_outputs(q, (B, Nq, Hq, d), (B, Hq, Nq), out_dtype, out, lse)
    odt = FA_F32 if out_dtype == torch.float32 else FA_BF16
    with _on_device(q, k, v, out, lse) as dev:
        rc = load().fa_fwd_bshd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)), int(window), odt,
                                _stream_handle(stream, dev))
    _check(rc)
    return out, lse


def fwd_window(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, window: int,
               scale: Optional[float] = None, out_dtype: torch.dtype = torch.bfloat16,
               out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
               stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Sliding-window causal attention (fa_fwd_window): row i sees keys j with
    i + Nk - Nq - window < j <= i + Nk - Nq.  Arguments as fwd."""
    if int(window) < 1:
        raise ValueError("window must be >= 1")
    return fwd(q, k, v, causal=True, scale=scale, out_dtype=out_dtype, out=out, lse=lse,
               stream=stream, window=int(window))


def fwd_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_scale: torch.Tensor,
            k_scale: torch.Tensor, v_scale: torch.Tensor, causal: bool = False,
            scale: Optional[float] = None, out_dtype: torch.dtype = torch.bfloat16,
            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
            stream=None, window: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention forward over FP8 E4M3 inputs: q (B,Hq,Nq,d), k/v (B,Hkv,Nk,d) uint8 bytes
    with fp32 per-head scales q_scale (Hq), k_scale/v_scale (Hkv) -> (o, lse).  The value
    of a q row of head h is q_scale[h] * e4m3(bytes); likewise K and V.  ``scale`` defaults
    to 1/sqrt(d); d must be 128."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n, torch.uint8, 4)
    for t, n in ((q_scale, "q_scale"), (k_scale, "k_scale"), (v_scale, "v_scale")):
        _require(t, n, torch.float32, 1)
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if Bk != B or dk != d or tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, v {tuple(v.shape)}")
    if q_scale.numel() != Hq or k_scale.numel() != Hkv or v_scale.numel() != Hkv:
        raise ValueError("q_scale must have Hq entries, k_scale and v_scale Hkv entries")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    out, lse = _fwd_outputs(q, (B, Hq, Nq, d), (B, Hq, Nq), out_dtype, out, lse)
    odt = FA_F32 if out_dtype == torch.float32 else FA_BF16
    with _on_device(q, k, v, q_scale, k_scale, v_scale, out, lse) as dev:
        rc = load().fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), q_scale.data_ptr(),
                               k_scale.data_ptr(), v_scale.data_ptr(), out.data_ptr(), lse.data_ptr(),
                               B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)), int(window), odt,
                               _stream_handle(stream, dev))
    _check(rc)
    return out, lse


def decode_workspace_size(B: int, Hq: int, Nmax: int, d: int) -> int:
    return int(load().fa_decode_workspace_size(B, Hq, Nmax, d))


def decode(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor, seqlens: torch.Tensor,
           scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
           out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
           want_lse: bool = True, stream=None):
    """Decode step: q (B,Hq,d) against caches (B,Hkv,Nmax,d) up to seqlens[b] (int32, device).

    Returns (o (B,Hq,d) bf16, lse (B,Hq) fp32 or None).  ``workspace`` is a uint8 CUDA
    tensor of at least decode_workspace_size(...) bytes; one is allocated if omitted.
    """
    _require(q, "q", torch.bfloat16, 3)
    _require(kcache, "kcache", torch.bfloat16, 4)
    _require(vcache, "vcache", torch.bfloat16, 4)
    _require(seqlens, "seqlens", torch.int32, 1)
    B, Hq, d = q.shape
    Bk, Hkv, Nmax, dk = kcache.shape
    if (Bk, dk) != (B, d) or tuple(vcache.shape) != tuple(kcache.shape) or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, kcache, vcache and seqlens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = decode_workspace_size(B, Hq, Nmax, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    elif not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    out, lse = _decode_outputs(q, out, lse, want_lse)
    with _on_device(q, kcache, vcache, seqlens, out, lse, workspace) as dev:
        rc = load().fa_decode(q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(), seqlens.data_ptr(),
                              out.data_ptr(), lse.data_ptr() if lse is not None else None,
                              B, Hq, Hkv, Nmax, d, float(scale), workspace.data_ptr(),
                              workspace.numel() * workspace.element_size(), _stream_handle(stream, dev))
    _check(rc)
    return out, lse


def decode_paged(q: torch.Tensor, kpages: torch.Tensor, vpages: torch.Tensor,
                 block_table: torch.Tensor, seqlens: torch.Tensor, scale: Optional[float] = None,
                 workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, want_lse: bool = True, stream=None):
    """Decode over a paged cache (fa_decode_paged): q (B,Hq,d); kpages/vpages
    (num_pages,Hkv,page_size,d) bf16; block_table int32 (B,max_pages) and seqlens int32[B]
    on the device.  Token t of sequence b is row t % page_size of page
    block_table[b, t // page_size].  Returns (o, lse) as decode does."""
    _require(q, "q", torch.bfloat16, 3)
    _require(kpages, "kpages", torch.bfloat16, 4)
    _require(vpages, "vpages", torch.bfloat16, 4)
    _require(block_table, "block_table", torch.int32, 2)
    _require(seqlens, "seqlens", torch.int32, 1)
    B, Hq, d = q.shape
    num_pages, Hkv, page_size, dk = kpages.shape
    max_pages = block_table.shape[1]
    if (dk != d or tuple(vpages.shape) != tuple(kpages.shape) or seqlens.shape[0] != B
            or block_table.shape[0] != B):
        raise ValueError("shape mismatch between q, kpages, vpages, block_table and seqlens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = decode_workspace_size(B, Hq, page_size * max_pages, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    elif not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    out, lse = _decode_outputs(q, out, lse, want_lse)
    with _on_device(q, kpages, vpages, block_table, seqlens, out, lse, workspace) as dev:
        rc = load().fa_decode_paged(q.data_ptr(), kpages.data_ptr(), vpages.data_ptr(),
                                    block_table.data_ptr(), seqlens.data_ptr(), out.data_ptr(),
                                    lse.data_ptr() if lse is not None else None, B, Hq, Hkv,
                                    num_pages, page_size, max_pages, d, float(scale),
                                    workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    _stream_handle(stream, dev))
    _check(rc)
    return out, lse


def _decode_outputs(q, out, lse, want_lse, out_dtype=torch.bfloat16):
    B, Hq, d = q.shape
    out = _output(out, "out", out_dtype, (B, Hq, d), q.device)
    if lse is not None or want_lse:
        lse = _output(lse, "lse", torch.float32, (B, Hq), q.device)
    return out, lse


def _workspace(workspace, need, device):
    if workspace is None:
        return torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace


def decode_ex(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor, seqlens: torch.Tensor,
              scale: Optional[float] = None, out_dtype: torch.dtype = torch.bfloat16,
              workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
              lse: Optional[torch.Tensor] = None, want_lse: bool = True, stream=None):
    """fa_decode_ex: decode with a bf16 or fp32 output (fp32 keeps a partial result exact
    enough to merge again with merge_lse)."""
    _require(q, "q", torch.bfloat16, 3)
    _require(kcache, "kcache", torch.bfloat16, 4)
    _require(vcache, "vcache", torch.bfloat16, 4)
    _require(seqlens, "seqlens", torch.int32, 1)
    B, Hq, d = q.shape
    Bk, Hkv, Nmax, dk = kcache.shape
    if (Bk, dk) != (B, d) or tuple(vcache.shape) != tuple(kcache.shape) or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, kcache, vcache and seqlens")
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    workspace = _workspace(workspace, decode_workspace_size(B, Hq, Nmax, d), q.device)
    out, lse = _decode_outputs(q, out, lse, want_lse, out_dtype)
    with _on_device(q, kcache, vcache, seqlens, out, lse, workspace) as dev:
        rc = load().fa_decode_ex(q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(), seqlens.data_ptr(),
                                 out.data_ptr(), lse.data_ptr() if lse is not None else None,
                                 B, Hq, Hkv, Nmax, d, float(scale),
                                 FA_F32 if out_dtype == torch.float32 else FA_BF16, workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), _stream_handle(stream, dev))
    _check(rc)
    return out, lse


def merge_lse(o_parts: torch.Tensor, lse_parts: torch.Tensor, out_dtype: torch.dtype = torch.bfloat16,
              out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, stream=None):
    """fa_merge_lse: o_parts (P, *rows, d) fp32 and lse_parts (P, *rows) fp32 (natural log,
    -inf = no keys) -> (o (*rows, d), lse (*rows))."""
    _require(o_parts, "o_parts", torch.float32, o_parts.dim())
    _require(lse_parts, "lse_parts", torch.float32, lse_parts.dim())
    if o_parts.dim() < 3 or tuple(o_parts.shape[:-1]) != tuple(lse_parts.shape):
        raise ValueError("o_parts must be (P, *rows, d) and lse_parts (P, *rows)")
    P, d = o_parts.shape[0], o_parts.shape[-1]
    row_shape = tuple(o_parts.shape[1:-1])
    rows = 1
    for x in row_shape:
        rows *= x
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    out = _output(out, "out", out_dtype, row_shape + (d,), o_parts.device)
    lse = _output(lse, "lse", torch.float32, row_shape, o_parts.device)
    with _on_device(o_parts, lse_parts, out, lse) as dev:
        rc = load().fa_merge_lse(o_parts.data_ptr(), lse_parts.data_ptr(), P, rows, d, out.data_ptr(),
                                 lse.data_ptr(), FA_F32 if out_dtype == torch.float32 else FA_BF16,
                                 _stream_handle(stream, dev))
    _check(rc)
    return out, lse


def decode_fp8(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor, k_scale: torch.Tensor,
               v_scale: torch.Tensor, seqlens: torch.Tensor, scale: Optional[float] = None,
               workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
               lse: Optional[torch.Tensor] = None, want_lse: bool = True, stream=None):
    """Decode over an FP8 E4M3 cache (fa_decode_fp8): kcache/vcache uint8 (B,Hkv,Nmax,d)
    holding E4M3 bytes; k_scale/v_scale float32 (Hkv,) per-head dequantization scales."""
    _require(q, "q", torch.bfloat16, 3)
    _require(kcache, "kcache", torch.uint8, 4)
    _require(vcache, "vcache", torch.uint8, 4)
    _require(k_scale, "k_scale", torch.float32, 1)
    _require(v_scale, "v_scale", torch.float32, 1)
    _require(seqlens, "seqlens", torch.int32, 1)
    B, Hq, d = q.shape
    Bk, Hkv, Nmax, dk = kcache.shape
    if ((Bk, dk) != (B, d) or tuple(vcache.shape) != tuple(kcache.shape) or seqlens.shape[0] != B
            or k_scale.shape[0] != Hkv or v_scale.shape[0] != Hkv):
        raise ValueError("shape mismatch between q, the caches, the scales and seqlens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    workspace = _workspace(workspace, decode_workspace_size(B, Hq, Nmax, d), q.device)
    out, lse = _decode_outputs(q, out, lse, want_lse)
    with _on_device(q, kcache, vcache, k_scale, v_scale, seqlens, out, lse, workspace) as dev:
        rc = load().fa_decode_fp8(q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(), k_scale.data_ptr(),
                                  v_scale.data_ptr(), seqlens.data_ptr(), out.data_ptr(),
                                  lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Nmax, d,
                                  float(scale), workspace.data_ptr(),
                                  workspace.numel() * workspace.element_size(), _stream_handle(stream, dev))
    _check(rc)
    return out, lse


def decode_paged_fp8(q: torch.Tensor, kpages: torch.Tensor, vpages: torch.Tensor,
                     k_scale: torch.Tensor, v_scale: torch.Tensor, block_table: torch.Tensor,
                     seqlens: torch.Tensor, scale: Optional[float] = None,
                     workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, want_lse: bool = True, stream=None):
    """FP8 decode over a paged cache (fa_decode_paged_fp8): pools uint8
    (num_pages,Hkv,page_size,d) of E4M3 bytes, per-head scales, block table as decode_paged."""
    _require(q, "q", torch.bfloat16, 3)
    _require(kpages, "kpages", torch.uint8, 4)
    _require(vpages, "vpages", torch.uint8, 4)
    _require(k_scale, "k_scale", torch.float32, 1)
    _require(v_scale, "v_scale", torch.float32, 1)
    _require(block_table, "block_table", torch.int32, 2)
    _require(seqlens, "seqlens", torch.int32, 1)
    B, Hq, d = q.shape
    num_pages, Hkv, page_size, dk = kpages.shape
    max_pages = block_table.shape[1]
    if (dk != d or tuple(vpages.shape) != tuple(kpages.shape) or seqlens.shape[0] != B
            or block_table.shape[0] != B or k_scale.shape[0] != Hkv or v_scale.shape[0] != Hkv):
        raise ValueError("shape mismatch between q, the pools, the scales, block_table and seqlens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    workspace = _workspace(workspace, decode_workspace_size(B, Hq, page_size * max_pages, d), q.device)
    out, lse = _decode_outputs(q, out, lse, want_lse)
    with _on_device(q, kpages, vpages, k_scale, v_scale, block_table, seqlens, out, lse, workspace) as dev:
        rc = load().fa_decode_paged_fp8(q.data_ptr(), kpages.data_ptr(), vpages.data_ptr(),
                                        k_scale.data_ptr(), v_scale.data_ptr(), block_table.data_ptr(),
                                        seqlens.data_ptr(), out.data_ptr(),
                                        lse.data_ptr() if lse is not None else None, B, Hq, Hkv,
                                        num_pages, page_size, max_pages, d, float(scale),
                                        workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                        _stream_handle(stream, dev))
    _check(rc)
    return out, lse


def get_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device-side status."""
    return int(load().fa_get_error(_stream_handle(stream)))


def set_wait_limit_ns(ns: int):
    load().fa_set_wait_limit_ns(int(ns))


def fwd_selftest_timeout(q, k, v, causal=False, scale=None, stream=None):
    """Run the prefill kernel with its score-ready signal withheld (time-limit self-test)."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    with _on_device(q, k, v, out, lse) as dev:
        rc = load().fa_fwd_selftest_timeout(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                            lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale),
                                            int(bool(causal)), _stream_handle(stream, dev))
    _check(rc)
    return out, lse


def decode_selftest_timeout(q, kcache, vcache, seqlens, k_scale=None, v_scale=None, scale=None, stream=None):
    """Run a decode (bf16 caches, or E4M3 caches when both scales are given) with the split
    kernel's first copy withheld in every CTA (time-limit self-test)."""
    B, Hq, d = q.shape
    Hkv, Nmax = kcache.shape[1], kcache.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    ws = torch.empty(decode_workspace_size(B, Hq, Nmax, d), dtype=torch.uint8, device=q.device)
    with _on_device(q, kcache, vcache, seqlens, out, lse, ws, k_scale, v_scale) as dev:
        rc = load().fa_decode_selftest_timeout(
            q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(),
            k_scale.data_ptr() if k_scale is not None else None,
            v_scale.data_ptr() if v_scale is not None else None, seqlens.data_ptr(), out.data_ptr(),
            lse.data_ptr(), B, Hq, Hkv, Nmax, d, float(scale), ws.data_ptr(), ws.numel(),
            _stream_handle(stream, dev))
    _check(rc)
    return out, lse


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def decode_noalloc(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor,
                   seqlens: torch.Tensor, scale: Optional[float] = None,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   stream=None):
    """Decode step through fa_decode_noalloc: same result as ``decode`` but the library
    uses its own fixed 32 MiB scratch instead of a workspace, for callers that cannot
    allocate device memory.  ``out`` and ``lse`` must then be passed in by the caller;
    calls that overlap on the GPU share the scratch and must be ordered."""
    _require(q, "q", torch.bfloat16, 3)
    _require(kcache, "kcache", torch.bfloat16, 4)
    _require(vcache, "vcache", torch.bfloat16, 4)
    _require(seqlens, "seqlens", torch.int32, 1)
    B, Hq, d = q.shape
    Bk, Hkv, Nmax, dk = kcache.shape
    if (Bk, dk) != (B, d) or tuple(vcache.shape) != tuple(kcache.shape) or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, kcache, vcache and seqlens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        raise ValueError("decode_noalloc writes into a caller-provided `out`")
    out, lse = _decode_outputs(q, out, lse, False)
    with _on_device(q, kcache, vcache, seqlens, out, lse) as dev:
        rc = load().fa_decode_noalloc(q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(),
                                      seqlens.data_ptr(), out.data_ptr(),
                                      lse.data_ptr() if lse is not None else None,
                                      B, Hq, Hkv, Nmax, d, float(scale), _stream_handle(stream, dev))
    _check(rc)
    return out, lse
