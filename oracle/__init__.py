"""CPU oracle for exact attention -- TEST INFRASTRUCTURE, not part of the library.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  It shares no code with the CUDA path (``exact_io_aware_81_b200``)
and never imports it; the two meet only through the seeded inputs.

Contents:
  * ``attn_fwd`` / ``attn_fwd_fp8`` / ``decode`` / ``decode_paged`` / ``decode_fp8`` /
    ``probs``: the fp64
    two-pass definition, in plain C with OpenMP (``attn_oracle.c``), called through
    ctypes; ``e4m3_to_double`` decodes one FP8 E4M3 byte.
  * ``online.online_attention``: a restatement of the block-by-block online softmax
    (youngju.dev "attention variants", section 3), used only to check that the online
    and two-pass forms agree.
  * ``split_kv.split_kv_decode``: split-KV partials combined by a log-sum-exp merge,
    used only to check that any chunking gives the unsplit result.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c with gcc -O2 -fopenmp into oracle/_build/liboracle.so."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def declare(lib):
    """Set the ctypes signatures of the oracle's C entry points on a loaded library."""
    P = ctypes.c_void_p
    I = ctypes.c_int
    D = ctypes.c_double
    lib.oracle_attn_fwd.argtypes = [P, P, P, I, I, I, I, I, I, D, I, P, I, P, P]
    lib.oracle_attn_fwd_window.argtypes = [P, P, P, I, I, I, I, I, I, D, I, I, P, I, P, P]
    lib.oracle_attn_probs.argtypes = [P, P, I, I, I, I, I, I, D, I, P]
    lib.oracle_attn_probs_window.argtypes = [P, P, I, I, I, I, I, I, D, I, I, P]
    lib.oracle_decode.argtypes = [P, P, P, P, I, I, I, I, I, D, P, P]
    lib.oracle_decode_paged.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, D, P, P]
    lib.oracle_decode_fp8.argtypes = [P, P, P, P, P, P, I, I, I, I, I, D, P, P]
    lib.oracle_attn_fwd_fp8.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, D, I, I, P, I, P, P]
    lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_double.restype = D
    lib.oracle_num_threads.argtypes = []
    for f in (lib.oracle_attn_fwd, lib.oracle_attn_fwd_window, lib.oracle_attn_probs,
              lib.oracle_attn_probs_window, lib.oracle_decode, lib.oracle_decode_paged,
              lib.oracle_decode_fp8, lib.oracle_attn_fwd_fp8, lib.oracle_num_threads):
        f.restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = declare(ctypes.CDLL(build()))
    return _lib


def _bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.bfloat16, t.dtype
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy()).view(np.uint16)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float, causal: bool,
             rows: Optional[torch.Tensor] = None, window: int = 0):
    """fp64 attention of bf16 q (B,Hq,Nq,d), k/v (B,Hkv,Nk,d).

    ``window`` = W >= 1 restricts causal row i to its W most recent keys
    (i + Nk - Nq - W < j <= i + Nk - Nq); 0 means no window.
    Returns (o, lse) as float64 torch tensors of shape (B,Hq,R,d) and (B,Hq,R), where R
    is len(rows) if a row sample is given, else Nq.
    """
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    if rows is not None:
        rw = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        nr = int(rw.shape[0])
        rp = _ptr(rw)
    else:
        rw, nr, rp = None, Nq, None
    o = np.empty((B, Hq, nr, d), dtype=np.float64)
    lse = np.empty((B, Hq, nr), dtype=np.float64)
    lib = _load()
    if window:
        rc = lib.oracle_attn_fwd_window(_ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Nq, Nk, d,
                                        float(scale), int(bool(causal)), int(window), rp, nr,
                                        _ptr(o), _ptr(lse))
    else:
        rc = lib.oracle_attn_fwd(_ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Nq, Nk, d,
                                 float(scale), int(bool(causal)), rp, nr, _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_fwd rejected its arguments")
    return torch.from_numpy(o), torch.from_numpy(lse)


def probs(q: torch.Tensor, k: torch.Tensor, scale: float, causal: bool,
          window: int = 0) -> torch.Tensor:
    """Softmax weights P (B,Hq,Nq,Nk) in fp64, for tiny problems (window as in attn_fwd)."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    qb, kb = _bits(q), _bits(k)
    p = np.empty((B, Hq, Nq, Nk), dtype=np.float64)
    lib = _load()
    if window:
        rc = lib.oracle_attn_probs_window(_ptr(qb), _ptr(kb), B, Hq, Hkv, Nq, Nk, d,
                                          float(scale), int(bool(causal)), int(window), _ptr(p))
    else:
        rc = lib.oracle_attn_probs(_ptr(qb), _ptr(kb), B, Hq, Hkv, Nq, Nk, d, float(scale),
                                   int(bool(causal)), _ptr(p))
    if rc != 0:
        raise ValueError("oracle_attn_probs rejected its arguments")
    return torch.from_numpy(p)


def decode(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor, seqlens: torch.Tensor,
           scale: float):
    """fp64 decode: q (B,Hq,d) against caches (B,Hkv,Nmax,d) up to seqlens[b]."""
    B, Hq, d = q.shape
    Hkv, Nmax = kcache.shape[1], kcache.shape[2]
    qb, kb, vb = _bits(q), _bits(kcache), _bits(vcache)
    sl = np.ascontiguousarray(seqlens.detach().cpu().numpy().astype(np.int32))
    o = np.empty((B, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    rc = _load().oracle_decode(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(sl), B, Hq, Hkv, Nmax, d,
                               float(scale), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return torch.from_numpy(o), torch.from_numpy(lse)


def decode_paged(q: torch.Tensor, kpages: torch.Tensor, vpages: torch.Tensor,
                 block_table: torch.Tensor, seqlens: torch.Tensor, scale: float):
    """fp64 decode over a paged cache: q (B,Hq,d); kpages/vpages (num_pages,Hkv,page_size,d);
    block_table int32 (B,max_pages); token t of sequence b is row t % page_size of page
    block_table[b, t // page_size]."""
    B, Hq, d = q.shape
    num_pages, Hkv, page_size = kpages.shape[0], kpages.shape[1], kpages.shape[2]
    max_pages = block_table.shape[1]
    qb, kb, vb = _bits(q), _bits(kpages), _bits(vpages)
    bt = np.ascontiguousarray(block_table.detach().cpu().numpy().astype(np.int32))
    sl = np.ascontiguousarray(seqlens.detach().cpu().numpy().astype(np.int32))
    o = np.empty((B, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    rc = _load().oracle_decode_paged(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), _ptr(sl), B, Hq, Hkv,
                                     num_pages, page_size, max_pages, d, float(scale),
                                     _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode_paged rejected its arguments")
    return torch.from_numpy(o), torch.from_numpy(lse)


def e4m3_to_double(x: int) -> float:
    """Value of one FP8 E4M3 byte (OCP "e4m3fn": bias 7, no infinities, S.1111.111 = NaN)."""
    return float(_load().oracle_e4m3_to_double(int(x) & 0xFF))


def decode_fp8(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor,
               k_scale: torch.Tensor, v_scale: torch.Tensor, seqlens: torch.Tensor, scale: float):
    """fp64 decode over an FP8 E4M3 cache: kcache/vcache uint8 (B,Hkv,Nmax,d) holding E4M3
    bytes; key j of head g is k_scale[g] * e4m3(byte) (likewise V with v_scale)."""
    B, Hq, d = q.shape
    Hkv, Nmax = kcache.shape[1], kcache.shape[2]
    assert kcache.dtype == torch.uint8 and vcache.dtype == torch.uint8
    qb = _bits(q)
    kb = np.ascontiguousarray(kcache.detach().cpu().numpy())
    vb = np.ascontiguousarray(vcache.detach().cpu().numpy())
    ks = np.ascontiguousarray(k_scale.detach().cpu().numpy().astype(np.float32))
    vs = np.ascontiguousarray(v_scale.detach().cpu().numpy().astype(np.float32))
    sl = np.ascontiguousarray(seqlens.detach().cpu().numpy().astype(np.int32))
    o = np.empty((B, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    rc = _load().oracle_decode_fp8(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(ks), _ptr(vs), _ptr(sl),
                                   B, Hq, Hkv, Nmax, d, float(scale), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode_fp8 rejected its arguments")
    return torch.from_numpy(o), torch.from_numpy(lse)


def attn_fwd_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_scale: torch.Tensor,
                 k_scale: torch.Tensor, v_scale: torch.Tensor, scale: float, causal: bool,
                 rows: Optional[torch.Tensor] = None, window: int = 0):
    """fp64 attention of FP8 E4M3 q (B,Hq,Nq,d), k/v (B,Hkv,Nk,d) (uint8 bytes) with
    per-head dequantization scales: q row of head h is q_scale[h] * e4m3(bytes), K and V
    rows of head g are k_scale[g] * e4m3 and v_scale[g] * e4m3.  Rows and window as in
    attn_fwd; returns (o, lse) float64."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    for t in (q, k, v):
        assert t.dtype == torch.uint8, t.dtype
    qb, kb, vb = (np.ascontiguousarray(t.detach().cpu().numpy()) for t in (q, k, v))
    qs, ks, vs = (np.ascontiguousarray(t.detach().cpu().numpy().astype(np.float32))
                  for t in (q_scale, k_scale, v_scale))
    if rows is not None:
        rw = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        nr, rp = int(rw.shape[0]), _ptr(rw)
    else:
        rw, nr, rp = None, Nq, None
    o = np.empty((B, Hq, nr, d), dtype=np.float64)
    lse = np.empty((B, Hq, nr), dtype=np.float64)
    rc = _load().oracle_attn_fwd_fp8(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(qs), _ptr(ks), _ptr(vs),
                                     B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)),
                                     int(window), rp, nr, _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_fwd_fp8 rejected its arguments")
    return torch.from_numpy(o), torch.from_numpy(lse)
