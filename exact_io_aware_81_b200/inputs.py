"""Seeded synthetic workloads for exact attention (prefill and KV-cache decode).

This module only draws random tensors: it holds none of the attention arithmetic, so
both the CPU oracle (through the tests) and the CUDA path consume exactly the same
bf16 bits.  Shapes follow the notation of the pages' cost analysis (youngju.dev,
"attention variants", section 1: B batch, H heads, N sequence length, d_k head dim)
and their grouped-query layout (same page, section 2: q is (B, H, N, d_k), k/v are
(B, G, N, d_k) with G key/value heads).  In this library G is called ``Hkv`` and the
number of query heads per key/value head is ``R = Hq // Hkv``.

Recipe (fixed so that every run and every machine sees the same bits):

* one ``torch.Generator('cpu')`` per workload, seeded with ``seed``;
* draw order: decode lengths -> per-head standard deviations -> Q -> K -> V ->
  outlier key rows;
* values are drawn as fp32 ``randn`` (times the per-head std or outlier factor, in
  fp32) and cast once to bf16 (round to nearest even, as torch does).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass
class Prefill:
    """One prefill problem: q (B,Hq,Nq,d), k/v (B,Hkv,Nk,d), all bf16 on the CPU."""
    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    causal: bool
    scale: float
    out_dtype: torch.dtype
    window: int = 0   # sliding window W (causal only); 0 = none

    @property
    def shape(self):
        B, Hq, Nq, d = self.q.shape
        Hkv, Nk = self.k.shape[1], self.k.shape[2]
        return B, Hq, Hkv, Nq, Nk, d

    def pairs(self) -> int:
        """Number of (query row, key) pairs that the mask allows, summed over B and Hq."""
        B, Hq, Hkv, Nq, Nk, d = self.shape
        return B * Hq * allowed_pairs(Nq, Nk, self.causal, self.window)

    def flops(self) -> float:
        """Algorithmic flops: 2*d for q.k plus 2*d for p*v, per allowed pair."""
        return 4.0 * self.shape[5] * self.pairs()

    def io_bytes(self) -> int:
        """Bytes that must cross HBM at least once: read Q, K, V, write O and LSE."""
        B, Hq, Hkv, Nq, Nk, d = self.shape
        ob = 4 if self.out_dtype == torch.float32 else 2
        return 2 * (B * Hq * Nq * d + 2 * B * Hkv * Nk * d) + ob * B * Hq * Nq * d + 4 * B * Hq * Nq


@dataclasses.dataclass
class Decode:
    """One decode step: q (B,Hq,d), caches (B,Hkv,Nmax,d) bf16, seqlens int32[B]."""
    name: str
    q: torch.Tensor
    kcache: torch.Tensor
    vcache: torch.Tensor
    seqlens: torch.Tensor
    scale: float

    @property
    def shape(self):
        B, Hq, d = self.q.shape
        Hkv, Nmax = self.kcache.shape[1], self.kcache.shape[2]
        return B, Hq, Hkv, Nmax, d

    def cache_bytes(self) -> int:
        """K and V bytes that the step must read: 2 tensors * Hkv * d * 2 B per cached token."""
        B, Hq, Hkv, Nmax, d = self.shape
        return int(self.seqlens.to(torch.int64).sum().item()) * Hkv * d * 2 * 2

    def io_bytes(self) -> int:
        """Cache bytes plus the q read and the bf16 o write."""
        B, Hq, Hkv, Nmax, d = self.shape
        return self.cache_bytes() + 2 * 2 * B * Hq * d + 4 * B

    def flops(self) -> float:
        B, Hq, Hkv, Nmax, d = self.shape
        return 4.0 * Hq * d * float(self.seqlens.to(torch.int64).sum().item())


@dataclasses.dataclass
class PagedDecode:
    """One decode step over a paged cache: q (B,Hq,d); kpages/vpages
    (num_pages,Hkv,page_size,d) bf16; block_table int32 (B,max_pages), -1 where unused;
    seqlens int32[B].  Token t of sequence b is row t % page_size of physical page
    block_table[b, t // page_size]."""
    name: str
    q: torch.Tensor
    kpages: torch.Tensor
    vpages: torch.Tensor
    block_table: torch.Tensor
    seqlens: torch.Tensor
    scale: float

    @property
    def shape(self):
        B, Hq, d = self.q.shape
        num_pages, Hkv, page_size = self.kpages.shape[:3]
        return B, Hq, Hkv, num_pages, page_size, self.block_table.shape[1], d

    def cache_bytes(self) -> int:
        B, Hq, Hkv, num_pages, page_size, max_pages, d = self.shape
        return int(self.seqlens.to(torch.int64).sum().item()) * Hkv * d * 2 * 2

    def io_bytes(self) -> int:
        """Cache bytes, q read, bf16 o write, seqlens and the block-table entries used."""
        B, Hq, Hkv, num_pages, page_size, max_pages, d = self.shape
        pages_used = int(((self.seqlens.to(torch.int64) + page_size - 1) // page_size).sum().item())
        return self.cache_bytes() + 2 * 2 * B * Hq * d + 4 * B + 4 * pages_used

    def flops(self) -> float:
        B, Hq, Hkv, num_pages, page_size, max_pages, d = self.shape
        return 4.0 * Hq * d * float(self.seqlens.to(torch.int64).sum().item())


@dataclasses.dataclass
class Fp8Decode:
    """One decode step over an FP8 E4M3 cache: q (B,Hq,d) bf16; kcache/vcache uint8
    (B,Hkv,Nmax,d) holding E4M3 bytes; k_scale/v_scale float32 (Hkv,): key j of head g is
    k_scale[g] * e4m3(kcache[b,g,j,:]) (likewise V); seqlens int32[B]."""
    name: str
    q: torch.Tensor
    kcache: torch.Tensor
    vcache: torch.Tensor
    k_scale: torch.Tensor
    v_scale: torch.Tensor
    seqlens: torch.Tensor
    scale: float

    @property
    def shape(self):
        B, Hq, d = self.q.shape
        Hkv, Nmax = self.kcache.shape[1], self.kcache.shape[2]
        return B, Hq, Hkv, Nmax, d

    def cache_bytes(self) -> int:
        """K and V bytes the step must read: 2 tensors * Hkv * d * 1 B per cached token."""
        B, Hq, Hkv, Nmax, d = self.shape
        return int(self.seqlens.to(torch.int64).sum().item()) * Hkv * d * 2

    def io_bytes(self) -> int:
        B, Hq, Hkv, Nmax, d = self.shape
        return self.cache_bytes() + 2 * 2 * B * Hq * d + 4 * B + 2 * 4 * Hkv

    def flops(self) -> float:
        B, Hq, Hkv, Nmax, d = self.shape
        return 4.0 * Hq * d * float(self.seqlens.to(torch.int64).sum().item())


E4M3_MAX = 448.0


def quantize_e4m3(x: torch.Tensor, head_dim: int = 1):
    """Per-head FP8 E4M3 encoding of an fp32 tensor: scale[g] = max|x[:, g]| / 448 and
    bytes = e4m3(x / scale) (torch's round-to-nearest-even cast, clamped to +-448).
    Returns (uint8 bytes, float32 scales).  Used only to prepare cache contents."""
    xt = x.transpose(0, head_dim)
    amax = xt.reshape(xt.shape[0], -1).abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax)).to(torch.float32)
    shape = [1] * x.dim()
    shape[head_dim] = -1
    y = (x / scale.view(shape)).clamp(-E4M3_MAX, E4M3_MAX)
    return y.to(torch.float8_e4m3fn).view(torch.uint8), scale


def make_fp8_decode(B: int, Hq: int, Hkv: int, Nmax: int, d: int, *, seed: int,
                    len_range: tuple, head_std_range: Optional[tuple] = (0.5, 2.0),
                    scale: Optional[float] = None, name: str = "fp8_decode") -> Fp8Decode:
    """Draw a seeded decode step over an FP8 cache.

    Draw order: seqlens -> per-K/V-head standard deviations (uniform in head_std_range,
    so every head gets its own scale) -> q -> K -> V, all fp32; K and V are then encoded
    per head with quantize_e4m3.
    """
    assert Hq % Hkv == 0
    gen = torch.Generator("cpu")
    gen.manual_seed(seed)
    lo, hi = len_range
    seqlens = torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    k_std = v_std = None
    if head_std_range is not None:
        a, b_ = head_std_range
        k_std = (a + (b_ - a) * torch.rand((Hkv,), generator=gen)).view(1, Hkv, 1, 1)
        v_std = (a + (b_ - a) * torch.rand((Hkv,), generator=gen)).view(1, Hkv, 1, 1)
    q = _randn(gen, (B, Hq, d))
    kc = _randn(gen, (B, Hkv, Nmax, d), k_std)
    vc = _randn(gen, (B, Hkv, Nmax, d), v_std)
    kq, ks = quantize_e4m3(kc)
    vq, vs = quantize_e4m3(vc)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return Fp8Decode(name=name, q=q.to(torch.bfloat16), kcache=kq, vcache=vq, k_scale=ks,
                     v_scale=vs, seqlens=seqlens, scale=float(scale))


@dataclasses.dataclass
class Fp8Prefill:
    """One prefill problem over FP8 E4M3 tensors: q (B,Hq,Nq,d), k/v (B,Hkv,Nk,d) uint8
    bytes; q_scale (Hq,), k_scale/v_scale (Hkv,) float32.  Row i of query head h is
    q_scale[h] * e4m3(q[b, h, i, :]); likewise K and V with their head's scale."""
    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    q_scale: torch.Tensor
    k_scale: torch.Tensor
    v_scale: torch.Tensor
    causal: bool
    scale: float
    window: int = 0
    out_dtype: torch.dtype = torch.bfloat16

    @property
    def shape(self):
        B, Hq, Nq, d = self.q.shape
        Hkv, Nk = self.k.shape[1], self.k.shape[2]
        return B, Hq, Hkv, Nq, Nk, d

    def pairs(self) -> int:
        B, Hq, Hkv, Nq, Nk, d = self.shape
        return B * Hq * allowed_pairs(Nq, Nk, self.causal, self.window)

    def flops(self) -> float:
        """Algorithmic flops: 2*d for q.k plus 2*d for p*v, per allowed pair."""
        return 4.0 * self.shape[5] * self.pairs()

    def io_bytes(self) -> int:
        """Read the E4M3 Q, K, V and the scales, write O and LSE."""
        B, Hq, Hkv, Nq, Nk, d = self.shape
        ob = 4 if self.out_dtype == torch.float32 else 2
        return (B * Hq * Nq * d + 2 * B * Hkv * Nk * d) + ob * B * Hq * Nq * d + 4 * B * Hq * Nq + 4 * (Hq + 2 * Hkv)


def make_fp8_prefill(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, *, seed: int,
                     causal: bool, window: int = 0, scale: Optional[float] = None,
                     head_std_range: Optional[tuple] = (0.5, 2.0),
                     outlier_rows_frac: float = 0.0, outlier_factor: float = 3.0,
                     name: str = "fp8_prefill") -> Fp8Prefill:
    """Draw a seeded prefill problem and encode it in FP8 E4M3 with one scale per head.

    Draw order: per-head standard deviations (Q heads, then K heads, then V heads, uniform
    in head_std_range) -> Q -> K -> V (fp32) -> outlier key rows (as make_prefill); then
    each tensor is encoded per head with quantize_e4m3.
    """
    assert Hq % Hkv == 0
    gen = torch.Generator("cpu")
    gen.manual_seed(seed)
    q_std = k_std = v_std = None
    if head_std_range is not None:
        lo, hi = head_std_range
        q_std = (lo + (hi - lo) * torch.rand((Hq,), generator=gen)).view(1, Hq, 1, 1)
        k_std = (lo + (hi - lo) * torch.rand((Hkv,), generator=gen)).view(1, Hkv, 1, 1)
        v_std = (lo + (hi - lo) * torch.rand((Hkv,), generator=gen)).view(1, Hkv, 1, 1)
    q = _randn(gen, (B, Hq, Nq, d), q_std)
    k = _randn(gen, (B, Hkv, Nk, d), k_std)
    v = _randn(gen, (B, Hkv, Nk, d), v_std)
    if outlier_rows_frac > 0.0:
        n_out = int(round(outlier_rows_frac * Nk))
        for b in range(B):
            for g in range(Hkv):
                rows = torch.randperm(Nk, generator=gen)[:n_out]
                k[b, g, rows, :] *= outlier_factor
    q8, qs = quantize_e4m3(q)
    k8, ks = quantize_e4m3(k)
    v8, vs = quantize_e4m3(v)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return Fp8Prefill(name=name, q=q8, k=k8, v=v8, q_scale=qs, k_scale=ks, v_scale=vs, causal=causal,
                      scale=float(scale), window=int(window))


def allowed_pairs(Nq: int, Nk: int, causal: bool, window: int = 0) -> int:
    """Pairs (i, j) with key j visible to query i.

    Causal masks use bottom-right alignment (row i sees keys 0 .. i + Nk - Nq), which
    requires Nq <= Nk; every row then sees c_i = i + Nk - Nq + 1 keys, or min(c_i, W)
    with a sliding window of W keys.
    """
    if not causal:
        return Nq * Nk
    assert Nq <= Nk
    off = Nk - Nq
    if window <= 0 or window >= Nk:
        return Nq * (off + 1) + Nq * (Nq - 1) // 2
    lo, hi = off + 1, Nk            # c_i runs over lo .. hi
    top = min(hi, window)           # rows with c_i <= W see all c_i keys
    full = (top - lo + 1) * (lo + top) // 2 if top >= lo else 0
    capped = hi - max(lo, window + 1) + 1
    return full + window * max(0, capped)


def _randn(gen, shape, std=None):
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if std is not None:
        x.mul_(std)
    return x


def make_prefill(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, *, seed: int,
                 causal: bool, scale: Optional[float] = None,
                 out_dtype: torch.dtype = torch.bfloat16,
                 head_std_range: Optional[tuple] = None,
                 outlier_rows_frac: float = 0.0, outlier_factor: float = 3.0,
                 window: int = 0, name: str = "prefill") -> Prefill:
    """Draw a seeded prefill problem.

    head_std_range=(lo, hi): each Q head and each K and V head gets its own standard
    deviation, uniform in [lo, hi], drawn before any tensor value.
    outlier_rows_frac: per (b, kv head), round(frac * Nk) key rows chosen by a seeded
    permutation are multiplied by ``outlier_factor`` in fp32 before the bf16 cast.
    """
    assert Hq % Hkv == 0
    gen = torch.Generator("cpu")
    gen.manual_seed(seed)
    q_std = k_std = v_std = None
    if head_std_range is not None:
        lo, hi = head_std_range
        q_std = (lo + (hi - lo) * torch.rand((Hq,), generator=gen)).view(1, Hq, 1, 1)
        k_std = (lo + (hi - lo) * torch.rand((Hkv,), generator=gen)).view(1, Hkv, 1, 1)
        v_std = (lo + (hi - lo) * torch.rand((Hkv,), generator=gen)).view(1, Hkv, 1, 1)
    q = _randn(gen, (B, Hq, Nq, d), q_std)
    k = _randn(gen, (B, Hkv, Nk, d), k_std)
    v = _randn(gen, (B, Hkv, Nk, d), v_std)
    if outlier_rows_frac > 0.0:
        n_out = int(round(outlier_rows_frac * Nk))
        for b in range(B):
            for g in range(Hkv):
                rows = torch.randperm(Nk, generator=gen)[:n_out]
                k[b, g, rows, :] *= outlier_factor
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return Prefill(name=name, q=q.to(torch.bfloat16), k=k.to(torch.bfloat16),
                   v=v.to(torch.bfloat16), causal=causal, scale=float(scale),
                   out_dtype=out_dtype, window=int(window))


def make_decode(B: int, Hq: int, Hkv: int, Nmax: int, d: int, *, seed: int,
                len_range: tuple, scale: Optional[float] = None,
                name: str = "decode") -> Decode:
    """Draw a seeded decode step; seqlens uniform on the inclusive range ``len_range``."""
    assert Hq % Hkv == 0
    gen = torch.Generator("cpu")
    gen.manual_seed(seed)
    lo, hi = len_range
    seqlens = torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    q = _randn(gen, (B, Hq, d))
    kc = _randn(gen, (B, Hkv, Nmax, d))
    vc = _randn(gen, (B, Hkv, Nmax, d))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return Decode(name=name, q=q.to(torch.bfloat16), kcache=kc.to(torch.bfloat16),
                  vcache=vc.to(torch.bfloat16), seqlens=seqlens, scale=float(scale))


def make_paged_decode(B: int, Hq: int, Hkv: int, page_size: int, max_pages: int, d: int, *,
                      seed: int, len_range: tuple, num_pages: Optional[int] = None,
                      scale: Optional[float] = None, name: str = "paged_decode") -> PagedDecode:
    """Draw a seeded decode step over a paged cache.

    Draw order: seqlens (uniform on the inclusive ``len_range``) -> a random permutation
    of the pool's pages, handed out in order to sequence 0's logical pages, then sequence
    1's, ... (so a sequence's pages are scattered over the pool) -> q -> kpages -> vpages.
    The pool holds ``num_pages`` pages (default: B * max_pages, room for every sequence at
    full length); block-table entries past a sequence's last page are -1.
    """
    assert Hq % Hkv == 0
    num_pages = num_pages or B * max_pages
    gen = torch.Generator("cpu")
    gen.manual_seed(seed)
    lo, hi = len_range
    assert 0 <= lo <= hi <= page_size * max_pages
    seqlens = torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    need = ((seqlens.to(torch.int64) + page_size - 1) // page_size).tolist()
    assert sum(need) <= num_pages, "pool too small"
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    used = 0
    for b in range(B):
        table[b, :need[b]] = perm[used:used + need[b]]
        used += need[b]
    q = _randn(gen, (B, Hq, d))
    kp = _randn(gen, (num_pages, Hkv, page_size, d))
    vp = _randn(gen, (num_pages, Hkv, page_size, d))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return PagedDecode(name=name, q=q.to(torch.bfloat16), kpages=kp.to(torch.bfloat16),
                       vpages=vp.to(torch.bfloat16), block_table=table, seqlens=seqlens,
                       scale=float(scale))


# The named workloads.  1-5 follow the pages' examples (H=32 and d_k=128 in the
# cost analysis, G=8 in the grouped-query section, contexts from 2K up to 32K).
WORKLOADS = {
    1: "mha_fwd_b1_h2_n256_d64_noncausal_f32out",
    2: "mha_causal_prefill_b8_h32_n2048_d128",
    3: "gqa_causal_prefill_b4_hq32_hkv8_n8192_d128",
    4: "gqa_causal_prefill_b1_hq32_hkv8_n32768_d128_headstd",
    5: "gqa_decode_b32_hq32_hkv8_nmax8192_d128",
    # sliding window and chunked prefill (youngju.dev sections 4 and 5), same head layout
    6: "gqa_swa_prefill_b1_hq32_hkv8_n32768_w4096_d128",
    7: "gqa_chunked_prefill_b1_hq32_hkv8_nq4096_nk32768_d128",
    8: "gqa_swa_chunked_prefill_b4_hq32_hkv8_nq2048_nk16384_w4096_d128",
    # decode 5 over a paged cache of 64-token pages (youngju.dev section 5)
    9: "gqa_paged_decode_b32_hq32_hkv8_page64_nmax8192_d128",
    # decode 5 over an FP8 (E4M3) cache with per-head scales (youngju.dev sections 5, 7)
    10: "gqa_fp8kv_decode_b32_hq32_hkv8_nmax8192_d128",
    # prefill over FP8 (E4M3) Q, K, V with per-head scales (toolsku.com, FlashAttention
    # generations table: FP8 among FA3's data types): workloads 2 and 3 encoded in FP8
    11: "fp8_mha_causal_prefill_b8_h32_n2048_d128",
    12: "fp8_gqa_causal_prefill_b4_hq32_hkv8_n8192_d128",
}


def workload(k: int):
    """Return named workload k (see WORKLOADS) drawn with seed 1000+k."""
    seed = 1000 + k
    name = WORKLOADS[k]
    if k == 1:
        return make_prefill(1, 2, 2, 256, 256, 64, seed=seed, causal=False,
                            out_dtype=torch.float32, name=name)
    if k == 2:
        return make_prefill(8, 32, 32, 2048, 2048, 128, seed=seed, causal=True,
                            outlier_rows_frac=0.01, outlier_factor=3.0, name=name)
    if k == 3:
        return make_prefill(4, 32, 8, 8192, 8192, 128, seed=seed, causal=True, name=name)
    if k == 4:
        return make_prefill(1, 32, 8, 32768, 32768, 128, seed=seed, causal=True,
                            head_std_range=(0.5, 2.0), name=name)
    if k == 5:
        return make_decode(32, 32, 8, 8192, 128, seed=seed, len_range=(1024, 8192), name=name)
    if k == 6:
        return make_prefill(1, 32, 8, 32768, 32768, 128, seed=seed, causal=True, window=4096,
                            name=name)
    if k == 7:
        return make_prefill(1, 32, 8, 4096, 32768, 128, seed=seed, causal=True, name=name)
    if k == 8:
        return make_prefill(4, 32, 8, 2048, 16384, 128, seed=seed, causal=True, window=4096,
                            name=name)
    if k == 9:
        return make_paged_decode(32, 32, 8, 64, 8192 // 64, 128, seed=seed, len_range=(1024, 8192),
                                 name=name)
    if k == 10:
        return make_fp8_decode(32, 32, 8, 8192, 128, seed=seed, len_range=(1024, 8192), name=name)
    if k == 11:
        return make_fp8_prefill(8, 32, 32, 2048, 2048, 128, seed=seed, causal=True, head_std_range=None,
                                outlier_rows_frac=0.01, outlier_factor=3.0, name=name)
    if k == 12:
        return make_fp8_prefill(4, 32, 8, 8192, 8192, 128, seed=seed, causal=True, name=name)
    raise KeyError(k)


def sample_rows(N: int, interior: int, seed: int, tile: int = 128) -> torch.Tensor:
    """Seeded sorted row sample: the fixed rows 0, 1, N-1 and both edges of every tile
    boundary (t*tile - 1, t*tile), plus ``interior`` further rows drawn at random, without
    replacement, from the rows not already fixed (all of them if fewer remain).

    With 128-row tiles the fixed rows are tensor-memory lanes 0, 1 and 127 of a tile; the
    random rows land on every other lane, so a sample checks the rows of every softmax warp.
    """
    fixed = {0, 1, N - 1}
    for t in range(1, (N + tile - 1) // tile):
        fixed.add(t * tile - 1)
        fixed.add(t * tile)
    fixed = {r for r in fixed if 0 <= r < N}
    gen = torch.Generator("cpu")
    gen.manual_seed(seed)
    rows = set(fixed)
    added = 0
    for r in torch.randperm(N, generator=gen).tolist():
        if added >= interior:
            break
        if r not in fixed:
            rows.add(r)
            added += 1
    return torch.tensor(sorted(rows), dtype=torch.int32)
