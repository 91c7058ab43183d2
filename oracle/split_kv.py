"""Split-KV decode with a log-sum-exp merge -- TEST INFRASTRUCTURE (oracle side).

The pages do not print a split-KV decode; its merge is the same rescaling that the
online softmax of youngju.dev "attention variants", section 3 applies between blocks,
applied across independently computed chunks of the cache:

  per chunk s (keys [s*C, min((s+1)*C, L))):  o_s = softmax(s_chunk) @ V_chunk,
                                              lse_s = ln sum exp(s_chunk)
  merge:  M = max_s lse_s,  w_s = exp(lse_s - M),
          o = sum_s w_s o_s / sum_s w_s,   lse = M + ln sum_s w_s

Written in float64 numpy, one (b, h) at a time; only for checking that every chunk size
reproduces the unsplit definition.  ``merge_lse`` is the merge step alone, over any number
of partials (the cross-device merge of context-parallel decode uses the same algebra).
"""
from __future__ import annotations

import numpy as np


def merge_lse(o_parts, lse_parts):
    """Merge P partial results: o_parts (P, ..., d), lse_parts (P, ...) natural-log sums.

    A partial with lse = -inf (no keys) has weight 0; if every partial has none, o = 0 and
    lse = -inf.  Returns (o (..., d), lse (...)) in float64.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    M = lse_parts.max(axis=0)
    empty = np.isneginf(M)
    Ms = np.where(empty, 0.0, M)
    w = np.exp(lse_parts - Ms)                      # exp(-inf) = 0 for empty partials
    den = w.sum(axis=0)
    num = (w[..., None] * np.where(np.isneginf(lse_parts)[..., None], 0.0, o_parts)).sum(axis=0)
    o = np.where(empty[..., None], 0.0, num / np.where(empty, 1.0, den)[..., None])
    lse = np.where(empty, -np.inf, Ms + np.log(np.where(empty, 1.0, den)))
    return o, lse


def split_kv_decode(q, kcache, vcache, seqlens, scale, chunk):
    """q (B,Hq,d), caches (B,Hkv,Nmax,d) float64; returns (o (B,Hq,d), lse (B,Hq))."""
    q = np.asarray(q, dtype=np.float64)
    kc = np.asarray(kcache, dtype=np.float64)
    vc = np.asarray(vcache, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = kc.shape[1]
    R = Hq // Hkv
    o = np.zeros((B, Hq, vc.shape[3]))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        L = int(seqlens[b])
        for h in range(Hq):
            g = h // R
            parts = []
            for c0 in range(0, L, chunk):
                kk = kc[b, g, c0:min(c0 + chunk, L)]
                vv = vc[b, g, c0:min(c0 + chunk, L)]
                s = (kk @ q[b, h]) * scale
                m = s.max()
                e = np.exp(s - m)
                parts.append(((e @ vv) / e.sum(), m + np.log(e.sum())))
            if not parts:
                continue
            o[b, h], lse[b, h] = merge_lse(np.stack([p[0] for p in parts]),
                                           np.array([p[1] for p in parts]))
    return o, lse
