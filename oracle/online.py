"""Block-by-block online softmax -- TEST INFRASTRUCTURE (oracle side).

A plain numpy restatement of the tiled loop on youngju.dev "attention variants",
section 3 ("FlashAttention"): an outer loop over query blocks, an inner loop over
key/value blocks, a block score, a running row maximum, and a rescale of what was
accumulated so far before adding the new block.  The page leaves the running sum,
the rescale step and the final normalisation unwritten; they are completed in the
plainest way consistent with its statement that the online form gives exactly the
two-pass result:

    alpha   = exp(m_old - m_new)                per row
    l       = alpha * l + sum_j exp(s_j - m_new)
    acc     = alpha * acc + exp(s - m_new) @ V_block
    O_block = acc / l,   lse = m + ln l

A partial last block is simply shorter.  ``lazy_threshold`` optionally keeps a stale
maximum until the new one exceeds it by more than the threshold (natural-log units);
that changes only rounding, never the exact result.  Only for tiny inputs.
"""
from __future__ import annotations

import numpy as np


def online_attention(q, k, v, scale, causal, block_q, block_k, lazy_threshold=None):
    """q (Nq,d), k/v (Nk,d) float64 arrays -> (o (Nq,d), lse (Nq,))."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Nq, d = q.shape
    Nk = k.shape[0]
    off = Nk - Nq
    o = np.zeros((Nq, v.shape[1]))
    lse = np.zeros(Nq)
    for i0 in range(0, Nq, block_q):                      # query blocks
        qb = q[i0:i0 + block_q]
        nb = qb.shape[0]
        rows = np.arange(i0, i0 + nb)
        m = np.full(nb, -np.inf)
        l = np.zeros(nb)
        acc = np.zeros((nb, v.shape[1]))
        for j0 in range(0, Nk, block_k):                  # key/value blocks
            kb = k[j0:j0 + block_k]
            vb = v[j0:j0 + block_k]
            s = (qb @ kb.T) * scale
            if causal:
                keys = np.arange(j0, j0 + kb.shape[0])
                s = np.where(keys[None, :] <= rows[:, None] + off, s, -np.inf)
            bmax = s.max(axis=1)
            m_new = np.maximum(m, bmax)
            if lazy_threshold is not None:
                keep = np.isfinite(m) & (m_new - m <= lazy_threshold)
                m_new = np.where(keep, m, m_new)
            with np.errstate(invalid="ignore"):
                alpha = np.where(np.isfinite(m), np.exp(m - m_new), 0.0)
            p = np.where(np.isfinite(s), np.exp(s - m_new[:, None]), 0.0)
            l = alpha * l + p.sum(axis=1)
            acc = alpha[:, None] * acc + p @ vb
            m = m_new
        o[i0:i0 + nb] = acc / l[:, None]
        lse[i0:i0 + nb] = m + np.log(l)
    return o, lse
