"""Context-parallel decode: every sequence's KV cache split across the ranks of a group.

Rank r holds keys [r * C, (r + 1) * C) of every sequence in a cache shard of C rows
(kcache_shard, vcache_shard: (B, Hkv, C, d)); a sequence of length L_b has
clamp(L_b - r * C, 0, C) of its keys there.  One decode step is then

  1. local split-KV decode of the shard (fa_decode_ex, fp32 output and LSE),
  2. all-gather of every rank's (o, lse) over the group (NCCL on GPUs),
  3. the log-sum-exp merge of the gathered parts (fa_merge_lse),

which gives exactly the decode over the whole cache: attention over disjoint key sets
combines by the same rescaling the online softmax applies between key blocks
(youngju.dev "attention variants", section 3).  It serves contexts longer than one
device's cache holds (same page, section 4: long-context attention).  Only step 2 moves
data between devices: B * Hq * (d + 1) * 4 bytes per rank.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

from . import ops


def shard_seqlens(seqlens: torch.Tensor, rank: int, shard_len: int) -> torch.Tensor:
    """Keys of each sequence that fall in rank `rank`'s shard of `shard_len` rows."""
    return (seqlens.to(torch.int64) - rank * shard_len).clamp(0, shard_len).to(torch.int32)


def _local_decode(q, kc, vc, sl, scale):
    return ops.decode_ex(q, kc, vc, sl, scale=scale, out_dtype=torch.float32)


def _merge(o_parts, lse_parts, out_dtype):
    return ops.merge_lse(o_parts, lse_parts, out_dtype=out_dtype)


def decode_context_parallel(q: torch.Tensor, kcache_shard: torch.Tensor, vcache_shard: torch.Tensor,
                            seqlens: torch.Tensor, group=None, *, scale: Optional[float] = None,
                            out_dtype: torch.dtype = torch.bfloat16,
                            local_decode: Optional[Callable] = None,
                            merge: Optional[Callable] = None):
    """Decode step over a cache split across the ranks of `group` (see the module text).

    q (B, Hq, d) bf16 and seqlens int32 (B,) (the full lengths) are the same on every rank;
    the shards hold this rank's keys, and every rank's shard has the same number of rows C
    (rank r holds keys r * C .. r * C + C - 1; a last, partly filled shard is padded).  Returns (o (B, Hq, d) out_dtype, lse (B, Hq) fp32),
    the same on every rank.  `local_decode(q, kc, vc, seqlens, scale) -> (o fp32, lse)` and
    `merge(o_parts, lse_parts, out_dtype) -> (o, lse)` default to the CUDA kernels; they
    are parameters so that the exchange can be exercised on CPU ranks.
    """
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    shard_len = kcache_shard.shape[2]
    sl_local = shard_seqlens(seqlens, rank, shard_len).to(seqlens.device)
    o_l, lse_l = (local_decode or _local_decode)(q, kcache_shard, vcache_shard, sl_local, scale)
    if o_l.dtype != torch.float32 or lse_l.dtype != torch.float32:
        raise ValueError("local decode must return fp32 o and lse")
    # gathered as the concatenation of the ranks' tensors along dim 0, viewed as stacked
    o_cat = torch.empty((world * o_l.shape[0],) + tuple(o_l.shape[1:]), dtype=torch.float32,
                        device=o_l.device)
    lse_cat = torch.empty((world * lse_l.shape[0],) + tuple(lse_l.shape[1:]), dtype=torch.float32,
                          device=lse_l.device)
    dist.all_gather_into_tensor(o_cat, o_l.contiguous(), group=group)
    dist.all_gather_into_tensor(lse_cat, lse_l.contiguous(), group=group)
    o_parts = o_cat.view((world,) + tuple(o_l.shape))
    lse_parts = lse_cat.view((world,) + tuple(lse_l.shape))
    return (merge or _merge)(o_parts, lse_parts, out_dtype)
