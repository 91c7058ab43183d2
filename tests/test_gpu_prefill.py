"""Parity of the sm_100a prefill kernel (fa_fwd through the C ABI) with the fp64 oracle.

Small problems are compared in full; they span several 128-row tiles, ragged tails, the
GQA / MQA / MHA head mappings (and an odd group size), d = 64 and 128, causal and not,
Nq < Nk causal, and N = 1.  The named full-size workloads run in the benchmark's launch
configuration: workload 2 on every row, the long grouped-query workloads on 256 random
rows per (b, h) on top of the first, last and tile-edge rows, so that every softmax
warp's rows are compared.  Outputs are written into guarded buffers whose NaN guard bands
must stay untouched.
"""
import math

import pytest
import torch

import oracle
from exact_io_aware_81_b200 import inputs, ops
from parity import compare, guarded, guards_intact

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_gpu(w: inputs.Prefill, out_dtype=None):
    out_dtype = out_dtype or w.out_dtype
    B, Hq, Hkv, Nq, Nk, d = w.shape
    q, k, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
    obuf, o = guarded((B, Hq, Nq, d), out_dtype, DEV)
    lbuf, lse = guarded((B, Hq, Nq), torch.float32, DEV)
    ops.fwd(q, k, v, causal=w.causal, scale=w.scale, out_dtype=out_dtype, out=o, lse=lse)
    assert ops.get_error() == ops.FA_OK
    assert guards_intact(obuf) and guards_intact(lbuf), "write outside the output tensors"
    return o, lse


SMALL = [  # (B, Hq, Hkv, Nq, Nk, d, causal)
    (1, 2, 2, 256, 256, 64, False),
    (1, 2, 2, 256, 256, 64, True),
    (2, 4, 4, 300, 300, 128, True),     # MHA, ragged, odd tile count
    (2, 4, 4, 300, 300, 128, False),
    (1, 8, 2, 129, 129, 128, True),     # GQA R=4
    (1, 8, 2, 385, 385, 64, False),
    (1, 4, 1, 200, 200, 128, True),     # MQA
    (1, 3, 1, 77, 77, 128, True),       # odd group size R=3
    (1, 6, 2, 250, 250, 64, True),      # R=3
    (1, 6, 6, 1, 1, 128, False),        # N = 1
    (1, 6, 6, 1, 1, 64, True),
    (1, 2, 2, 17, 17, 128, True),
    (1, 4, 2, 64, 320, 128, True),      # chunked prefill: Nq < Nk, bottom-right causal
    (1, 4, 2, 200, 1000, 64, True),
    (1, 4, 4, 130, 77, 128, False),     # Nq > Nk (non-causal)
    (1, 2, 1, 255, 255, 128, True),
    (2, 2, 2, 513, 513, 128, True),
    (1, 16, 2, 384, 384, 128, True),    # R=8
    (64, 16, 16, 64, 64, 128, True),    # 1024 short work slots over the persistent CTAs
    (64, 16, 16, 64, 64, 64, False),
    (1, 4, 2, 1, 5000, 128, False),     # one query row against a long key range
    (2, 8, 8, 3, 2000, 64, True),       # three new rows at the end of a long context
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal", SMALL,
                         ids=[f"b{c[0]}h{c[1]}g{c[2]}q{c[3]}k{c[4]}d{c[5]}{'c' if c[6] else 'n'}" for c in SMALL])
def test_small_parity(B, Hq, Hkv, Nq, Nk, d, causal):
    w = inputs.make_prefill(B, Hq, Hkv, Nq, Nk, d, seed=hash((B, Hq, Hkv, Nq, Nk, d, causal)) % 10000,
                            causal=causal)
    o, lse = run_gpu(w)
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, w.causal)
    compare(o, lse, ro, rl, "small")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_workload1_full(out_dtype):
    w = inputs.workload(1)
    o, lse = run_gpu(w, out_dtype)
    assert o.dtype == out_dtype
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, w.causal)
    compare(o, lse, ro, rl, "workload 1")


def test_workload2_full():
    """The causal MHA workload, every row of every (b, h) against the oracle."""
    w = inputs.workload(2)
    o, lse = run_gpu(w)
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, w.causal)
    compare(o, lse, ro, rl, "workload 2 (all rows)")


def interior_lanes(rows: torch.Tensor) -> dict:
    """How many sampled rows fall on each 32-lane quarter of a 128-row tile, edge lanes
    0, 1 and 127 left out: every softmax warp must have rows in the comparison."""
    lanes = rows.long() % 128
    inner = lanes[(lanes >= 2) & (lanes <= 126)]
    return {qtr: int(((inner // 32) == qtr).sum()) for qtr in range(4)}


@pytest.mark.parametrize("k,interior", [(3, 256), (4, 256)])
def test_named_workload_sampled(k, interior):
    """The long GQA workloads on 256 random rows per (b, h) on top of the first, last and
    tile-edge rows."""
    w = inputs.workload(k)
    B, Hq, Hkv, Nq, Nk, d = w.shape
    o, lse = run_gpu(w)
    rows = inputs.sample_rows(Nq, interior, seed=77 + k)
    assert min(interior_lanes(rows).values()) >= 32, interior_lanes(rows)
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, w.causal, rows=rows)
    idx = rows.long().to(DEV)
    compare(o.index_select(2, idx), lse.index_select(2, idx), ro, rl,
            f"workload {k} ({len(rows)} rows per head, interior lanes {interior_lanes(rows)})")
    # properties at full size: every LSE finite and every O row a convex combination of V
    assert torch.isfinite(lse).all()
    assert torch.isfinite(o.float()).all()


def test_gqa_equals_mha_after_repeat_interleave():
    w = inputs.make_prefill(2, 8, 2, 300, 300, 128, seed=5, causal=True)
    q, k, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
    o1, l1 = ops.fwd(q, k, v, causal=True)
    o2, l2 = ops.fwd(q, k.repeat_interleave(4, 1).contiguous(), v.repeat_interleave(4, 1).contiguous(),
                     causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_deterministic():
    w = inputs.make_prefill(2, 8, 8, 700, 700, 128, seed=6, causal=True)
    q, k, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
    a = ops.fwd(q, k, v, causal=True)
    b = ops.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_first_causal_row_is_v0():
    w = inputs.make_prefill(1, 4, 2, 256, 256, 128, seed=8, causal=True)
    o, lse = ops.fwd(w.q.to(DEV), w.k.to(DEV), w.v.to(DEV), causal=True, scale=w.scale)
    v0 = w.v[:, :, 0, :].repeat_interleave(2, 1)
    assert torch.equal(o[:, :, 0, :].cpu(), v0)
    s00 = w.scale * (w.q[:, :, 0].double() * w.k[:, :, 0].double().repeat_interleave(2, 1)).sum(-1)
    assert (lse[:, :, 0].cpu().double() - s00).abs().max().item() < 1e-4


def test_mask_boundaries_large_scores():
    # scores spread over ~100 in natural-log units: exercises the lazy rescale and masks
    w = inputs.make_prefill(1, 4, 4, 384, 384, 128, seed=9, causal=True)
    w.q = (w.q.float() * 4).to(torch.bfloat16)
    o, lse = run_gpu(w)
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, True)
    compare(o, lse, ro, rl, "large scores")
