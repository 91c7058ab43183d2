"""Parity of the (batch, sequence, heads, dim) entry point fa_fwd_bshd -- the layout the
flash_attn_func call on the toolsku.com page ("attention mechanism evolution",
FlashAttention usage example) takes -- with the fp64 oracle, and its bit-for-bit agreement
with the head-major entry points on the same tensors transposed.

The kernel reads the same tiles through strided 4-D TMA descriptors, so every output of the
two layouts must be identical; the oracle comparison pins each one independently.  The
cases cover MHA, GQA and MQA, d = 64 and 128, causal and non-causal, chunked rows
(Nq < Nk), a sliding window, an fp32 output and ragged tails; a full-size workload in this
layout is compared on seeded row samples.
"""
import pytest
import torch

import oracle
from exact_io_aware_81_b200 import inputs, ops
from parity import compare, guarded, guards_intact

pytestmark = pytest.mark.gpu

DEV = "cuda"


def bshd(t: torch.Tensor) -> torch.Tensor:
    """(B, H, N, d) -> contiguous (B, N, H, d)."""
    return t.transpose(1, 2).contiguous()


def run_bshd(w: inputs.Prefill, causal: bool, window: int = 0, out_dtype=torch.bfloat16):
    B, Hq, Hkv, Nq, Nk, d = w.shape
    q, k, v = bshd(w.q).to(DEV), bshd(w.k).to(DEV), bshd(w.v).to(DEV)
    obuf, o = guarded((B, Nq, Hq, d), out_dtype, DEV)
    lbuf, lse = guarded((B, Hq, Nq), torch.float32, DEV)
    ops.fwd_bshd(q, k, v, causal=causal, scale=w.scale, out_dtype=out_dtype, out=o, lse=lse, window=window)
    assert ops.get_error() == ops.FA_OK
    assert guards_intact(obuf) and guards_intact(lbuf), "write outside the output tensors"
    return o, lse


CASES = [  # (B, Hq, Hkv, Nq, Nk, d, causal, W, out fp32)
    (1, 2, 2, 300, 300, 128, True, 0, False),
    (2, 4, 4, 257, 257, 64, False, 0, False),
    (2, 8, 2, 700, 700, 128, True, 0, False),     # GQA head pairs
    (1, 4, 1, 513, 513, 128, True, 0, True),      # MQA, fp32 output
    (1, 3, 1, 400, 400, 64, True, 0, False),      # odd group size (row-pair tiling)
    (1, 8, 2, 200, 1000, 128, True, 0, False),    # chunked rows
    (1, 4, 2, 130, 900, 128, False, 0, True),
    (1, 8, 2, 777, 777, 128, True, 37, False),    # sliding window
    (2, 4, 4, 250, 1100, 64, True, 300, True),    # chunked rows with a window, fp32 output
    (3, 6, 3, 1, 129, 128, True, 0, False),       # one new row per sequence
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,W,f32", CASES,
                         ids=[f"b{c[0]}h{c[1]}g{c[2]}q{c[3]}k{c[4]}d{c[5]}{'c' if c[6] else 'n'}w{c[7]}"
                              f"{'f32' if c[8] else ''}" for c in CASES])
def test_bshd_parity(B, Hq, Hkv, Nq, Nk, d, causal, W, f32):
    w = inputs.make_prefill(B, Hq, Hkv, Nq, Nk, d, seed=hash((B, Hq, Hkv, Nq, Nk, d, causal, W)) % 10000,
                            causal=causal, window=W)
    odt = torch.float32 if f32 else torch.bfloat16
    o, lse = run_bshd(w, causal, W, odt)
    assert o.dtype == odt and tuple(o.shape) == (B, Nq, Hq, d)
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, causal, window=W)
    compare(o.transpose(1, 2), lse, ro, rl, "bshd")
    # the head-major entry point on the transposed tensors gives the same bits
    o2, l2 = ops.fwd(w.q.to(DEV), w.k.to(DEV), w.v.to(DEV), causal=causal, scale=w.scale, out_dtype=odt,
                     window=W)
    torch.cuda.synchronize()
    assert torch.equal(o.transpose(1, 2), o2) and torch.equal(lse, l2)


def test_bshd_workload3_sampled():
    w = inputs.workload(3)
    B, Hq, Hkv, Nq, Nk, d = w.shape
    o, lse = run_bshd(w, True)
    rows = inputs.sample_rows(Nq, 16, seed=91)
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, True, rows=rows)
    idx = rows.long().to(DEV)
    compare(o.index_select(1, idx).transpose(1, 2), lse.index_select(2, idx), ro, rl, "workload 3 bshd")
    assert torch.isfinite(lse).all() and torch.isfinite(o.float()).all()


def test_bshd_rejects_mismatched_outputs():
    w = inputs.make_prefill(1, 4, 2, 64, 64, 64, seed=3, causal=True)
    q, k, v = bshd(w.q).to(DEV), bshd(w.k).to(DEV), bshd(w.v).to(DEV)
    with pytest.raises(ValueError):   # a head-major output buffer
        ops.fwd_bshd(q, k, v, causal=True, out=torch.empty(1, 4, 64, 64, dtype=torch.bfloat16, device=DEV))
    with pytest.raises(ValueError):
        ops.fwd_bshd(q, k, v, causal=True, lse=torch.empty(1, 64, 4, dtype=torch.float32, device=DEV))
    with pytest.raises(ValueError):
        ops.fwd_bshd(q, k, v, causal=False, window=8)
