"""Parity of the FP8 (E4M3) prefill (fa_fwd_fp8 through the C ABI) with the fp64 oracle.

Q, K and V are E4M3 bytes with one fp32 dequantization scale per head (toolsku.com,
FlashAttention generations table: FP8 among FA3's data types; the scale convention is this
library's).  The oracle is the attention of the dequantized tensors.  The small cases span
the MHA row-pair and GQA head-pair tilings, MQA, an odd group size, ragged tails, chunked
causal (Nq < Nk), non-causal, sliding windows and both output types; the two named FP8
workloads run at full size, workload 11 (the causal MHA workload in FP8) compared on every
row, workload 12 (the 8K GQA workload in FP8) on 256 random rows per (b, h) plus the edges.
Same tolerance as the bf16 path.
"""
import pytest
import torch

import oracle
from exact_io_aware_81_b200 import inputs, ops
from parity import compare, guarded, guards_intact

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_gpu(w: inputs.Fp8Prefill, out_dtype=torch.bfloat16):
    B, Hq, Hkv, Nq, Nk, d = w.shape
    t = [x.to(DEV) for x in (w.q, w.k, w.v, w.q_scale, w.k_scale, w.v_scale)]
    obuf, o = guarded((B, Hq, Nq, d), out_dtype, DEV)
    lbuf, lse = guarded((B, Hq, Nq), torch.float32, DEV)
    ops.fwd_fp8(*t, causal=w.causal, scale=w.scale, out_dtype=out_dtype, out=o, lse=lse, window=w.window)
    assert ops.get_error() == ops.FA_OK
    assert guards_intact(obuf) and guards_intact(lbuf), "write outside the output tensors"
    return o, lse


def run_oracle(w: inputs.Fp8Prefill, rows=None):
    return oracle.attn_fwd_fp8(w.q, w.k, w.v, w.q_scale, w.k_scale, w.v_scale, w.scale, w.causal,
                               rows=rows, window=w.window)


SMALL = [  # (B, Hq, Hkv, Nq, Nk, causal, window)
    (1, 2, 2, 256, 256, True, 0),
    (2, 4, 4, 300, 300, True, 0),      # MHA row pairs, ragged, odd tile count
    (2, 4, 4, 300, 300, False, 0),
    (1, 8, 2, 385, 385, True, 0),      # GQA head pairs (R = 4)
    (1, 8, 2, 129, 129, False, 0),
    (1, 4, 1, 200, 200, True, 0),      # MQA
    (1, 3, 1, 77, 77, True, 0),        # odd group size
    (1, 6, 6, 1, 1, True, 0),          # N = 1
    (1, 4, 2, 64, 320, True, 0),       # chunked prefill
    (1, 4, 2, 200, 1000, True, 0),
    (1, 4, 4, 130, 77, False, 0),      # Nq > Nk, non-causal
    (1, 16, 2, 384, 384, True, 0),     # R = 8
    (1, 2, 2, 700, 700, True, 100),    # windows: row pairs and head pairs, chunked
    (1, 8, 2, 777, 777, True, 37),
    (1, 4, 2, 200, 1000, True, 300),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,causal,W", SMALL,
                         ids=[f"b{c[0]}h{c[1]}g{c[2]}q{c[3]}k{c[4]}{'c' if c[5] else 'n'}w{c[6]}" for c in SMALL])
def test_small_fp8_parity(B, Hq, Hkv, Nq, Nk, causal, W):
    w = inputs.make_fp8_prefill(B, Hq, Hkv, Nq, Nk, 128, seed=hash((B, Hq, Hkv, Nq, Nk, causal, W)) % 10000,
                                causal=causal, window=W)
    o, lse = run_gpu(w)
    compare(o, lse, *run_oracle(w), f"fp8 small w{W}")


def test_fp8_f32_output_and_large_scores():
    # wide per-head scales: scores spread over tens of natural-log units, so the lazy
    # rescale (threshold 2^8 for fp16 P) is taken
    w = inputs.make_fp8_prefill(1, 4, 2, 640, 640, 128, seed=41, causal=True, head_std_range=(0.5, 4.0))
    w.q_scale = w.q_scale * 4
    o, lse = run_gpu(w, torch.float32)
    assert o.dtype == torch.float32
    compare(o, lse, *run_oracle(w), "fp8 f32 large scores")


def test_fp8_first_causal_row_is_v0():
    w = inputs.make_fp8_prefill(1, 4, 2, 256, 256, 128, seed=42, causal=True)
    o, lse = run_gpu(w, torch.float32)
    v0 = (w.v[:, :, 0, :].view(torch.float8_e4m3fn).float() * w.v_scale.view(1, -1, 1)).repeat_interleave(2, 1)
    assert torch.allclose(o[:, :, 0, :].cpu(), v0, rtol=1e-6, atol=1e-6)


def test_fp8_deterministic():
    w = inputs.make_fp8_prefill(2, 8, 2, 700, 700, 128, seed=43, causal=True)
    a, b = run_gpu(w), run_gpu(w)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_workload11_full():
    """The causal MHA workload (B=8, H=32, N=2048) in FP8, every row against the oracle."""
    w = inputs.workload(11)
    o, lse = run_gpu(w)
    compare(o, lse, *run_oracle(w), "workload 11 (all rows)")


def test_workload12_sampled():
    """The 8K GQA workload in FP8 on 256 random rows per (b, h) on top of the edge rows."""
    w = inputs.workload(12)
    B, Hq, Hkv, Nq, Nk, d = w.shape
    o, lse = run_gpu(w)
    rows = inputs.sample_rows(Nq, 256, seed=89)
    idx = rows.long().to(DEV)
    compare(o.index_select(2, idx), lse.index_select(2, idx), *run_oracle(w, rows),
            f"workload 12 ({len(rows)} rows per head)")
    assert torch.isfinite(lse).all() and torch.isfinite(o.float()).all()
