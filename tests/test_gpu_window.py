"""Parity of sliding-window causal attention (fa_fwd_window through the C ABI) with the
fp64 oracle, and of chunked prefill (Nq < Nk).

Row i sees keys j with i + Nk - Nq - W < j <= i + Nk - Nq (youngju.dev "attention
variants", section 4).  The small cases span windows narrower than one 128-key tile, equal
to it and a little wider, windows that start mid-tile, the MHA row-pair and GQA head-pair
tilings, d = 64 and 128, ragged tails and Nq < Nk.  The full-size window and chunked
workloads are compared on 256 random rows per (b, h) on top of the first, last and
tile-edge rows.
"""
import pytest
import torch

import oracle
from exact_io_aware_81_b200 import inputs, ops
from parity import compare, guarded, guards_intact

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_gpu(w: inputs.Prefill, window: int, out_dtype=None):
    out_dtype = out_dtype or w.out_dtype
    B, Hq, Hkv, Nq, Nk, d = w.shape
    q, k, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
    obuf, o = guarded((B, Hq, Nq, d), out_dtype, DEV)
    lbuf, lse = guarded((B, Hq, Nq), torch.float32, DEV)
    ops.fwd_window(q, k, v, window, scale=w.scale, out_dtype=out_dtype, out=o, lse=lse)
    assert ops.get_error() == ops.FA_OK
    assert guards_intact(obuf) and guards_intact(lbuf), "write outside the output tensors"
    return o, lse


SMALL = [  # (B, Hq, Hkv, Nq, Nk, d, W)
    (1, 2, 2, 300, 300, 128, 1),       # only the diagonal key
    (1, 2, 2, 300, 300, 128, 64),
    (2, 4, 4, 700, 700, 64, 128),      # exactly one tile wide
    (1, 2, 2, 1000, 1000, 128, 129),
    (1, 2, 2, 1000, 1000, 128, 300),
    (1, 8, 2, 777, 777, 128, 37),      # GQA head pairs
    (1, 8, 2, 777, 777, 64, 256),
    (1, 4, 1, 513, 513, 128, 200),     # MQA
    (1, 3, 1, 400, 400, 128, 100),     # odd group size (row-pair tiling)
    (1, 4, 2, 200, 1000, 128, 300),    # chunked prefill with a window
    (1, 4, 4, 130, 900, 64, 50),
    (1, 8, 2, 256, 2048, 128, 384),
    (1, 8, 2, 1, 5000, 128, 1000),     # a single new row
    (1, 2, 2, 2000, 2000, 128, 1999),  # one key short of plain causal
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,W", SMALL,
                         ids=[f"b{c[0]}h{c[1]}g{c[2]}q{c[3]}k{c[4]}d{c[5]}w{c[6]}" for c in SMALL])
def test_small_window_parity(B, Hq, Hkv, Nq, Nk, d, W):
    w = inputs.make_prefill(B, Hq, Hkv, Nq, Nk, d, seed=hash((B, Hq, Hkv, Nq, Nk, d, W)) % 10000,
                            causal=True, window=W)
    o, lse = run_gpu(w, W)
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, True, window=W)
    compare(o, lse, ro, rl, f"window {W}")


def test_window_one_is_the_diagonal_value():
    w = inputs.make_prefill(1, 4, 2, 300, 420, 128, seed=31, causal=True)
    o, lse = run_gpu(w, 1)
    want = w.v[:, :, 120:, :].repeat_interleave(2, 1)
    assert torch.equal(o.cpu(), want)


@pytest.mark.parametrize("W", [300, 301, 100000])
def test_window_covering_every_key_is_causal(W):
    w = inputs.make_prefill(1, 4, 2, 250, 300, 128, seed=32, causal=True)
    q, k, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
    oc, lc = ops.fwd(q, k, v, causal=True, scale=w.scale)
    ow, lw = ops.fwd_window(q, k, v, W, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(oc, ow) and torch.equal(lc, lw)


def test_window_f32_output_and_large_scores():
    # scores spread over ~100 natural-log units: rows whose first key tile is wholly
    # outside the window start from -inf and must rescale cleanly
    w = inputs.make_prefill(1, 4, 4, 640, 640, 128, seed=33, causal=True)
    w.q = (w.q.float() * 4).to(torch.bfloat16)
    for W in (70, 200):
        o, lse = run_gpu(w, W, torch.float32)
        assert o.dtype == torch.float32
        ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, True, window=W)
        compare(o, lse, ro, rl, f"large scores, window {W}")


def test_window_deterministic():
    w = inputs.make_prefill(2, 8, 2, 900, 900, 128, seed=34, causal=True)
    q, k, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
    a = ops.fwd_window(q, k, v, 200)
    b = ops.fwd_window(q, k, v, 200)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("k", [6, 7, 8])
def test_named_window_workload_sampled(k):
    w = inputs.workload(k)
    B, Hq, Hkv, Nq, Nk, d = w.shape
    q, kk, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
    if w.window:
        o, lse = ops.fwd_window(q, kk, v, w.window, scale=w.scale)
    else:
        o, lse = ops.fwd(q, kk, v, causal=True, scale=w.scale)
    assert ops.get_error() == ops.FA_OK
    # 256 random rows per (b, h) on top of the first, last and tile-edge rows
    rows = inputs.sample_rows(Nq, 256, seed=77 + k)
    lanes = rows.long() % 128
    inner = lanes[(lanes >= 2) & (lanes <= 126)] // 32
    assert all(int((inner == qtr).sum()) >= 32 for qtr in range(4))
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, True, rows=rows, window=w.window)
    idx = rows.long().to(DEV)
    compare(o.index_select(2, idx), lse.index_select(2, idx), ro, rl, f"workload {k} ({len(rows)} rows per head)")
    assert torch.isfinite(lse).all()
    assert torch.isfinite(o.float()).all()
