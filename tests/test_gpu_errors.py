"""Device-side error reporting, without faulting, trapping or hanging the GPU.

Each time-limit test withholds one internal signal so that a bounded wait runs out after a
short limit: in the prefill kernel the score-ready arrive of the MMA warp, in the decode
split kernels (bf16 shared ring, FP8 per-warp rings) the first copy of every CTA's producer.
The kernel must record FA_ERR_TIMEOUT, stop every role at its next wait, let the copies
already issued land, free its tensor memory and return; for decode the merge kernel, a
programmatic dependent of the split kernel, then still runs and ends.  The context must stay
usable: a normal call right after matches the oracle.
"""
import pytest
import torch

import oracle
from exact_io_aware_81_b200 import inputs, ops
from parity import compare

pytestmark = pytest.mark.gpu


def test_wait_limit_expires_cleanly():
    w = inputs.make_prefill(1, 4, 4, 512, 512, 128, seed=12, causal=True)
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    ops.set_wait_limit_ns(20_000_000)  # 20 ms
    try:
        ops.fwd_selftest_timeout(q, k, v, causal=True)
        assert ops.get_error() == ops.FA_ERR_TIMEOUT
        assert ops.get_error() == ops.FA_OK  # cleared
    finally:
        ops.set_wait_limit_ns(0)
    # the context still works
    o, lse = ops.fwd(q, k, v, causal=True, scale=w.scale)
    assert ops.get_error() == ops.FA_OK
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, True)
    compare(o, lse, ro, rl, "after timeout")


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 2, 128), (6, 6, 64)])
def test_decode_wait_limit_expires_cleanly(Hq, Hkv, d):
    w = inputs.make_decode(5, Hq, Hkv, 1500, d, seed=13, len_range=(1, 1500))
    q, kc, vc, sl = w.q.cuda(), w.kcache.cuda(), w.vcache.cuda(), w.seqlens.cuda()
    ops.set_wait_limit_ns(20_000_000)
    try:
        ops.decode_selftest_timeout(q, kc, vc, sl, scale=w.scale)
        assert ops.get_error() == ops.FA_ERR_TIMEOUT
        assert ops.get_error() == ops.FA_OK
    finally:
        ops.set_wait_limit_ns(0)
    o, lse = ops.decode(q, kc, vc, sl, scale=w.scale)
    assert ops.get_error() == ops.FA_OK
    compare(o, lse, *oracle.decode(w.q, w.kcache, w.vcache, w.seqlens, w.scale), "decode after timeout")


def test_fp8_decode_wait_limit_expires_cleanly():
    w = inputs.make_fp8_decode(5, 8, 2, 1500, 128, seed=14, len_range=(1, 1500))
    args = [t.cuda() for t in (w.q, w.kcache, w.vcache, w.seqlens)]
    ks, vs = w.k_scale.cuda(), w.v_scale.cuda()
    ops.set_wait_limit_ns(20_000_000)
    try:
        ops.decode_selftest_timeout(*args, k_scale=ks, v_scale=vs, scale=w.scale)
        assert ops.get_error() == ops.FA_ERR_TIMEOUT
        assert ops.get_error() == ops.FA_OK
    finally:
        ops.set_wait_limit_ns(0)
    q, kc, vc, sl = args
    o, lse = ops.decode_fp8(q, kc, vc, ks, vs, sl, scale=w.scale)
    assert ops.get_error() == ops.FA_OK
    compare(o, lse, *oracle.decode_fp8(w.q, w.kcache, w.vcache, w.k_scale, w.v_scale, w.seqlens, w.scale),
            "FP8 decode after timeout")
