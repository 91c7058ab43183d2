"""Runs every library path once through the debug build (FA_LIBRARY=.../libfa_debug.so, set by
the caller) and checks each against the fp64 oracle with no bounds check firing; then makes
the bounds self-test fire.  Prints "debug build ok" on success."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import torch  # noqa: E402

import oracle  # noqa: E402
from exact_io_aware_81_b200 import inputs, ops  # noqa: E402
from parity import compare  # noqa: E402

DEV = "cuda"


def main():
    lib = ops.load()
    assert lib.fa_build_flags() & 1, "not the debug build"

    def ok():
        rc = ops.get_error()
        assert rc == ops.FA_OK, (rc, lib.fa_last_error_message())

    for (B, Hq, Hkv, N, d, W) in [(2, 4, 4, 300, 128, 0), (1, 8, 2, 385, 64, 0), (1, 8, 2, 777, 128, 37)]:
        w = inputs.make_prefill(B, Hq, Hkv, N, N, d, seed=N, causal=True, window=W)
        q, k, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
        ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, True, window=W)
        for odt in (torch.bfloat16, torch.float32):
            o, lse = ops.fwd(q, k, v, causal=True, scale=w.scale, out_dtype=odt, window=W)
            ok()
            compare(o, lse, ro, rl, f"debug prefill {N} {odt}")
        o, lse = ops.fwd_bshd(*(t.transpose(1, 2).contiguous() for t in (q, k, v)), causal=True, scale=w.scale,
                              window=W)
        ok()
        compare(o.transpose(1, 2), lse, ro, rl, "debug bshd")
    w8 = inputs.make_fp8_prefill(1, 8, 2, 300, 300, 128, seed=7, causal=True)
    o, lse = ops.fwd_fp8(*[t.to(DEV) for t in (w8.q, w8.k, w8.v, w8.q_scale, w8.k_scale, w8.v_scale)], causal=True,
                         scale=w8.scale)
    ok()
    compare(o, lse, *oracle.attn_fwd_fp8(w8.q, w8.k, w8.v, w8.q_scale, w8.k_scale, w8.v_scale, w8.scale, True),
            "debug fp8 prefill")
    for d in (64, 128):
        dw = inputs.make_decode(5, 8, 2, 700, d, seed=d, len_range=(0, 700))
        o, lse = ops.decode(dw.q.to(DEV), dw.kcache.to(DEV), dw.vcache.to(DEV), dw.seqlens.to(DEV), scale=dw.scale)
        ok()
        compare(o, lse, *oracle.decode(dw.q, dw.kcache, dw.vcache, dw.seqlens, dw.scale), f"debug decode d{d}")
    pg = inputs.make_paged_decode(4, 8, 2, 64, 10, 128, seed=3, len_range=(1, 640))
    o, lse = ops.decode_paged(pg.q.to(DEV), pg.kpages.to(DEV), pg.vpages.to(DEV), pg.block_table.to(DEV),
                              pg.seqlens.to(DEV), scale=pg.scale)
    ok()
    compare(o, lse, *oracle.decode_paged(pg.q, pg.kpages, pg.vpages, pg.block_table, pg.seqlens, pg.scale),
            "debug paged")
    f8 = inputs.make_fp8_decode(4, 8, 2, 600, 128, seed=4, len_range=(1, 600))
    o, lse = ops.decode_fp8(f8.q.to(DEV), f8.kcache.to(DEV), f8.vcache.to(DEV), f8.k_scale.to(DEV),
                            f8.v_scale.to(DEV), f8.seqlens.to(DEV), scale=f8.scale)
    ok()
    compare(o, lse, *oracle.decode_fp8(f8.q, f8.kcache, f8.vcache, f8.k_scale, f8.v_scale, f8.seqlens, f8.scale),
            "debug fp8 decode")

    # the self-test moves every LSE index out of range: each store is skipped and reported
    w = inputs.make_prefill(1, 4, 4, 256, 256, 128, seed=9, causal=True)
    q, k, v = w.q.to(DEV), w.k.to(DEV), w.v.to(DEV)
    o = torch.empty((1, 4, 256, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((1, 4, 256), 12345.0, dtype=torch.float32, device=DEV)
    rc = lib.fa_debug_selftest_bounds(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                      1, 4, 4, 256, 256, 128, w.scale, 1, torch.cuda.current_stream().cuda_stream)
    assert rc == ops.FA_OK, lib.fa_last_error_message()
    assert ops.get_error() == ops.FA_ERR_DEBUG_CHECK
    assert ops.get_error() == ops.FA_OK
    assert (lse == 12345.0).all(), "an out-of-range LSE store was not skipped"
    ro, rl = oracle.attn_fwd(w.q, w.k, w.v, w.scale, True)
    err = (o.cpu().double() - ro).abs().max().item()
    assert err <= 2e-2, err
    print("debug build ok")


if __name__ == "__main__":
    main()
