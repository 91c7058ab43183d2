"""The kernels of context-parallel decode on one GPU: fa_decode_ex with fp32 output, and
fa_merge_lse combining the parts of a cache cut into R contiguous slabs (the ranks are
emulated one after another on the same device; the exchange between ranks is covered by
the gloo test on CPU).  The merged result must match the oracle's decode over the whole
cache."""
import numpy as np
import pytest
import torch

import oracle
from oracle.split_kv import merge_lse as merge_ref
from exact_io_aware_81_b200 import inputs, ops
from exact_io_aware_81_b200.context_parallel import shard_seqlens
from parity import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_decode_ex_f32_output():
    w = inputs.make_decode(3, 8, 2, 700, 128, seed=41, len_range=(1, 700))
    sl = torch.tensor([0, 1, 700], dtype=torch.int32)
    o, lse = ops.decode_ex(w.q.to(DEV), w.kcache.to(DEV), w.vcache.to(DEV), sl.to(DEV), scale=w.scale,
                           out_dtype=torch.float32)
    assert ops.get_error() == ops.FA_OK and o.dtype == torch.float32
    ro, rl = oracle.decode(w.q, w.kcache, w.vcache, sl, w.scale)
    res = compare(o, lse, ro, rl, "decode fp32 out")
    assert res["o_max_abs"] < 1e-2  # no bf16 rounding of the output
    ob, lb = ops.decode(w.q.to(DEV), w.kcache.to(DEV), w.vcache.to(DEV), sl.to(DEV), scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(ob, o.to(torch.bfloat16)) and torch.equal(lb, lse)


@pytest.mark.parametrize("d,P", [(128, 1), (128, 3), (64, 8), (128, 40)])
def test_merge_lse_kernel(d, P):
    g = torch.Generator().manual_seed(d + P)
    rows = 37
    o_parts = torch.randn((P, rows, d), generator=g)
    lse_parts = torch.randn((P, rows), generator=g) * 5
    lse_parts[0, 3] = float("-inf")                # one empty part
    lse_parts[:, 5] = float("-inf")                # a row with no keys anywhere
    o_parts[0, 3] = float("nan")                   # an empty part's output is ignored
    ro, rl = merge_ref(o_parts.double().numpy(), lse_parts.double().numpy())
    for dt in (torch.float32, torch.bfloat16):
        o, lse = ops.merge_lse(o_parts.to(DEV), lse_parts.to(DEV), out_dtype=dt)
        torch.cuda.synchronize()
        o, lse = o.double().cpu().numpy(), lse.double().cpu().numpy()
        tol = 2e-6 if dt == torch.float32 else 1.6e-2
        assert np.allclose(o, ro, atol=tol, rtol=0), np.abs(o - ro).max()
        fin = np.isfinite(rl)
        assert np.allclose(lse[fin], rl[fin], atol=2e-6, rtol=0)
        assert np.isneginf(lse[5]) and (o[5] == 0).all()


@pytest.mark.parametrize("R", [2, 3, 4])
def test_emulated_context_parallel_decode(R):
    B, Hq, Hkv, Nmax, d = 8, 32, 8, 2048, 128
    w = inputs.make_decode(B, Hq, Hkv, Nmax, d, seed=43, len_range=(1, Nmax))
    sl = w.seqlens.clone()
    sl[0] = 0
    sl[1] = 5
    C = -(-Nmax // R)
    q = w.q.to(DEV)
    parts_o, parts_l = [], []
    for r in range(R):
        # every rank's shard has C rows (the last one padded): rank r holds keys r*C ..
        kc = torch.zeros((B, Hkv, C, d), dtype=torch.bfloat16)
        vc = torch.zeros((B, Hkv, C, d), dtype=torch.bfloat16)
        n = min(C, Nmax - r * C)
        kc[:, :, :n] = w.kcache[:, :, r * C:r * C + n]
        vc[:, :, :n] = w.vcache[:, :, r * C:r * C + n]
        o, l = ops.decode_ex(q, kc.to(DEV), vc.to(DEV), shard_seqlens(sl, r, C).to(DEV), scale=w.scale,
                             out_dtype=torch.float32)
        parts_o.append(o)
        parts_l.append(l)
    o, lse = ops.merge_lse(torch.stack(parts_o), torch.stack(parts_l))
    assert ops.get_error() == ops.FA_OK
    ro, rl = oracle.decode(w.q, w.kcache, w.vcache, sl, w.scale)
    compare(o, lse, ro, rl, f"context parallel R={R}")
