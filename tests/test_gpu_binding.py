"""The Python binding refuses caller-provided outputs of the wrong shape or dtype before it
calls the library (nothing is launched), and passes through outputs of the right shape."""
import pytest
import torch

from exact_io_aware_81_b200 import inputs, ops

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16, device=DEV)


def _f32(*shape):
    return torch.zeros(shape, dtype=torch.float32, device=DEV)


def test_fwd_outputs_checked():
    q, k = _bf(1, 4, 64, 64), _bf(1, 2, 64, 64)
    with pytest.raises(ValueError):
        ops.fwd(q, k, k, causal=True, out=_bf(1, 4, 63, 64))
    with pytest.raises(ValueError):
        ops.fwd(q, k, k, causal=True, out=_f32(1, 4, 64, 64))      # dtype differs from out_dtype
    with pytest.raises(ValueError):
        ops.fwd(q, k, k, causal=True, lse=_f32(1, 4, 64, 1))
    o, lse = ops.fwd(q, k, k, causal=True, out=_bf(1, 4, 64, 64), lse=_f32(1, 4, 64))
    torch.cuda.synchronize()
    assert ops.get_error() == ops.FA_OK and tuple(o.shape) == (1, 4, 64, 64)


def test_decode_outputs_checked():
    d = inputs.make_decode(2, 8, 2, 300, 128, seed=3, len_range=(1, 300))
    q, kc, vc, sl = d.q.to(DEV), d.kcache.to(DEV), d.vcache.to(DEV), d.seqlens.to(DEV)
    for fn in (ops.decode, ops.decode_ex, ops.decode_noalloc):
        with pytest.raises(ValueError):
            fn(q, kc, vc, sl, out=_bf(2, 8, 64))
        with pytest.raises(ValueError):
            fn(q, kc, vc, sl, out=_bf(2, 8, 128), lse=_f32(8, 2))
    with pytest.raises(ValueError):
        ops.decode_ex(q, kc, vc, sl, out_dtype=torch.float32, out=_bf(2, 8, 128))


def test_merge_outputs_checked():
    op, lp = _f32(2, 5, 64), _f32(2, 5)
    with pytest.raises(ValueError):
        ops.merge_lse(op, lp, out=_bf(5, 32))
    with pytest.raises(ValueError):
        ops.merge_lse(op, lp, lse=_f32(4))
