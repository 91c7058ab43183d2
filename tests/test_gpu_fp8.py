"""Parity of the FP8 (E4M3) KV-cache decode (fa_decode_fp8, fa_decode_paged_fp8 through the
C ABI) with the fp64 oracle on the dequantized cache.

Key j of K/V head g is k_scale[g] * e4m3(byte) (likewise V): one scale per head, which the
seeded caches set per head from each head's largest magnitude.  The cases span every
query-head grouping the kernel instantiates, lengths on and around the 256-key chunk
edges, empty sequences, extreme scales and q magnitudes, and paged pools of several page
sizes, which must give bit for bit the result of the contiguous cache.
"""
import pytest
import torch

import oracle
from exact_io_aware_81_b200 import inputs, ops
from parity import compare, guarded, guards_intact

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_fp8(w: inputs.Fp8Decode, seqlens=None, q=None):
    B, Hq, Hkv, Nmax, d = w.shape
    sl = (w.seqlens if seqlens is None else seqlens).to(DEV)
    q = w.q if q is None else q
    obuf, o = guarded((B, Hq, d), torch.bfloat16, DEV)
    lbuf, lse = guarded((B, Hq), torch.float32, DEV)
    ws = torch.full((ops.decode_workspace_size(B, Hq, Nmax, d),), 0xFF, dtype=torch.uint8, device=DEV)
    ops.decode_fp8(q.to(DEV), w.kcache.to(DEV), w.vcache.to(DEV), w.k_scale.to(DEV), w.v_scale.to(DEV),
                   sl, scale=w.scale, workspace=ws, out=o, lse=lse)
    status = ops.get_error()
    assert guards_intact(obuf) and guards_intact(lbuf), "write outside the output tensors"
    return o, lse, status


CASES = [  # (B, Hq, Hkv, Nmax, lengths)
    (3, 8, 2, 300, [0, 1, 300]),                 # R = 4
    (4, 8, 8, 1000, [255, 256, 257, 999]),       # MHA (R = 1), chunk edges
    (2, 8, 1, 513, [513, 100]),                  # MQA R = 8
    (2, 6, 2, 700, [700, 3]),                    # R = 3
    (2, 12, 6, 600, [600, 512]),                 # R = 2
    (1, 32, 8, 8192, [8192]),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nmax,lengths", CASES,
                         ids=[f"b{c[0]}h{c[1]}g{c[2]}n{c[3]}" for c in CASES])
def test_fp8_parity(B, Hq, Hkv, Nmax, lengths):
    w = inputs.make_fp8_decode(B, Hq, Hkv, Nmax, 128, seed=31 + Nmax, len_range=(1, Nmax))
    sl = torch.tensor(lengths, dtype=torch.int32)
    o, lse, status = run_fp8(w, sl)
    assert status == ops.FA_OK
    ro, rl = oracle.decode_fp8(w.q, w.kcache, w.vcache, w.k_scale, w.v_scale, sl, w.scale)
    compare(o, lse, ro, rl, "fp8 decode")
    for b, L in enumerate(lengths):
        if L == 0:
            assert (o[b] == 0).all() and torch.isneginf(lse[b]).all()


def test_workload10_full():
    w = inputs.workload(10)
    o, lse, status = run_fp8(w)
    assert status == ops.FA_OK
    ro, rl = oracle.decode_fp8(w.q, w.kcache, w.vcache, w.k_scale, w.v_scale, w.seqlens, w.scale)
    compare(o, lse, ro, rl, "workload 10")


@pytest.mark.parametrize("q_mult", [1e-6, 1e4])
def test_fp8_extreme_q_and_scales(q_mult):
    # q far from 1 in both directions exercises the per-row power-of-two scaling before the
    # fp16 conversion; scales spanning many binades exercise the dequantization factors
    w = inputs.make_fp8_decode(2, 8, 2, 400, 128, seed=33, len_range=(1, 400))
    # q * q_mult with k_scale / q_mult keeps the scores of order one
    w.k_scale = w.k_scale * torch.tensor([0.5, 2.0]) / q_mult
    vf = torch.tensor([1e-4, 40.0])
    w.v_scale = w.v_scale * vf
    q = (w.q.float() * q_mult).to(torch.bfloat16)
    o, lse, status = run_fp8(w, q=q)
    assert status == ops.FA_OK
    ro, rl = oracle.decode_fp8(q, w.kcache, w.vcache, w.k_scale, w.v_scale, w.seqlens, w.scale)
    # outputs scale with the value factor: compare O / factor (of order one) per head
    f = vf.repeat_interleave(4).view(1, 8, 1).double()
    compare(o.cpu().double() / f, lse, ro / f, rl, f"fp8 q x {q_mult}")


def _scatter(cache, seqlens, ps, mp, num_pages, seed):
    B, Hkv, Nmax, d = cache.shape
    g = torch.Generator("cpu").manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g)
    pool = torch.full((num_pages, Hkv, ps, d), 0x7F, dtype=torch.uint8)  # E4M3 NaN where unused
    table = torch.full((B, mp), -1, dtype=torch.int32)
    used = 0
    for b in range(B):
        for t in range(-(-int(seqlens[b]) // ps)):
            pg = int(perm[used])
            used += 1
            table[b, t] = pg
            pool[pg] = cache[b, :, t * ps:(t + 1) * ps]
    return pool, table


@pytest.mark.parametrize("ps", [16, 48, 64, 256])
def test_paged_fp8_equals_contiguous(ps):
    mp = -(-1024 // ps)
    Nmax = ps * mp
    w = inputs.make_fp8_decode(4, 16, 4, Nmax, 128, seed=34, len_range=(1, Nmax))
    sl = torch.tensor([Nmax, 1, 257, Nmax - 5], dtype=torch.int32)
    kp, table = _scatter(w.kcache, sl, ps, mp, 4 * mp + 2, seed=ps)
    vp, _ = _scatter(w.vcache, sl, ps, mp, 4 * mp + 2, seed=ps)
    o, lse = ops.decode_paged_fp8(w.q.to(DEV), kp.to(DEV), vp.to(DEV), w.k_scale.to(DEV),
                                  w.v_scale.to(DEV), table.to(DEV), sl.to(DEV), scale=w.scale)
    assert ops.get_error() == ops.FA_OK
    oc, lc, status = run_fp8(w, sl)
    assert status == ops.FA_OK
    assert torch.equal(o, oc) and torch.equal(lse, lc)
    ro, rl = oracle.decode_fp8(w.q, w.kcache, w.vcache, w.k_scale, w.v_scale, sl, w.scale)
    compare(o, lse, ro, rl, f"paged fp8 {ps}")


def test_fp8_many_sequences():
    # more than 32 sequences and more items than the kernel has workers
    B = 100
    w = inputs.make_fp8_decode(B, 8, 2, 1000, 128, seed=35, len_range=(0, 1000))
    sl = w.seqlens.clone()
    sl[::9] = 0
    sl[2::10] = 1
    o, lse, status = run_fp8(w, sl)
    assert status == ops.FA_OK
    ro, rl = oracle.decode_fp8(w.q, w.kcache, w.vcache, w.k_scale, w.v_scale, sl, w.scale)
    compare(o, lse, ro, rl, "fp8 many sequences")
