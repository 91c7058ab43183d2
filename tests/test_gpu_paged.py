"""Parity of the paged-cache decode (fa_decode_paged through the C ABI) with the fp64
oracle, and bitwise agreement with the contiguous decode on the same logical cache.

Pages are (num_pages, Hkv, page_size, d); token t of sequence b is row t % page_size of
page block_table[b, t // page_size] (youngju.dev "attention variants", section 5).  The
cases span page sizes from 16 to 512 (including 48, which is not a power of two), lengths
on and around page and 256-key chunk edges, empty sequences, every query-head grouping the
kernel instantiates and d = 64 and 128.
"""
import pytest
import torch

import oracle
from exact_io_aware_81_b200 import inputs, ops
from parity import compare, guarded, guards_intact

pytestmark = pytest.mark.gpu

DEV = "cuda"


def scatter_to_pages(cache, seqlens, page_size, max_pages, num_pages, seed):
    """Copy a contiguous cache (B,Hkv,Nmax,d) into a pool of pages taken in a seeded random
    order; unused pool pages hold NaN, unused table entries -1."""
    B, Hkv, Nmax, d = cache.shape
    g = torch.Generator("cpu").manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g)
    pool = torch.full((num_pages, Hkv, page_size, d), float("nan"), dtype=cache.dtype)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    used = 0
    for b in range(B):
        for t in range(-(-int(seqlens[b]) // page_size)):
            pg = int(perm[used])
            used += 1
            table[b, t] = pg
            rows = cache[b, :, t * page_size:(t + 1) * page_size]
            pool[pg, :, :rows.shape[1]] = rows
    return pool, table


def run_paged(q, kp, vp, table, sl, scale):
    B, Hq, d = q.shape
    page_size, max_pages = kp.shape[2], table.shape[1]
    obuf, o = guarded((B, Hq, d), torch.bfloat16, DEV)
    lbuf, lse = guarded((B, Hq), torch.float32, DEV)
    ws = torch.full((ops.decode_workspace_size(B, Hq, page_size * max_pages, d),), 0xFF,
                    dtype=torch.uint8, device=DEV)
    ops.decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), sl.to(DEV), scale=scale,
                     workspace=ws, out=o, lse=lse)
    status = ops.get_error()
    assert guards_intact(obuf) and guards_intact(lbuf), "write outside the output tensors"
    return o, lse, status


CASES = [  # (B, Hq, Hkv, page_size, max_pages, d, lengths)
    (3, 8, 2, 16, 20, 128, [0, 1, 320]),
    (4, 8, 8, 32, 32, 128, [255, 256, 257, 1023]),   # MHA, chunk edges
    (3, 8, 1, 48, 11, 64, [48, 49, 528]),            # page size not a power of two; MQA
    (2, 6, 2, 64, 11, 128, [700, 63]),               # R = 3
    (2, 12, 2, 128, 5, 64, [640, 129]),              # R = 6
    (2, 16, 2, 256, 4, 128, [1024, 257]),            # R = 8
    (2, 8, 4, 512, 3, 128, [1536, 511]),
]


@pytest.mark.parametrize("B,Hq,Hkv,ps,mp,d,lengths", CASES,
                         ids=[f"b{c[0]}h{c[1]}g{c[2]}p{c[3]}x{c[4]}d{c[5]}" for c in CASES])
def test_paged_parity_and_equal_to_contiguous(B, Hq, Hkv, ps, mp, d, lengths):
    Nmax = ps * mp
    w = inputs.make_decode(B, Hq, Hkv, Nmax, d, seed=21 + ps, len_range=(1, Nmax))
    sl = torch.tensor(lengths, dtype=torch.int32)
    kp, table = scatter_to_pages(w.kcache, sl, ps, mp, B * mp + 3, seed=ps)
    vp, _ = scatter_to_pages(w.vcache, sl, ps, mp, B * mp + 3, seed=ps)
    o, lse, status = run_paged(w.q, kp, vp, table, sl, w.scale)
    assert status == ops.FA_OK
    ro, rl = oracle.decode_paged(w.q, kp, vp, table, sl, w.scale)
    compare(o, lse, ro, rl, f"paged {ps}")
    oc, lc = ops.decode(w.q.to(DEV), w.kcache.to(DEV), w.vcache.to(DEV), sl.to(DEV), scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o, oc) and torch.equal(lse, lc)


def test_workload9_full():
    w = inputs.workload(9)
    o, lse, status = run_paged(w.q, w.kpages, w.vpages, w.block_table, w.seqlens, w.scale)
    assert status == ops.FA_OK
    ro, rl = oracle.decode_paged(w.q, w.kpages, w.vpages, w.block_table, w.seqlens, w.scale)
    compare(o, lse, ro, rl, "workload 9")


def test_bad_block_table_entry_is_reported():
    # an entry outside the pool is caught by the kernel's own range check: reported, and
    # that page's keys read as zeros; the other sequences are unaffected
    w = inputs.make_paged_decode(3, 8, 2, 64, 4, 128, seed=5, len_range=(100, 256))
    table = w.block_table.clone()
    table[1, 0] = w.kpages.shape[0] + 7
    table[2, 1] = -3
    o, lse, status = run_paged(w.q, w.kpages, w.vpages, table, w.seqlens, w.scale)
    assert status == ops.FA_ERR_DEVICE_ARG
    ro, rl = oracle.decode_paged(w.q, w.kpages, w.vpages, w.block_table, w.seqlens, w.scale)
    compare(o[:1], lse[:1], ro[:1], rl[:1], "unaffected sequence")
    assert ops.get_error() == ops.FA_OK


def test_paged_seqlen_out_of_range_is_clamped_and_reported():
    w = inputs.make_paged_decode(2, 4, 2, 16, 4, 64, seed=6, len_range=(64, 64))
    sl = torch.tensor([65, -1], dtype=torch.int32)
    o, lse, status = run_paged(w.q, w.kpages, w.vpages, w.block_table, sl, w.scale)
    assert status == ops.FA_ERR_DEVICE_ARG
    ro, rl = oracle.decode_paged(w.q, w.kpages, w.vpages, w.block_table,
                                 torch.tensor([64, 0], dtype=torch.int32), w.scale)
    compare(o, lse, ro, rl, "clamped")


def test_paged_many_sequences():
    # more than 32 sequences, some empty, pages scattered over the pool
    w = inputs.make_paged_decode(90, 8, 2, 32, 20, 128, seed=15, len_range=(0, 640))
    o, lse, status = run_paged(w.q, w.kpages, w.vpages, w.block_table, w.seqlens, w.scale)
    assert status == ops.FA_OK
    ro, rl = oracle.decode_paged(w.q, w.kpages, w.vpages, w.block_table, w.seqlens, w.scale)
    compare(o, lse, ro, rl, "paged many sequences")
