"""Parity of the split-KV decode (fa_decode through the C ABI) with the fp64 oracle."""
import pytest
import torch

import oracle
from exact_io_aware_81_b200 import inputs, ops
from parity import compare, guarded, guards_intact

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_gpu(w: inputs.Decode, seqlens=None):
    B, Hq, Hkv, Nmax, d = w.shape
    sl = (w.seqlens if seqlens is None else seqlens).to(DEV)
    obuf, o = guarded((B, Hq, d), torch.bfloat16, DEV)
    lbuf, lse = guarded((B, Hq), torch.float32, DEV)
    ws = torch.full((ops.decode_workspace_size(B, Hq, Nmax, d),), 0xFF, dtype=torch.uint8, device=DEV)
    ops.decode(w.q.to(DEV), w.kcache.to(DEV), w.vcache.to(DEV), sl, scale=w.scale, workspace=ws,
               out=o, lse=lse)
    status = ops.get_error()
    assert guards_intact(obuf) and guards_intact(lbuf), "write outside the output tensors"
    return o, lse, status


CASES = [  # (B, Hq, Hkv, Nmax, d, lengths)
    (3, 8, 2, 300, 128, [0, 1, 300]),
    (4, 8, 8, 1000, 128, [255, 256, 257, 999]),     # MHA, chunk edges
    (2, 8, 1, 513, 64, [513, 100]),                 # MQA R=8, d=64
    (2, 6, 2, 700, 128, [700, 3]),                  # R=3
    (2, 12, 2, 600, 64, [600, 512]),                # R=6
    (1, 32, 8, 8192, 128, [8192]),                  # one full-length sequence
    (2, 8, 1, 65536, 128, [65536, 40000]),          # 256 splits per sequence into the merge
    (3, 1, 1, 900, 64, [900, 1, 450]),              # a single head
]


@pytest.mark.parametrize("B,Hq,Hkv,Nmax,d,lengths", CASES,
                         ids=[f"b{c[0]}h{c[1]}g{c[2]}n{c[3]}d{c[4]}" for c in CASES])
def test_small_parity(B, Hq, Hkv, Nmax, d, lengths):
    w = inputs.make_decode(B, Hq, Hkv, Nmax, d, seed=11 + Nmax, len_range=(1, Nmax))
    sl = torch.tensor(lengths, dtype=torch.int32)
    o, lse, status = run_gpu(w, sl)
    assert status == ops.FA_OK
    ro, rl = oracle.decode(w.q, w.kcache, w.vcache, sl, w.scale)
    compare(o, lse, ro, rl, "decode")
    for b, L in enumerate(lengths):
        if L == 0:
            assert (o[b] == 0).all() and torch.isneginf(lse[b]).all()


def test_workload5_full():
    w = inputs.workload(5)
    o, lse, status = run_gpu(w)
    assert status == ops.FA_OK
    ro, rl = oracle.decode(w.q, w.kcache, w.vcache, w.seqlens, w.scale)
    compare(o, lse, ro, rl, "workload 5")


def test_seqlen_out_of_range_is_clamped_and_reported():
    w = inputs.make_decode(2, 4, 2, 300, 128, seed=3, len_range=(1, 300))
    sl = torch.tensor([400, -5], dtype=torch.int32)
    o, lse, status = run_gpu(w, sl)
    assert status == ops.FA_ERR_DEVICE_ARG
    ro, rl = oracle.decode(w.q, w.kcache, w.vcache, torch.tensor([300, 0], dtype=torch.int32), w.scale)
    compare(o, lse, ro, rl, "clamped")
    assert ops.get_error() == ops.FA_OK  # the word was cleared


def test_lse_optional_and_workspace_reuse():
    w = inputs.make_decode(2, 8, 2, 1024, 128, seed=4, len_range=(1, 1024))
    q, kc, vc, sl = w.q.to(DEV), w.kcache.to(DEV), w.vcache.to(DEV), w.seqlens.to(DEV)
    ws = torch.empty(ops.decode_workspace_size(2, 8, 1024, 128), dtype=torch.uint8, device=DEV)
    o1, l1 = ops.decode(q, kc, vc, sl, workspace=ws)
    o2, l2 = ops.decode(q, kc, vc, sl, workspace=ws, want_lse=False)
    torch.cuda.synchronize()
    assert l2 is None
    assert torch.equal(o1, o2)


def test_many_sequences_with_empty_and_short_ones():
    # more than 32 sequences: the work-item walk steps over the lengths 32 at a time
    B = 100
    w = inputs.make_decode(B, 8, 2, 700, 128, seed=12, len_range=(0, 700))
    g = torch.Generator().manual_seed(13)
    sl = torch.randint(0, 701, (B,), generator=g).to(torch.int32)
    sl[::7] = 0
    sl[3::11] = 1
    sl[5::13] = 700
    o, lse, status = run_gpu(w, sl)
    assert status == ops.FA_OK
    ro, rl = oracle.decode(w.q, w.kcache, w.vcache, sl, w.scale)
    compare(o, lse, ro, rl, "many sequences")
