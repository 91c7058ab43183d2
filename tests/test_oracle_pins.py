"""Pins for the CPU oracle, checked against facts that do not come from the oracle itself.

Each pin names what fixes it: a closed form of the softmax, a property stated on the
pages, a library routine (torch's fp64 CPU scaled_dot_product_attention), hand-expanded
arithmetic on tiny inputs, or a fixture under tests/golden/.  A mutation test at the end
plants plausible mistakes in a copy of the oracle's C source and checks that the pins
catch every one of them.
"""
import math
import os
import re
import shutil
import subprocess
import tempfile

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle.online import online_attention
from oracle.split_kv import split_kv_decode
from exact_io_aware_81_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return x.to(torch.bfloat16)


def _rand(shape, seed, std=1.0):
    g = torch.Generator("cpu").manual_seed(seed)
    return _bf16(torch.randn(shape, generator=g) * std)


def _sdpa_ref(q, k, v, scale, causal, window=0):
    """torch CPU fp64 SDPA with a bottom-right causal mask (optionally banded to the W most
    recent keys) and GQA expansion."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    R = Hq // Hkv
    qd = q.double()
    kd = k.double().repeat_interleave(R, dim=1)
    vd = v.double().repeat_interleave(R, dim=1)
    mask = None
    if causal:
        i = torch.arange(Nq).view(-1, 1)
        j = torch.arange(Nk).view(1, -1)
        mask = j <= i + (Nk - Nq)
        if window:
            mask = mask & (j > i + (Nk - Nq) - window)
    o = F.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask, scale=scale)
    s = torch.matmul(qd, kd.transpose(-1, -2)) * scale
    if mask is not None:
        s = s.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return o, lse


# --------------------------------------------------------------------------- pins

def pin_probs_rows_sum_to_one():
    q = _rand((1, 2, 9, 16), 1)
    k = _rand((1, 2, 13, 16), 2)
    for causal in (False, True):
        p = oracle.probs(q, k, 0.25, causal)
        assert torch.allclose(p.sum(-1), torch.ones(1, 2, 9, dtype=torch.float64), atol=1e-12, rtol=0)
        assert (p >= 0).all()
        if causal:
            i = torch.arange(9).view(-1, 1)
            j = torch.arange(13).view(1, -1)
            assert (p[..., ~(j <= i + 4)] == 0).all()


def pin_constant_v():
    q = _rand((2, 4, 37, 32), 3, 2.0)
    k = _rand((2, 2, 41, 32), 4, 2.0)
    c = _bf16(torch.linspace(-3, 3, 32))
    v = c.view(1, 1, 1, 32).expand(2, 2, 41, 32).contiguous()
    for causal in (False, True):
        o, _ = oracle.attn_fwd(q, k, v, 0.2, causal)
        assert torch.allclose(o, c.double().view(1, 1, 1, 32).expand_as(o), atol=1e-12, rtol=0)


def pin_first_causal_row():
    q = _rand((1, 3, 20, 16), 5)
    k = _rand((1, 3, 20, 16), 6)
    v = _rand((1, 3, 20, 16), 7)
    o, lse = oracle.attn_fwd(q, k, v, 0.3, True)
    assert torch.equal(o[:, :, 0, :], v[:, :, 0, :].double())
    s00 = 0.3 * (q[:, :, 0, :].double() * k[:, :, 0, :].double()).sum(-1)
    assert torch.allclose(lse[:, :, 0], s00, atol=1e-12, rtol=0)


def pin_zero_keys_mean_of_visible_values():
    Nq, Nk = 11, 17
    q = _rand((1, 2, Nq, 8), 8)
    k = torch.zeros((1, 2, Nk, 8), dtype=torch.bfloat16)
    v = _rand((1, 2, Nk, 8), 9)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, True)
    for i in range(Nq):
        n = i + (Nk - Nq) + 1
        assert torch.allclose(o[0, :, i], v[0, :, :n].double().mean(1), atol=1e-12, rtol=0)
        assert abs(lse[0, 0, i].item() - math.log(n)) < 1e-12
    o, lse = oracle.attn_fwd(q, k, v, 0.5, False)
    assert torch.allclose(o[0], v[0].double().mean(1, keepdim=True).expand(2, Nq, 8), atol=1e-12, rtol=0)
    assert torch.allclose(lse, torch.full_like(lse, math.log(Nk)), atol=1e-12, rtol=0)


def pin_key_permutation_invariance():
    q = _rand((1, 2, 7, 16), 10)
    k = _rand((1, 2, 29, 16), 11)
    v = _rand((1, 2, 29, 16), 12)
    perm = torch.randperm(29, generator=torch.Generator().manual_seed(0))
    o1, l1 = oracle.attn_fwd(q, k, v, 0.25, False)
    o2, l2 = oracle.attn_fwd(q, k[:, :, perm], v[:, :, perm], 0.25, False)
    assert torch.allclose(o1, o2, atol=1e-12, rtol=0)
    assert torch.allclose(l1, l2, atol=1e-12, rtol=0)


def pin_dominant_key():
    d = 64
    q = _rand((1, 1, 1, d), 13)
    k = _rand((1, 1, 50, d), 14)
    v = _rand((1, 1, 50, d), 15)
    k[0, 0, 23] = q[0, 0, 0] * 8  # exact in bf16 (power-of-two scaling)
    o, _ = oracle.attn_fwd(q, k, v, 1.0 / math.sqrt(d), False)
    assert torch.allclose(o[0, 0, 0], v[0, 0, 23].double(), atol=1e-9, rtol=0)


def pin_library_sdpa():
    cases = [  # (B, Hq, Hkv, Nq, Nk, d, causal)
        (2, 4, 4, 33, 33, 32, False),
        (2, 4, 4, 33, 33, 32, True),
        (1, 6, 2, 19, 45, 16, True),    # GQA, chunked-prefill shape (Nq < Nk)
        (1, 8, 1, 24, 24, 64, True),    # MQA
        (1, 3, 3, 1, 70, 128, False),
    ]
    for n, (B, Hq, Hkv, Nq, Nk, d, causal) in enumerate(cases):
        q = _rand((B, Hq, Nq, d), 100 + n)
        k = _rand((B, Hkv, Nk, d), 200 + n, 1.5)
        v = _rand((B, Hkv, Nk, d), 300 + n)
        scale = 1.0 / math.sqrt(d)
        o, lse = oracle.attn_fwd(q, k, v, scale, causal)
        ro, rl = _sdpa_ref(q, k, v, scale, causal)
        assert torch.allclose(o, ro, atol=1e-12, rtol=0), (n, (o - ro).abs().max())
        assert torch.allclose(lse, rl, atol=1e-12, rtol=0), n


def pin_brute_force_tiny():
    # Nq = 2, Nk = 3, d = 2, one head; every entry expanded by hand with math.exp.
    qv = [[1.0, -0.5], [0.25, 2.0]]
    kv = [[0.5, 1.0], [-1.0, 0.75], [2.0, -0.25]]
    vv = [[1.0, 2.0], [-3.0, 0.5], [0.125, -1.0]]
    scale = 0.7
    q = torch.tensor(qv, dtype=torch.bfloat16).view(1, 1, 2, 2)
    k = torch.tensor(kv, dtype=torch.bfloat16).view(1, 1, 3, 2)
    v = torch.tensor(vv, dtype=torch.bfloat16).view(1, 1, 3, 2)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, scale, causal)
        for i in range(2):
            nvis = 3 if not causal else i + 2  # bottom-right: row 0 sees keys 0,1; row 1 all
            s = [scale * (qv[i][0] * kv[j][0] + qv[i][1] * kv[j][1]) for j in range(nvis)]
            e = [math.exp(x) for x in s]
            z = sum(e)
            for t in range(2):
                want = sum(e[j] * vv[j][t] for j in range(nvis)) / z
                assert abs(o[0, 0, i, t].item() - want) < 1e-12
            assert abs(lse[0, 0, i].item() - math.log(z)) < 1e-12


def pin_gqa_equals_mha_after_repeat_interleave():
    q = _rand((2, 8, 21, 32), 16)
    k = _rand((2, 2, 30, 32), 17)
    v = _rand((2, 2, 30, 32), 18)
    for causal in (False, True):
        o1, l1 = oracle.attn_fwd(q, k, v, 0.2, causal)
        o2, l2 = oracle.attn_fwd(q, k.repeat_interleave(4, 1).contiguous(),
                                 v.repeat_interleave(4, 1).contiguous(), 0.2, causal)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def pin_gqa_head_map_golden():
    table = [tuple(map(int, ln.split())) for ln in open(os.path.join(GOLDEN, "gqa_head_map.txt"))
             if ln.strip() and not ln.startswith("#")]
    Hq, Hkv = 32, 8
    q = _rand((1, Hq, 5, 16), 19)
    k = _rand((1, Hkv, 9, 16), 20)
    v = torch.zeros((1, Hkv, 9, 16), dtype=torch.bfloat16)
    for g in range(Hkv):
        v[0, g] = float(g + 1)
    o, _ = oracle.attn_fwd(q, k, v, 0.25, True)
    for h, g in table:
        assert torch.allclose(o[0, h], torch.full((5, 16), float(g + 1), dtype=torch.float64),
                              atol=1e-12, rtol=0), (h, g)


def pin_causal_block_rule_golden():
    rules = [ln.split() for ln in open(os.path.join(GOLDEN, "causal_block_rule.txt"))
             if ln.strip() and not ln.startswith("#")]
    T = 5  # block edge
    N = 4 * T
    q = _rand((1, 1, N, 8), 21)
    k = _rand((1, 1, N, 8), 22)
    p = oracle.probs(q, k, 0.5, True)[0, 0]
    for i, j, rule in rules:
        i, j = int(i), int(j)
        blk = p[i * T:(i + 1) * T, j * T:(j + 1) * T] != 0
        if rule == "skip":
            assert not blk.any()
        elif rule == "full":
            assert blk.all()
        else:
            assert torch.equal(blk, torch.ones(T, T, dtype=torch.bool).tril())


def pin_online_equals_two_pass():
    q = _rand((1, 1, 45, 16), 23, 2.0)
    k = _rand((1, 1, 70, 16), 24, 2.0)
    v = _rand((1, 1, 70, 16), 25)
    for causal in (False, True):
        qq = q[0, 0, 25:] if causal else q[0, 0]      # causal needs Nq <= Nk
        qt = qq.view(1, 1, *qq.shape)
        o, lse = oracle.attn_fwd(qt, k, v, 0.3, causal)
        for bq, bk, lazy in [(1, 1, None), (3, 3, None), (64, 64, None), (4, 7, 8 * math.log(2)),
                             (16, 5, None)]:
            oo, ll = online_attention(qq.double().numpy(), k[0, 0].double().numpy(),
                                      v[0, 0].double().numpy(), 0.3, causal, bq, bk, lazy)
            assert np.allclose(oo, o[0, 0].numpy(), atol=1e-12, rtol=0), (bq, bk, causal)
            assert np.allclose(ll, lse[0, 0].numpy(), atol=1e-12, rtol=0)


def pin_decode_matches_library_and_split_merge():
    B, Hq, Hkv, Nmax, d = 3, 8, 2, 300, 32
    w = inputs.make_decode(B, Hq, Hkv, Nmax, d, seed=7, len_range=(0, Nmax))
    sl = torch.tensor([0, 1, 300], dtype=torch.int32)
    o, lse = oracle.decode(w.q, w.kcache, w.vcache, sl, w.scale)
    assert (o[0] == 0).all() and torch.isinf(lse[0]).all() and (lse[0] < 0).all()
    for b in (1, 2):
        L = int(sl[b])
        ro, rl = _sdpa_ref(w.q[b:b + 1].unsqueeze(2), w.kcache[b:b + 1, :, :L].contiguous(),
                           w.vcache[b:b + 1, :, :L].contiguous(), w.scale, False)
        assert torch.allclose(o[b], ro[0, :, 0], atol=1e-12, rtol=0)
        assert torch.allclose(lse[b], rl[0, :, 0], atol=1e-12, rtol=0)
    for chunk in (1, 7, 64, 256, 300):
        so, sll = split_kv_decode(w.q.double().numpy(), w.kcache.double().numpy(),
                                  w.vcache.double().numpy(), sl.numpy(), w.scale, chunk)
        assert np.allclose(so, o.numpy(), atol=1e-12, rtol=0), chunk
        assert np.allclose(sll[1:], lse[1:].numpy(), atol=1e-12, rtol=0)
        assert np.isneginf(sll[0]).all()


def pin_row_sample_matches_full():
    q = _rand((2, 4, 300, 64), 26)
    k = _rand((2, 2, 300, 64), 27)
    v = _rand((2, 2, 300, 64), 28)
    rows = inputs.sample_rows(300, 20, seed=3)
    o, l = oracle.attn_fwd(q, k, v, 0.125, True)
    os_, ls = oracle.attn_fwd(q, k, v, 0.125, True, rows=rows)
    assert torch.equal(o[:, :, rows.long()], os_) and torch.equal(l[:, :, rows.long()], ls)


def pin_sliding_window_golden():
    """The page's W = 3 example: exactly the listed keys get weight, and they sum to one."""
    rows = [list(map(int, ln.split())) for ln in open(os.path.join(GOLDEN, "sliding_window_w3.txt"))
            if ln.strip() and not ln.startswith("#")]
    N = 8
    q = _rand((1, 1, N, 8), 40)
    k = _rand((1, 1, N, 8), 41)
    p = oracle.probs(q, k, 0.5, True, window=3)[0, 0]
    for row in rows:
        i, keys = row[0], row[1:]
        assert torch.nonzero(p[i]).flatten().tolist() == keys, (i, keys)
        assert abs(p[i].sum().item() - 1.0) < 1e-12


def pin_sliding_window_library_sdpa():
    """Band-masked torch fp64 SDPA, square and chunked (Nq < Nk), MHA and GQA."""
    for (Hq, Hkv, Nq, Nk, W, seed) in [(2, 2, 37, 37, 5, 42), (4, 2, 23, 61, 9, 45),
                                       (4, 1, 50, 50, 1, 48), (2, 1, 17, 40, 64, 51)]:
        q = _rand((2, Hq, Nq, 16), seed)
        k = _rand((2, Hkv, Nk, 16), seed + 1)
        v = _rand((2, Hkv, Nk, 16), seed + 2)
        o, lse = oracle.attn_fwd(q, k, v, 0.3, True, window=W)
        ro, rl = _sdpa_ref(q, k, v, 0.3, True, window=W)
        assert torch.allclose(o, ro, atol=1e-12, rtol=0), (Hq, Hkv, Nq, Nk, W)
        assert torch.allclose(lse, rl, atol=1e-12, rtol=0), (Hq, Hkv, Nq, Nk, W)


def pin_window_special_cases():
    """W >= Nk is plain causal; W = 1 picks the diagonal key: o_i = v[i + Nk - Nq] and
    lse_i = scale * q_i . k_(i + Nk - Nq), by hand."""
    Nq, Nk, d = 9, 14, 8
    q = _rand((1, 2, Nq, d), 54)
    k = _rand((1, 1, Nk, d), 55)
    v = _rand((1, 1, Nk, d), 56)
    oc, lc = oracle.attn_fwd(q, k, v, 0.7, True)
    ow, lw = oracle.attn_fwd(q, k, v, 0.7, True, window=Nk)
    assert torch.equal(oc, ow) and torch.equal(lc, lw)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.7, True, window=1)
    for h in range(2):
        for i in range(Nq):
            j = i + Nk - Nq
            assert torch.equal(o1[0, h, i], v[0, 0, j].double())
            dot = sum(float(q[0, h, i, t]) * float(k[0, 0, j, t]) for t in range(d))
            assert abs(l1[0, h, i].item() - 0.7 * dot) < 1e-12


def _scatter_to_pages(kc, seqlens, page_size, max_pages, num_pages, seed):
    """Scatter a contiguous cache (B,Hkv,Nmax,d) into a page pool in a random page order;
    returns (pool, block_table).  Plain indexing only."""
    B, Hkv, Nmax, d = kc.shape
    g = torch.Generator("cpu").manual_seed(seed)
    perm = torch.randperm(num_pages, generator=g)
    pool = torch.zeros((num_pages, Hkv, page_size, d), dtype=kc.dtype)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    used = 0
    for b in range(B):
        for t in range(-(-int(seqlens[b]) // page_size)):
            pg = int(perm[used]); used += 1
            table[b, t] = pg
            rows = kc[b, :, t * page_size:(t + 1) * page_size]
            pool[pg, :, :rows.shape[1]] = rows
    return pool, table


def pin_paged_decode_equals_contiguous():
    """A cache scattered over pages in random order decodes exactly as the contiguous
    cache, and as torch fp64 SDPA on the keys gathered back by plain indexing."""
    B, Hq, Hkv, d = 4, 8, 2, 32
    for page_size, max_pages in [(16, 20), (48, 7), (1, 300)]:
        Nmax = page_size * max_pages
        w = inputs.make_decode(B, Hq, Hkv, Nmax, d, seed=60 + page_size, len_range=(0, Nmax))
        sl = torch.tensor([0, 1, Nmax, Nmax // 2 + 3], dtype=torch.int32)
        num_pages = B * max_pages + 5
        kp, table = _scatter_to_pages(w.kcache, sl, page_size, max_pages, num_pages, 70)
        vp, table2 = _scatter_to_pages(w.vcache, sl, page_size, max_pages, num_pages, 70)
        assert torch.equal(table, table2)
        o, lse = oracle.decode_paged(w.q, kp, vp, table, sl, w.scale)
        oc, lc = oracle.decode(w.q, w.kcache, w.vcache, sl, w.scale)
        assert torch.equal(o, oc) and torch.equal(lse, lc), page_size
        for b in range(1, B):
            L = int(sl[b])
            idx = torch.arange(L)
            pages = table[b, idx // page_size].long()
            kg = kp[pages, :, idx % page_size].permute(1, 0, 2).unsqueeze(0)
            vg = vp[pages, :, idx % page_size].permute(1, 0, 2).unsqueeze(0)
            ro, rl = _sdpa_ref(w.q[b:b + 1].unsqueeze(2), kg.contiguous(), vg.contiguous(), w.scale, False)
            assert torch.allclose(o[b], ro[0, :, 0], atol=1e-12, rtol=0)
            assert torch.allclose(lse[b], rl[0, :, 0], atol=1e-12, rtol=0)


def pin_paged_generator_tables_are_valid():
    """The seeded paged workloads: every used page is distinct and in range; unused -1."""
    w = inputs.make_paged_decode(5, 4, 2, 16, 9, 16, seed=3, len_range=(0, 144))
    B, Hq, Hkv, num_pages, ps, mp, d = w.shape
    used = []
    for b in range(B):
        n = -(-int(w.seqlens[b]) // ps)
        assert (w.block_table[b, n:] == -1).all()
        used += w.block_table[b, :n].tolist()
    assert len(set(used)) == len(used) and all(0 <= u < num_pages for u in used)


def pin_e4m3_decoding():
    """E4M3 bytes by hand from the format (bias 7, subnormals m/8 * 2^-6, S.1111.111 NaN,
    max 448), and all 256 against torch's float8_e4m3fn conversion."""
    by_hand = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
               0x3F: 1.875, 0x40: 2.0, 0x41: 2.25, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0,
               0x30: 0.5, 0x58: 16.0}
    for x, want in by_hand.items():
        assert oracle.e4m3_to_double(x) == want, hex(x)
    assert math.isnan(oracle.e4m3_to_double(0x7F)) and math.isnan(oracle.e4m3_to_double(0xFF))
    assert math.copysign(1.0, oracle.e4m3_to_double(0x80)) == -1.0
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double()
    for x in range(256):
        a, b = oracle.e4m3_to_double(x), lib[x].item()
        assert (math.isnan(a) and math.isnan(b)) or a == b, hex(x)


def _dequant(bytes_u8, scales):
    return bytes_u8.view(torch.float8_e4m3fn).double() * scales.double().view(1, -1, 1, 1)


def pin_fp8_decode_equals_bf16_decode_with_power_of_two_scales():
    """With power-of-two scales every dequantized value is exactly a bf16, so the FP8
    decode must equal the bf16 decode of the dequantized cache bit for bit."""
    w = inputs.make_fp8_decode(3, 8, 2, 300, 32, seed=80, len_range=(0, 300))
    sl = torch.tensor([0, 1, 300], dtype=torch.int32)
    ks = torch.tensor([0.125, 4.0], dtype=torch.float32)
    vs = torch.tensor([2.0, 0.0625], dtype=torch.float32)
    o, lse = oracle.decode_fp8(w.q, w.kcache, w.vcache, ks, vs, sl, w.scale)
    kb = _dequant(w.kcache, ks).to(torch.bfloat16)
    vb = _dequant(w.vcache, vs).to(torch.bfloat16)
    assert torch.equal(kb.double(), _dequant(w.kcache, ks))
    ob, lb = oracle.decode(w.q, kb, vb, sl, w.scale)
    assert torch.equal(o, ob) and torch.equal(lse, lb)


def pin_fp8_decode_library_sdpa():
    """Arbitrary per-head scales: torch fp64 SDPA on the dequantized cache."""
    w = inputs.make_fp8_decode(2, 8, 4, 200, 64, seed=81, len_range=(1, 200))
    o, lse = oracle.decode_fp8(w.q, w.kcache, w.vcache, w.k_scale, w.v_scale, w.seqlens, w.scale)
    assert not torch.equal(w.k_scale, w.v_scale)
    kd, vd = _dequant(w.kcache, w.k_scale), _dequant(w.vcache, w.v_scale)
    for b in range(2):
        L = int(w.seqlens[b])
        q = w.q[b:b + 1].unsqueeze(2).double()
        kk = kd[b:b + 1, :, :L].repeat_interleave(2, dim=1)
        vv = vd[b:b + 1, :, :L].repeat_interleave(2, dim=1)
        ro = F.scaled_dot_product_attention(q, kk, vv, scale=w.scale)
        rl = torch.logsumexp(torch.matmul(q, kk.transpose(-1, -2)) * w.scale, dim=-1)
        assert torch.allclose(o[b], ro[0, :, 0], atol=1e-12, rtol=0)
        assert torch.allclose(lse[b], rl[0, :, 0], atol=1e-12, rtol=0)


def _fp8_prefill_cases():
    # (B, Hq, Hkv, Nq, Nk, d, causal, window): MHA, GQA, chunked causal, a window
    return [(1, 2, 2, 40, 40, 32, True, 0), (2, 4, 2, 33, 50, 16, True, 0),
            (1, 4, 1, 20, 20, 64, False, 0), (1, 2, 1, 30, 45, 32, True, 7)]


def pin_fp8_prefill_equals_bf16_prefill_with_power_of_two_scales():
    """With power-of-two scales every dequantized Q, K and V value is exactly a bf16, so the
    FP8 prefill must equal the bf16 prefill of the dequantized tensors bit for bit."""
    for n, (B, Hq, Hkv, Nq, Nk, d, causal, W) in enumerate(_fp8_prefill_cases()):
        w = inputs.make_fp8_prefill(B, Hq, Hkv, Nq, Nk, d, seed=82 + n, causal=causal, window=W)
        qs = torch.tensor([2.0 ** (e % 5 - 2) for e in range(Hq)], dtype=torch.float32)
        ks = torch.tensor([2.0 ** (1 - e % 3) for e in range(Hkv)], dtype=torch.float32)
        vs = torch.tensor([2.0 ** (e % 4 - 3) for e in range(Hkv)], dtype=torch.float32)
        qb, kb, vb = (_dequant(t, sc).to(torch.bfloat16) for t, sc in ((w.q, qs), (w.k, ks), (w.v, vs)))
        assert torch.equal(qb.double(), _dequant(w.q, qs))
        rows = torch.tensor([0, Nq // 2, Nq - 1], dtype=torch.int32)
        for r in (None, rows):
            o, lse = oracle.attn_fwd_fp8(w.q, w.k, w.v, qs, ks, vs, w.scale, causal, rows=r, window=W)
            ob, lb = oracle.attn_fwd(qb, kb, vb, w.scale, causal, rows=r, window=W)
            assert torch.equal(o, ob) and torch.equal(lse, lb)


def pin_fp8_prefill_library_sdpa():
    """Arbitrary per-head scales (distinct for every Q, K and V head): torch fp64 SDPA, with
    torch's own E4M3 decoding, on the dequantized tensors."""
    for n, (B, Hq, Hkv, Nq, Nk, d, causal, W) in enumerate(_fp8_prefill_cases()):
        w = inputs.make_fp8_prefill(B, Hq, Hkv, Nq, Nk, d, seed=86 + n, causal=causal, window=W)
        assert len(set(w.q_scale.tolist())) == Hq and len(set(w.k_scale.tolist() + w.v_scale.tolist())) == 2 * Hkv
        o, lse = oracle.attn_fwd_fp8(w.q, w.k, w.v, w.q_scale, w.k_scale, w.v_scale, w.scale, causal, window=W)
        ro, rl = _sdpa_ref(_dequant(w.q, w.q_scale), _dequant(w.k, w.k_scale), _dequant(w.v, w.v_scale),
                           w.scale, causal, window=W)
        assert torch.allclose(o, ro, atol=1e-12, rtol=0)
        assert torch.allclose(lse, rl, atol=1e-12, rtol=0)


def pin_context_parallel_merge_equals_unsplit():
    """The cache cut into R contiguous shards (some empty for short sequences), each decoded
    on its own by the C oracle and merged by merge_lse, equals the unsplit decode."""
    from oracle.split_kv import merge_lse
    B, Hq, Hkv, Nmax, d = 4, 8, 2, 400, 32
    w = inputs.make_decode(B, Hq, Hkv, Nmax, d, seed=90, len_range=(0, Nmax))
    sl = torch.tensor([0, 57, 400, 250], dtype=torch.int32)
    full_o, full_l = oracle.decode(w.q, w.kcache, w.vcache, sl, w.scale)
    for R in (1, 2, 3, 4):
        C = -(-Nmax // R)
        parts_o, parts_l = [], []
        for r in range(R):
            kc = w.kcache[:, :, r * C:(r + 1) * C].contiguous()
            vc = w.vcache[:, :, r * C:(r + 1) * C].contiguous()
            slr = (sl - r * C).clamp(0, kc.shape[2]).to(torch.int32)
            o, l = oracle.decode(w.q, kc, vc, slr, w.scale)
            parts_o.append(o.numpy()); parts_l.append(l.numpy())
        mo, ml = merge_lse(np.stack(parts_o), np.stack(parts_l))
        assert np.allclose(mo, full_o.numpy(), atol=1e-12, rtol=0), R
        fin = np.isfinite(full_l.numpy())
        assert np.allclose(ml[fin], full_l.numpy()[fin], atol=1e-12, rtol=0)
        assert np.isneginf(ml[~fin]).all() and (mo[0] == 0).all()


PINS = [v for n, v in sorted(globals().items()) if n.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__[4:])
def test_pin(pin):
    pin()


# ------------------------------------------------------------------- mutation test
# Each mutant is one plausible slip in the oracle's C source.  The pins above must fail
# on every one of them.
MUTANTS = [
    ("gqa index", "long g = h / R;\n                long i", "long g = h % Hkv;\n                long i"),
    ("causal offset dropped", "long last = i + (Nk - Nq);", "long last = i;"),
    ("causal off by one", "return last < 0 ? 0 : last + 1;", "return last < 0 ? 0 : last;"),
    ("max sign", "l += exp(s[j] - m);\n", "l += exp(s[j] + m);\n"),
    ("scale dropped", "s[j] = scale * acc;", "s[j] = acc;"),
    ("lse without max", "*lse = m + log(l);", "*lse = log(l);"),
    ("transposed k index", "const uint16_t *kr = khead + j * d;", "const uint16_t *kr = khead + j;"),
    ("normaliser dropped", "double p = exp(s[j] - m) / l;", "double p = exp(s[j] - m);"),
    ("last key dropped", "for (long j = 0; j < nkeys; ++j) {\n        double p", "for (long j = 0; j + 1 < nkeys; ++j) {\n        double p"),
    ("window off by one", "long first = i + (Nk - Nq) - window + 1;", "long first = i + (Nk - Nq) - window;"),
    ("window offset dropped", "long first = i + (Nk - Nq) - window + 1;", "long first = i - window + 1;"),
    ("paged pool layout", "const long src = ((page * Hkv + g) * page_size + row) * d;",
     "const long src = ((g * num_pages + page) * page_size + row) * d;"),
    ("paged head map", "for (long h = g * R; h < (g + 1) * R; ++h)", "for (long h = g; h < Hq; h += Hkv)"),
    ("e4m3 bias", "v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("e4m3 subnormal", "v = ldexp((double)m / 8.0, -6);", "v = ldexp((double)m / 8.0, -7);"),
    ("fp8 scales swapped", "kd[e] = (double)k_scale[g] * oracle_e4m3_to_double(kh[e]);",
     "kd[e] = (double)v_scale[g] * oracle_e4m3_to_double(kh[e]);"),
    ("fp8 normaliser dropped", "double w = exp(s[j] - mx) / sum;", "double w = exp(s[j] - mx);"),
    ("fp8 prefill q scale of the kv head", "attend_row_fp8(qrow, q_scale[h],", "attend_row_fp8(qrow, q_scale[g],"),
    ("fp8 prefill v scale dropped", "orow[t] += p * (vs * lut[vr[t]]);", "orow[t] += p * lut[vr[t]];"),
    ("fp8 prefill k scale from v", "acc += qbuf[t] * (ks * lut[kr[t]]);", "acc += qbuf[t] * (vs * lut[kr[t]]);"),
    ("fp8 prefill window dropped", "long j0 = first_key(i, Nq, Nk, window);\n                long j1 = visible_keys(i, Nq, Nk, causal);\n                attend_row_fp8",
     "long j0 = 0;\n                long j1 = visible_keys(i, Nq, Nk, causal);\n                attend_row_fp8"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new, monkeypatch):
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, name
    mutated = src.replace(old, new)
    with tempfile.TemporaryDirectory() as td:
        c = os.path.join(td, "m.c")
        so = os.path.join(td, "m.so")
        open(c, "w").write(mutated)
        subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", so, c, "-lm"])
        import ctypes
        lib = oracle.declare(ctypes.CDLL(so))
        monkeypatch.setattr(oracle, "_lib", lib)
        caught = []
        for pin in PINS:
            try:
                pin()
            except AssertionError:
                caught.append(pin.__name__)
        assert caught, f"no pin caught mutant '{name}'"
