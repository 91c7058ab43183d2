"""The C ABI on the host: libfa.so builds, loads, exports every symbol include/fa.h declares,
and rejects bad arguments synchronously (nothing here touches a GPU: every call below has
an argument that the library refuses before it looks for a device)."""
import os
import re

import pytest

from exact_io_aware_81_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.load()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "fa.h")).read()
    return set(re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", src))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    assert {"fa_fwd", "fa_fwd_ex", "fa_decode", "fa_decode_workspace_size", "fa_get_error",
            "fa_status_str"} <= syms
    assert syms == set(ops.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.fa_version() == 10000


def test_status_strings(lib):
    names = {0: "FA_OK", 1: "FA_ERR_INVALID", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_WORKSPACE",
             4: "FA_ERR_CUDA", 5: "FA_ERR_TIMEOUT", 6: "FA_ERR_DEVICE_ARG"}
    for k, v in names.items():
        assert lib.fa_status_str(k).decode() == v
    assert lib.fa_status_str(99).decode() == "FA_ERR_UNKNOWN"


FAKE = 0x10000  # 16-byte aligned, never dereferenced: each call below fails validation first


def _fwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, Nq=8, Nk=8, d=64,
             scale=0.125, causal=0, dt=0)
    a.update(kw)
    return lib.fa_fwd_ex(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                         a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"], a["dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), ops.FA_ERR_INVALID),
    (dict(lse=None), ops.FA_ERR_INVALID),
    (dict(B=0), ops.FA_ERR_INVALID),
    (dict(Nq=-1), ops.FA_ERR_INVALID),
    (dict(Hq=6, Hkv=4), ops.FA_ERR_INVALID),          # H must be a multiple of G
    (dict(causal=1, Nq=9, Nk=8), ops.FA_ERR_INVALID),  # causal needs Nq <= Nk
    (dict(scale=0.0), ops.FA_ERR_INVALID),
    (dict(scale=float("inf")), ops.FA_ERR_INVALID),
    (dict(scale=float("nan")), ops.FA_ERR_INVALID),
    (dict(dt=7), ops.FA_ERR_INVALID),
    (dict(d=96), ops.FA_ERR_UNSUPPORTED),
    (dict(d=256), ops.FA_ERR_UNSUPPORTED),
    (dict(q=FAKE + 8), ops.FA_ERR_UNSUPPORTED),        # TMA needs 16-byte alignment
    (dict(o=FAKE + 2), ops.FA_ERR_UNSUPPORTED),
])
def test_fwd_rejects(lib, kw, status):
    assert _fwd(lib, **kw) == status
    assert lib.fa_last_error_message().decode() != ""


def _dec(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, sl=FAKE, o=FAKE, lse=None, B=2, Hq=8, Hkv=2, Nmax=300, d=128,
             scale=0.1, ws=FAKE, wsb=None)
    a.update(kw)
    if a["wsb"] is None:
        a["wsb"] = lib.fa_decode_workspace_size(a["B"], a["Hq"], a["Nmax"], a["d"])
    return lib.fa_decode(a["q"], a["kc"], a["vc"], a["sl"], a["o"], a["lse"], a["B"], a["Hq"],
                         a["Hkv"], a["Nmax"], a["d"], a["scale"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(sl=None), ops.FA_ERR_INVALID),
    (dict(Hq=8, Hkv=3), ops.FA_ERR_INVALID),
    (dict(Nmax=0), ops.FA_ERR_INVALID),
    (dict(scale=-1.0), ops.FA_ERR_INVALID),
    (dict(d=80), ops.FA_ERR_UNSUPPORTED),
    (dict(kc=FAKE + 4), ops.FA_ERR_UNSUPPORTED),
    (dict(ws=None), ops.FA_ERR_WORKSPACE),
    (dict(wsb=16), ops.FA_ERR_WORKSPACE),
])
def test_decode_rejects(lib, kw, status):
    assert _dec(lib, **kw) == status


def test_decode_workspace_size(lib):
    # fp32 partial output (d values) and partial lse per (b, head, 256-key chunk), each
    # region rounded up to 256 bytes
    B, Hq, Nmax, d = 32, 32, 8192, 128
    S = 32
    want = ((B * Hq * S * d * 4 + 255) // 256) * 256 + ((B * Hq * S * 4 + 255) // 256) * 256
    assert lib.fa_decode_workspace_size(B, Hq, Nmax, d) == want
    assert lib.fa_decode_workspace_size(0, Hq, Nmax, d) == 0
    assert lib.fa_decode_workspace_size(1, 1, 1, 64) == 256 * 2


def test_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.fwd(q, q, q)


def _fwd_window(lib, window, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, Nq=8, Nk=8, d=64,
             scale=0.125, dt=0)
    a.update(kw)
    return lib.fa_fwd_window(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                             a["Nq"], a["Nk"], a["d"], a["scale"], window, a["dt"], None)


@pytest.mark.parametrize("window,kw", [
    (0, {}),                       # a window holds at least the row's own key
    (-3, {}),
    (4, dict(Nq=9, Nk=8)),         # causal (hence windowed) attention needs Nq <= Nk
    (4, dict(d=96)),
])
def test_fwd_window_rejects(lib, window, kw):
    rc = _fwd_window(lib, window, **kw)
    assert rc in (ops.FA_ERR_INVALID, ops.FA_ERR_UNSUPPORTED) and rc != ops.FA_OK
    if window <= 0 or kw.get("Nq", 0) > kw.get("Nk", 10 ** 9):
        assert rc == ops.FA_ERR_INVALID


def test_binding_window_needs_causal(lib):
    import torch
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.fwd(q, q, q, causal=False, window=4)
    with pytest.raises(ValueError):
        ops.fwd_window(q, q, q, window=0)


def _paged(lib, **kw):
    a = dict(q=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sl=FAKE, o=FAKE, lse=None, B=2, Hq=8, Hkv=2,
             num_pages=10, ps=64, mp=5, d=128, scale=0.1, ws=FAKE, wsb=None)
    a.update(kw)
    if a["wsb"] is None:
        a["wsb"] = lib.fa_decode_workspace_size(a["B"], a["Hq"], a["ps"] * a["mp"], a["d"])
    return lib.fa_decode_paged(a["q"], a["kp"], a["vp"], a["bt"], a["sl"], a["o"], a["lse"],
                               a["B"], a["Hq"], a["Hkv"], a["num_pages"], a["ps"], a["mp"], a["d"],
                               a["scale"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(bt=None), ops.FA_ERR_INVALID),
    (dict(kp=None), ops.FA_ERR_INVALID),
    (dict(num_pages=0), ops.FA_ERR_INVALID),
    (dict(ps=0), ops.FA_ERR_INVALID),
    (dict(mp=-1), ops.FA_ERR_INVALID),
    (dict(Hq=8, Hkv=3), ops.FA_ERR_INVALID),
    (dict(scale=float("nan")), ops.FA_ERR_INVALID),
    (dict(ps=40), ops.FA_ERR_UNSUPPORTED),           # pages are multiples of 16 rows
    (dict(ps=8), ops.FA_ERR_UNSUPPORTED),
    (dict(d=96), ops.FA_ERR_UNSUPPORTED),
    (dict(vp=FAKE + 8), ops.FA_ERR_UNSUPPORTED),
    (dict(ws=None), ops.FA_ERR_WORKSPACE),
    (dict(wsb=256), ops.FA_ERR_WORKSPACE),
])
def test_decode_paged_rejects(lib, kw, status):
    assert _paged(lib, **kw) == status


def _fp8(lib, **kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, ks=FAKE, vs=FAKE, sl=FAKE, o=FAKE, lse=None, B=2, Hq=8, Hkv=2,
             Nmax=300, d=128, scale=0.1, ws=FAKE, wsb=None)
    a.update(kw)
    if a["wsb"] is None:
        a["wsb"] = lib.fa_decode_workspace_size(a["B"], a["Hq"], a["Nmax"], a["d"])
    return lib.fa_decode_fp8(a["q"], a["kc"], a["vc"], a["ks"], a["vs"], a["sl"], a["o"], a["lse"],
                             a["B"], a["Hq"], a["Hkv"], a["Nmax"], a["d"], a["scale"], a["ws"],
                             a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(ks=None), ops.FA_ERR_INVALID),
    (dict(vs=None), ops.FA_ERR_INVALID),
    (dict(kc=None), ops.FA_ERR_INVALID),
    (dict(Nmax=0), ops.FA_ERR_INVALID),
    (dict(Hq=8, Hkv=3), ops.FA_ERR_INVALID),
    (dict(d=64), ops.FA_ERR_UNSUPPORTED),            # FP8 rows are one 128-byte box
    (dict(kc=FAKE + 4), ops.FA_ERR_UNSUPPORTED),
    (dict(wsb=16), ops.FA_ERR_WORKSPACE),
])
def test_decode_fp8_rejects(lib, kw, status):
    assert _fp8(lib, **kw) == status


def test_decode_paged_fp8_rejects(lib):
    rc = lib.fa_decode_paged_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, 2, 8, 2, 10,
                                 64, 5, 128, 0.1, FAKE, 1 << 20, None)
    assert rc == ops.FA_ERR_INVALID                  # no block table
    rc = lib.fa_decode_paged_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 8, 2, 10,
                                 40, 5, 128, 0.1, FAKE, 1 << 20, None)
    assert rc == ops.FA_ERR_UNSUPPORTED              # page size not a multiple of 16


@pytest.mark.parametrize("kw,status", [
    (dict(op=None), ops.FA_ERR_INVALID),
    (dict(P=0), ops.FA_ERR_INVALID),
    (dict(rows=0), ops.FA_ERR_INVALID),
    (dict(dt=3), ops.FA_ERR_INVALID),
    (dict(d=96), ops.FA_ERR_UNSUPPORTED),
])
def test_merge_lse_rejects(lib, kw, status):
    a = dict(op=FAKE, lp=FAKE, P=2, rows=4, d=128, o=FAKE, lse=None, dt=0)
    a.update(kw)
    assert lib.fa_merge_lse(a["op"], a["lp"], a["P"], a["rows"], a["d"], a["o"], a["lse"], a["dt"], None) == status


def test_decode_ex_rejects(lib):
    ws = lib.fa_decode_workspace_size(2, 8, 300, 128)
    rc = lib.fa_decode_ex(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 8, 2, 300, 128, 0.1, 7, FAKE, ws, None)
    assert rc == ops.FA_ERR_INVALID                  # unknown output dtype
    rc = lib.fa_decode_ex(FAKE, FAKE, FAKE, None, FAKE, None, 2, 8, 2, 300, 128, 0.1, 1, FAKE, ws, None)
    assert rc == ops.FA_ERR_INVALID                  # no seqlens


def _fwd_bshd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, Nq=8, Nk=8, d=64,
             scale=0.125, causal=1, window=0, dt=0)
    a.update(kw)
    return lib.fa_fwd_bshd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                           a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"], a["window"], a["dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(window=-1), ops.FA_ERR_INVALID),
    (dict(causal=0, window=4), ops.FA_ERR_INVALID),    # a window needs causal attention
    (dict(Nq=9, Nk=8), ops.FA_ERR_INVALID),
    (dict(Hq=6, Hkv=4), ops.FA_ERR_INVALID),
    (dict(dt=3), ops.FA_ERR_INVALID),
    (dict(d=96), ops.FA_ERR_UNSUPPORTED),
    (dict(k=FAKE + 8), ops.FA_ERR_UNSUPPORTED),
])
def test_fwd_bshd_rejects(lib, kw, status):
    assert _fwd_bshd(lib, **kw) == status



def _fwd_fp8(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, qs=FAKE, ks=FAKE, vs=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, Nq=8,
             Nk=8, d=128, scale=0.125, causal=1, window=0, dt=0)
    a.update(kw)
    return lib.fa_fwd_fp8(a["q"], a["k"], a["v"], a["qs"], a["ks"], a["vs"], a["o"], a["lse"], a["B"], a["Hq"],
                          a["Hkv"], a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"], a["window"], a["dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(qs=None), ops.FA_ERR_INVALID),
    (dict(ks=None), ops.FA_ERR_INVALID),
    (dict(vs=None), ops.FA_ERR_INVALID),
    (dict(q=None), ops.FA_ERR_INVALID),
    (dict(window=-2), ops.FA_ERR_INVALID),
    (dict(causal=0, window=4), ops.FA_ERR_INVALID),    # a window needs causal attention
    (dict(Nq=9, Nk=8), ops.FA_ERR_INVALID),            # causal needs Nq <= Nk
    (dict(Hq=6, Hkv=4), ops.FA_ERR_INVALID),
    (dict(dt=5), ops.FA_ERR_INVALID),
    (dict(scale=-0.5), ops.FA_ERR_INVALID),
    (dict(d=64), ops.FA_ERR_UNSUPPORTED),              # FP8 rows are one 128-byte box
    (dict(v=FAKE + 4), ops.FA_ERR_UNSUPPORTED),
])
def test_fwd_fp8_rejects(lib, kw, status):
    assert _fwd_fp8(lib, **kw) == status
    assert lib.fa_last_error_message().decode() != ""


def test_decode_selftest_timeout_rejects_one_scale(lib):
    ws = lib.fa_decode_workspace_size(2, 8, 300, 128)
    rc = lib.fa_decode_selftest_timeout(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, 2, 8, 2, 300, 128, 0.1,
                                        FAKE, ws, None)
    assert rc == ops.FA_ERR_INVALID
