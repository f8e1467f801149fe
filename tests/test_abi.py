"""The C ABI on the CPU: libfa.so loads without a GPU, exports every function
include/fa.h declares, and rejects bad arguments before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

from io_aware_exact_flashattention_b200 import build as fabuild
from io_aware_exact_flashattention_b200 import fa

HEADER = os.path.join(fabuild.INCLUDE, "fa.h")

OK, INVALID, UNSUPPORTED, ALIGNMENT = 0, 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    fabuild.build()
    return fa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_calls():
    names = declared_functions()
    for n in ("fa_fwd", "fa_fwd_fp8", "fa_decode_splitkv", "fa_combine", "fa_status_string"):
        assert n in names
    assert set(names) == set(fa.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (fa_[a-z0-9_]+)\b", out))
    missing = set(declared_functions()) - exported
    assert not missing, "not exported: %s" % sorted(missing)


def test_status_strings(lib):
    for code in range(6):
        s = fa.status_string(code)
        assert s.startswith(fa.STATUS_NAMES[code])
    assert "unknown" in fa.status_string(99)


A = 256  # an aligned fake address (never dereferenced: checks fail first)


def fwd(lib, *, q=A, k=A, v=A, o=A, lse=A, B=1, Hq=4, Hkv=4, Sq=128, Skv=128, d=128,
        causal=0, scale=0.125):
    return lib.fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, d, causal, scale, None)


@pytest.mark.parametrize("kw,want", [
    (dict(d=96), UNSUPPORTED),
    (dict(d=256), UNSUPPORTED),
    (dict(Hq=4, Hkv=3), INVALID),
    (dict(Hq=0), INVALID),
    (dict(Hkv=0), INVALID),
    (dict(B=-1), INVALID),
    (dict(Sq=-5), INVALID),
    (dict(Skv=-1), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(scale=float("inf")), INVALID),
    (dict(scale=-0.125), UNSUPPORTED),   # the kernel follows the largest raw score
    (dict(q=None), INVALID),
    (dict(lse=None), INVALID),
    (dict(v=A + 8), ALIGNMENT),
    (dict(o=A + 2), ALIGNMENT),
    (dict(B=0, q=None, k=None), OK),   # empty batch: nothing to do
    (dict(Sq=0, q=None, o=None), OK),  # no query rows: nothing to do
])
def test_fwd_rejects_before_cuda(lib, kw, want):
    assert fwd(lib, **kw) == want


def fwd8(lib, *, q=A, k=A, v=A, dq=None, dk=None, dv=None, o=A, lse=A, B=1, Hq=4, Hkv=4,
         Sq=128, Skv=128, d=128, causal=0, scale=0.125):
    return lib.fa_fwd_fp8(q, k, v, dq, dk, dv, o, lse, B, Hq, Hkv, Sq, Skv, d, causal, scale,
                          None)


@pytest.mark.parametrize("kw,want", [
    (dict(d=64), UNSUPPORTED),          # 8-bit inputs: d = 128 only
    (dict(d=256), UNSUPPORTED),
    (dict(Hq=4, Hkv=3), INVALID),
    (dict(Hkv=0), INVALID),
    (dict(Sq=-1), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(scale=-1.0), UNSUPPORTED),
    (dict(q=None), INVALID),
    (dict(lse=None), INVALID),
    (dict(k=A + 8), ALIGNMENT),
    (dict(dq=A + 2), ALIGNMENT),        # factor arrays: 4-byte aligned
    (dict(dv=A + 1), ALIGNMENT),
    (dict(B=0, q=None), OK),
    (dict(Sq=0, q=None, o=None), OK),
])
def test_fwd_fp8_rejects_before_cuda(lib, kw, want):
    assert fwd8(lib, **kw) == want


def dec(lib, *, q=A, kc=A, vc=A, sl=A, op=A, lp=A, B=2, Hq=8, Hkv=2, Lmax=64, d=128, n=4,
        scale=0.1):
    return lib.fa_decode_splitkv(q, kc, vc, sl, op, lp, B, Hq, Hkv, Lmax, d, n, scale, None)


@pytest.mark.parametrize("kw,want", [
    (dict(d=80), UNSUPPORTED),
    (dict(Hq=24, Hkv=2), UNSUPPORTED),   # group of 12 query heads
    (dict(Hq=8, Hkv=3), INVALID),
    (dict(n=0), INVALID),
    (dict(n=257), INVALID),
    (dict(Lmax=-1), INVALID),
    (dict(scale=-0.1), UNSUPPORTED),
    (dict(sl=None), INVALID),
    (dict(op=A + 4), ALIGNMENT),
    (dict(sl=A + 2), ALIGNMENT),
    (dict(B=0, q=None), OK),
])
def test_decode_rejects_before_cuda(lib, kw, want):
    assert dec(lib, **kw) == want


def paged(lib, *, q=A, kp=A, vp=A, bt=A, sl=A, op=A, lp=A, B=2, Hq=8, Hkv=2, pages=16, P=16,
          max_pages=8, d=128, n=4, scale=0.1):
    return lib.fa_decode_paged_splitkv(q, kp, vp, bt, sl, op, lp, B, Hq, Hkv, pages, P,
                                       max_pages, d, n, scale, None)


@pytest.mark.parametrize("kw,want", [
    (dict(P=24), UNSUPPORTED),           # not a power of two
    (dict(P=8), UNSUPPORTED),            # below 16
    (dict(P=512), UNSUPPORTED),          # above 256
    (dict(d=80), UNSUPPORTED),
    (dict(Hq=24, Hkv=2), UNSUPPORTED),
    (dict(Hq=8, Hkv=3), INVALID),
    (dict(pages=0), INVALID),
    (dict(max_pages=0), INVALID),
    (dict(n=0), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(scale=-0.1), UNSUPPORTED),
    (dict(bt=None), INVALID),
    (dict(vp=None), INVALID),
    (dict(bt=A + 2), ALIGNMENT),
    (dict(kp=A + 8), ALIGNMENT),
    (dict(max_pages=1 << 24, P=256), UNSUPPORTED),  # max_pages * P beyond int32
    (dict(B=0, q=None, bt=None), OK),
])
def test_paged_decode_rejects_before_cuda(lib, kw, want):
    assert paged(lib, **kw) == want


def bwd(lib, *, q=A, k=A, v=A, o=A, lse=A, do=A, dq=A, dk=A, dv=A, ws=A, B=1, Hq=4, Hkv=2,
        Sq=128, Skv=128, d=128, causal=1, scale=0.1):
    return lib.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, B, Hq, Hkv, Sq, Skv, d, causal, scale,
                      None)


@pytest.mark.parametrize("kw,want", [
    (dict(d=96), UNSUPPORTED),
    (dict(Hq=4, Hkv=3), INVALID),
    (dict(Sq=-1), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(ws=None), INVALID),
    (dict(do=None), INVALID),
    (dict(dk=A + 8), ALIGNMENT),
    (dict(ws=A + 4), ALIGNMENT),
    (dict(B=0, q=None), OK),
])
def test_bwd_rejects_before_cuda(lib, kw, want):
    assert bwd(lib, **kw) == want


def bpt(lib, *, o=A, w1=A, w2=A, y=A, ws=A, B=1, Hq=2, S=300, d=128, F=512, chunk=2):
    return lib.fa_bpt_ffn(o, w1, w2, y, ws, B, Hq, S, d, F, chunk, None)


@pytest.mark.parametrize("kw,want", [
    (dict(d=96), UNSUPPORTED),
    (dict(Hq=1), UNSUPPORTED),           # D = 128 is not a multiple of 256
    (dict(F=300), UNSUPPORTED),
    (dict(chunk=0), INVALID),
    (dict(chunk=70000), UNSUPPORTED),
    (dict(B=-1), INVALID),
    (dict(S=-1), INVALID),
    (dict(o=None), INVALID),
    (dict(ws=None), INVALID),
    (dict(y=A + 8), ALIGNMENT),
    (dict(w2=A + 2), ALIGNMENT),
    (dict(B=0, o=None), OK),
    (dict(S=0, o=None), OK),
])
def test_bpt_ffn_rejects_before_cuda(lib, kw, want):
    assert bpt(lib, **kw) == want


def bpt_layer(lib, q=A, k=A, v=A, w1=A, w2=A, y=A, lse=A, ws=A, B=1, Hq=2, Hkv=1, S=300,
              d=128, F=512, causal=1, scale=0.1, chunk=2):
    return lib.fa_bpt_layer(q, k, v, w1, w2, y, lse, ws, B, Hq, Hkv, S, d, F, causal, scale,
                            chunk, None)


@pytest.mark.parametrize("kw,want", [
    (dict(d=96), UNSUPPORTED),
    (dict(Hq=1), UNSUPPORTED),           # D = 128 is not a multiple of 256
    (dict(F=300), UNSUPPORTED),
    (dict(Hq=4, Hkv=3), INVALID),
    (dict(chunk=0), INVALID),
    (dict(scale=-1.0), UNSUPPORTED),
    (dict(scale=float("nan")), INVALID),
    (dict(B=-1), INVALID),
    (dict(q=None), INVALID),
    (dict(lse=None), INVALID),
    (dict(ws=None), INVALID),
    (dict(y=A + 8), ALIGNMENT),
    (dict(k=A + 2), ALIGNMENT),
    (dict(B=0, q=None), OK),
    (dict(S=0, q=None), OK),
])
def test_bpt_layer_rejects_before_cuda(lib, kw, want):
    assert bpt_layer(lib, **kw) == want


def test_bpt_layer_workspace_bytes(lib):
    rows = 3 * 128
    o_bytes = 2 * 4 * rows * 64 * 2
    assert fa.bpt_layer_workspace_bytes(2, 4, 64, 512, 3) == o_bytes + 2 * rows * 512 * 2
    assert fa.bpt_layer_workspace_bytes(0, 4, 64, 512, 3) == 0


def test_bpt_workspace_bytes(lib):
    assert fa.bpt_workspace_bytes(512, 3) == 3 * 128 * 512 * 2
    assert fa.bpt_workspace_bytes(0, 3) == 0


def test_bwd_workspace_bytes(lib):
    assert fa.bwd_workspace_bytes(2, 4, 100, 128) == 2 * 4 * 1 * 256 * 4
    assert fa.bwd_workspace_bytes(2, 4, 300, 64) == 2 * 4 * 3 * 256 * 4
    assert fa.bwd_workspace_bytes(0, 4, 100, 128) == 0


@pytest.mark.parametrize("args,want", [
    ((A, A, A, A, 2, 8, 0, 128), INVALID),
    ((A, A, A, A, 2, 8, 4, 96), UNSUPPORTED),
    ((None, A, A, A, 2, 8, 4, 128), INVALID),
    ((A, A, A + 4, A, 2, 8, 4, 128), ALIGNMENT),
    ((A, A, A, A, 2, 0, 4, 128), INVALID),
])
def test_combine_rejects_before_cuda(lib, args, want):
    assert lib.fa_combine(*args, None) == want


def test_default_splits(lib):
    n = fa.decode_default_splits(64, 8, 16384, 148)
    assert 1 <= n <= 256
    assert fa.decode_default_splits(1, 1, 100, 148) >= 1
    assert fa.decode_default_splits(0, 0, 0, 0) == 1
    # small caches are not split below ~64 keys per chunk
    assert fa.decode_default_splits(1, 1, 128, 148) <= 2


def test_timeout_probe_rejects_bad_limit(lib):
    assert lib.fa_debug_timeout_probe(0, None) == INVALID
