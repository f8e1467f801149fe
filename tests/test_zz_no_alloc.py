"""fa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers can neither call cudaMalloc nor give the library a workspace --
a plugin whose host framework owns all device memory, or a serving loop that
must not allocate while it runs.  fa_decode_noalloc keeps the split partials
in a fixed array inside libfa.so instead.  These tests call it through the C
ABI and check that it returns what the workspace-based pair
fa_decode_splitkv + fa_combine returns, on two calls in a row (the second
call must not see the first call's leftovers), that repeated calls leave the
device's free memory unchanged, and that it refuses work that does not fit
the fixed array.  This file is collected last on purpose.

Both paths run the same split and merge kernels with the same split count, so
their results are compared bit for bit (torch.equal), not within a tolerance.
"""
import os
import re

import pytest
import torch

from io_aware_exact_flashattention_b200 import build as fabuild
from io_aware_exact_flashattention_b200 import fa
from io_aware_exact_flashattention_b200.inputs import decode_inputs

pytestmark = pytest.mark.gpu


def scratch_bytes():
    """FA_DECODE_NOALLOC_BYTES as include/fa.h defines it."""
    text = open(os.path.join(fabuild.INCLUDE, "fa.h")).read()
    m = re.search(r"#define\s+FA_DECODE_NOALLOC_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m, "FA_DECODE_NOALLOC_BYTES not found in fa.h"
    return int(m.group(1)) << int(m.group(2))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.lib()


def noalloc(q, kc, vc, sl, n, scale):
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = kc.shape
    o = torch.empty((B, Hq, d), device="cuda", dtype=torch.bfloat16)
    lse = torch.empty((B, Hq), device="cuda", dtype=torch.float32)
    st = fa.lib().fa_decode_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sl.data_ptr(),
                                    o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Lmax, d, n,
                                    float(scale), None)
    assert st == 0, fa.status_string(st)
    return o, lse


def with_workspace(q, kc, vc, sl, n, scale):
    B, Hq, d = q.shape
    op = torch.empty((B, Hq, n, d), device="cuda", dtype=torch.float32)
    lp = torch.empty((B, Hq, n), device="cuda", dtype=torch.float32)
    fa.fa_decode_splitkv(q, kc, vc, sl, op, lp, scale)
    o = torch.empty((B, Hq, d), device="cuda", dtype=torch.bfloat16)
    lse = torch.empty((B, Hq), device="cuda", dtype=torch.float32)
    fa.fa_combine(op, lp, o, lse)
    return o, lse


def assert_same(got, want):
    o, lse = got
    o_ref, lse_ref = want
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert torch.equal(o, o_ref), "O differs from the workspace path"
    assert torch.equal(lse, lse_ref), "LSE differs from the workspace path"


def test_two_calls_in_a_row_match_workspace_path():
    # first call: 16 splits over long sequences fills much of the array
    q1, k1, v1, s1 = decode_inputs(8, 32, 8, 2000, 6000, 128, seed=41, device="cuda")
    ref1 = with_workspace(q1, k1, v1, s1, 16, 0.088)
    got1 = noalloc(q1, k1, v1, s1, 16, 0.088)
    assert_same(got1, ref1)
    # second call, right after: other shapes and split count, including a
    # sequence of length 0 whose chunks are all empty
    q2, k2, v2, s2 = decode_inputs(5, 16, 4, 1, 900, 64, seed=42, device="cuda")
    s2[2] = 0
    ref2 = with_workspace(q2, k2, v2, s2, 5, 0.125)
    got2 = noalloc(q2, k2, v2, s2, 5, 0.125)
    assert_same(got2, ref2)
    assert torch.isneginf(got2[1][2]).all() and (got2[0][2] == 0).all()


def test_repeated_calls_leave_free_device_memory_unchanged():
    """The property the call exists for: after a first call (which looks up
    the array's address), further calls take no device memory."""
    q, kc, vc, sl = decode_inputs(4, 16, 4, 500, 3000, 128, seed=43, device="cuda")
    o = torch.empty((4, 16, 128), device="cuda", dtype=torch.bfloat16)
    lse = torch.empty((4, 16), device="cuda", dtype=torch.float32)

    def call():
        st = fa.lib().fa_decode_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                        sl.data_ptr(), o.data_ptr(), lse.data_ptr(), 4, 16, 4,
                                        3000, 128, 8, 0.09, None)
        assert st == 0, fa.status_string(st)
    call()
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        call()
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before


def test_rejects_work_larger_than_the_array():
    B, Hq, d = 64, 32, 128
    n = 64  # B*Hq*n*d*4 = 64 MiB > 32 MiB
    assert B * Hq * n * d * 4 > scratch_bytes()
    st = fa.lib().fa_decode_noalloc(256, 256, 256, 256, 256, 256, B, Hq, 8, 16384, d, n, 0.1,
                                    None)
    assert st == 2  # FA_ERR_UNSUPPORTED, before any CUDA call
