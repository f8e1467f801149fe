"""fa_decode_splitkv + fa_combine (through the C ABI) against the fp64 oracle
on a B200.  Cache positions at or beyond a sequence's length are filled with
NaN, so any read of them would poison the output."""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_flashattention_b200 import fa
from io_aware_exact_flashattention_b200.inputs import CONFIGS, decode_inputs, decode_inputs_for

pytestmark = pytest.mark.gpu

O_TOL = 2e-2
LSE_TOL = 1e-3
# Partials are fp32, but their P.V product takes the probabilities in bf16:
# each weight carries a relative rounding error <= 2^-9, so a partial (a convex
# combination of value rows) is off by at most 2^-9 * max|v| (~0.01 for
# N(0,1) values); the same bound covers the fp32 normaliser's mismatch.
PART_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.lib()


def run_decode(q, kc, vc, sl, scale, n):
    B, Hq, d = q.shape
    op = torch.empty((B, Hq, n, d), device="cuda", dtype=torch.float32)
    lp = torch.empty((B, Hq, n), device="cuda", dtype=torch.float32)
    fa.fa_decode_splitkv(q, kc, vc, sl, op, lp, scale)
    o = torch.empty((B, Hq, d), device="cuda", dtype=torch.bfloat16)
    lse = torch.empty((B, Hq), device="cuda", dtype=torch.float32)
    fa.fa_combine(op, lp, o, lse)
    torch.cuda.synchronize()
    return op, lp, o, lse


def cmp(got, want, tol, what):
    got = np.asarray(got, dtype=np.float64)
    ninf = np.isneginf(want)
    assert (np.isneginf(got) == ninf).all(), what + ": -inf pattern differs"
    g = np.where(ninf, 0, got)
    w = np.where(ninf, 0, want)
    assert np.isfinite(g).all(), what + ": non-finite values"
    err = float(np.abs(g - w).max()) if g.size else 0.0
    assert err <= tol, "%s: max abs error %.3e > %.1e" % (what, err, tol)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (16, 4), (32, 4)])
@pytest.mark.parametrize("n", [1, 3, 16])
def test_small_decode(d, Hq, Hkv, n):
    q, kc, vc, sl = decode_inputs(3, Hq, Hkv, 1, 700, d, seed=d + Hq + n, device="cuda",
                                  pad_value=None)
    sl = torch.tensor([700, 1, 2], device="cuda", dtype=torch.int32)  # ragged, incl. L < n
    kc[1, :, 1:] = float("nan")
    vc[1, :, 1:] = float("nan")
    kc[2, :, 2:] = float("nan")
    vc[2, :, 2:] = float("nan")
    scale = 1.0 / math.sqrt(d)
    op, lp, o, lse = run_decode(q, kc, vc, sl, scale, n)
    op_ref, lp_ref = oracle.split_partials(q, kc, vc, sl, n, scale)
    cmp(op.cpu().numpy(), op_ref, PART_TOL, "o_partial")
    cmp(lp.cpu().numpy(), lp_ref, LSE_TOL, "lse_partial")
    o_ref, lse_ref = oracle.decode(q, kc, vc, sl, scale)
    cmp(o.float().cpu().numpy(), o_ref, O_TOL, "O")
    cmp(lse.cpu().numpy(), lse_ref, LSE_TOL, "LSE")


def test_zero_length_sequence():
    q, kc, vc, _ = decode_inputs(2, 8, 2, 1, 64, 128, seed=4, device="cuda", pad_value=None)
    sl = torch.tensor([0, 64], device="cuda", dtype=torch.int32)
    _, lp, o, lse = run_decode(q, kc, vc, sl, 0.1, 4)
    assert torch.isneginf(lp[0]).all() and torch.isneginf(lse[0]).all()
    assert (o[0] == 0).all()
    o_ref, lse_ref = oracle.decode(q[1:], kc[1:], vc[1:], sl[1:], 0.1)
    cmp(o[1:].float().cpu().numpy(), o_ref, O_TOL, "O")


def test_combine_alone():
    """fa_combine on random partials with empty chunks, against the oracle's
    merge."""
    g = torch.Generator().manual_seed(3)
    B, Hq, n, d = 4, 8, 7, 128
    op = torch.randn(B, Hq, n, d, generator=g)
    lp = torch.randn(B, Hq, n, generator=g) * 5
    lp[0, 0, :] = -math.inf          # a row with every chunk empty
    lp[1, :, 2] = -math.inf          # one empty chunk per row
    op[1, :, 2] = 0
    op[0, 0] = 0
    o = torch.empty(B, Hq, d, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(B, Hq, device="cuda")
    fa.fa_combine(op.cuda(), lp.cuda(), o, lse)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.combine(op, lp)
    cmp(o.float().cpu().numpy(), o_ref, O_TOL, "O")
    cmp(lse.cpu().numpy(), lse_ref, LSE_TOL, "LSE")


def test_decode_equals_prefill_row():
    """Decode of one query equals the prefill kernel with Sq = 1 (non-causal)."""
    q, kc, vc, _ = decode_inputs(2, 8, 2, 1, 640, 128, seed=8, device="cuda", pad_value=None)
    sl = torch.tensor([640, 640], device="cuda", dtype=torch.int32)
    _, _, o, lse = run_decode(q, kc, vc, sl, 0.088, 5)
    o2 = torch.empty(2, 8, 1, 128, device="cuda", dtype=torch.bfloat16)
    l2 = torch.empty(2, 8, 1, device="cuda")
    fa.fa_fwd(q[:, :, None].contiguous(), kc, vc, o2, l2, False, 0.088)
    torch.cuda.synchronize()
    assert float((o.float() - o2[:, :, 0].float()).abs().max()) <= 2 * O_TOL
    assert float((lse - l2[:, :, 0]).abs().max()) <= 2 * LSE_TOL


def test_full_size_decode_config_every_sequence():
    """The full decode workload (B=64, Hq=32, Hkv=8, L in [4096, 16384], d=128)
    in the launch the benchmark times; every sequence and head element-wise
    against the oracle (one oracle call per sequence, on its L_b keys)."""
    c = CONFIGS["decode_b64_splitkv_d128"]
    q, kc, vc, sl = decode_inputs_for(c, device="cuda")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n = fa.decode_default_splits(c.B, c.Hkv, c.Lmax, sms)
    _, _, o, lse = run_decode(q, kc, vc, sl, c.scale, n)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    lens = sl.cpu().tolist()
    for b in range(c.B):
        L = lens[b]
        o_ref, lse_ref = oracle.decode(q[b:b + 1], kc[b:b + 1, :, :L], vc[b:b + 1, :, :L],
                                       np.array([L], np.int32), c.scale)
        cmp(o[b:b + 1].float().cpu().numpy(), o_ref, O_TOL, "O b=%d" % b)
        cmp(lse[b:b + 1].cpu().numpy(), lse_ref, LSE_TOL, "LSE b=%d" % b)


def test_combine_after_partials_written_just_before():
    """fa_combine is a programmatic dependent of the kernel before it: it must
    wait for it before reading the partials.  Partials rewritten in place on
    the same stream right before the call (no synchronisation) give the
    synchronised result bit for bit."""
    g = torch.Generator().manual_seed(5)
    B, Hq, n, d = 8, 16, 9, 128
    op = torch.randn(B, Hq, n, d, generator=g).cuda()
    lp = (torch.randn(B, Hq, n, generator=g) * 5).cuda()
    o_ref = torch.empty(B, Hq, d, device="cuda", dtype=torch.bfloat16)
    lse_ref = torch.empty(B, Hq, device="cuda")
    fa.fa_combine(op, lp, o_ref, lse_ref)
    torch.cuda.synchronize()
    saved = (op.clone(), lp.clone())
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(lse_ref)
    for _ in range(3):
        op.fill_(1.0e6)
        lp.fill_(100.0)
        op.copy_(saved[0])
        lp.copy_(saved[1])
        fa.fa_combine(op, lp, o, lse)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
