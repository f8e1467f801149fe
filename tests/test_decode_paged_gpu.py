"""fa_decode_paged_splitkv + fa_combine (through the C ABI) against the fp64
oracle on a B200.  The oracle reads the paged cache through its block table
with plain index loops and decodes the gathered keys; the pool's pages are
scattered by a seeded permutation, unused rows of a last page are NaN, and
block-table entries past a sequence's pages are -1, so a read of anything a
sequence does not own would poison the output."""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_flashattention_b200 import fa
from io_aware_exact_flashattention_b200.inputs import (CONFIGS, decode_inputs,
                                                       paged_decode_inputs)

pytestmark = pytest.mark.gpu

O_TOL = 2e-2
LSE_TOL = 1e-3
PART_TOL = 1e-2  # the contiguous decode tests derive this bound (bf16 P in P.V)
CHUNK_ALIGN = 128


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.lib()


def run_paged(q, kp, vp, bt, sl, scale, n):
    B, Hq, d = q.shape
    op = torch.empty((B, Hq, n, d), device="cuda", dtype=torch.float32)
    lp = torch.empty((B, Hq, n), device="cuda", dtype=torch.float32)
    fa.fa_decode_paged_splitkv(q, kp, vp, bt, sl, op, lp, scale)
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


def to_device(*ts):
    return [t.cuda() for t in ts]


@pytest.mark.parametrize("P", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (32, 8)])
def test_paged_matches_oracle(P, d, Hq, Hkv):
    n = 5
    q, kp, vp, bt, sl = paged_decode_inputs(4, Hq, Hkv, 900, 900, d, seed=P + d + Hq,
                                            page_size=P)
    # ragged lengths: full, one key, ending on a page boundary, in mid-page
    sl = torch.tensor([900, 1, 2 * P, 517], dtype=torch.int32)
    q, kp, vp, bt, sl = _with_lengths(q, kp, vp, bt, sl, P)
    qd, kpd, vpd, btd, sld = to_device(q, kp, vp, bt, sl)
    scale = 1.0 / math.sqrt(d)
    op, lp, o, lse = run_paged(qd, kpd, vpd, btd, sld, scale, n)
    kg, vg = oracle.paged_gather(kp, vp, bt, sl)
    op_ref, lp_ref = oracle.split_partials_aligned(q, kg, vg, sl, n, CHUNK_ALIGN, scale)
    cmp(op.cpu().numpy(), op_ref, PART_TOL, "o_partial")
    cmp(lp.cpu().numpy(), lp_ref, LSE_TOL, "lse_partial")
    o_ref, lse_ref = oracle.decode_paged(q, kp, vp, bt, sl, scale)
    cmp(o.float().cpu().numpy(), o_ref, O_TOL, "O")
    cmp(lse.cpu().numpy(), lse_ref, LSE_TOL, "LSE")


def _with_lengths(q, kp, vp, bt, sl, P):
    """Shorten sequences to the lengths in sl (never lengthen past the pages
    they own): rows past the new length become NaN and table entries past
    the new last page become -1."""
    kp, vp, bt = kp.clone(), vp.clone(), bt.clone()
    for b in range(bt.shape[0]):
        L = int(sl[b])
        owned = int((bt[b] >= 0).sum()) * P
        assert L <= owned, "test asks for more keys than the sequence's pages hold"
        for j in range(bt.shape[1]):
            page = int(bt[b, j])
            if page < 0:
                continue
            lo = j * P
            if lo >= L:
                kp[page] = float("nan")
                vp[page] = float("nan")
                bt[b, j] = -1
            elif lo + P > L:
                kp[page, :, L - lo:] = float("nan")
                vp[page, :, L - lo:] = float("nan")
    return q, kp, vp, bt, sl


def test_many_splits_give_empty_chunks():
    q, kp, vp, bt, sl = paged_decode_inputs(2, 16, 4, 100, 400, 128, seed=31, page_size=16)
    qd, kpd, vpd, btd, sld = to_device(q, kp, vp, bt, sl)
    op, lp, o, lse = run_paged(qd, kpd, vpd, btd, sld, 0.1, 16)  # 16 chunks of >= 128 keys
    kg, vg = oracle.paged_gather(kp, vp, bt, sl)
    op_ref, lp_ref = oracle.split_partials_aligned(q, kg, vg, sl, 16, CHUNK_ALIGN, 0.1)
    assert np.isneginf(lp_ref).any(), "the case must contain empty chunks"
    cmp(lp.cpu().numpy(), lp_ref, LSE_TOL, "lse_partial")
    cmp(op.cpu().numpy(), op_ref, PART_TOL, "o_partial")
    o_ref, lse_ref = oracle.decode_paged(q, kp, vp, bt, sl, 0.1)
    cmp(o.float().cpu().numpy(), o_ref, O_TOL, "O")
    cmp(lse.cpu().numpy(), lse_ref, LSE_TOL, "LSE")


def test_zero_length_sequence():
    q, kp, vp, bt, sl = paged_decode_inputs(2, 8, 2, 1, 64, 128, seed=4, page_size=32)
    sl[0] = 0
    q, kp, vp, bt, sl = _with_lengths(q, kp, vp, bt, sl, 32)
    qd, kpd, vpd, btd, sld = to_device(q, kp, vp, bt, sl)
    _, lp, o, lse = run_paged(qd, kpd, vpd, btd, sld, 0.1, 4)
    assert torch.isneginf(lp[0]).all() and torch.isneginf(lse[0]).all()
    assert (o[0] == 0).all()
    o_ref, lse_ref = oracle.decode_paged(q, kp, vp, bt, sl, 0.1)
    cmp(o[1].float().cpu().numpy(), o_ref[1], O_TOL, "O")


def test_paged_equals_contiguous_cache():
    """The same sequences from a contiguous cache and from a scattered paged
    pool decode to the same result (within the rounding of both paths)."""
    args = (6, 32, 8, 1, 2000, 128, 77)
    q, kc, vc, sl = decode_inputs(*args, device="cuda")
    qp, kp, vp, bt, slp = paged_decode_inputs(*args, page_size=64, device="cuda")
    assert torch.equal(q, qp) and torch.equal(sl, slp)
    o1, l1 = fa.decode_attention(q, kc, vc, sl, num_splits=4)
    o2, l2 = fa.decode_attention_paged(qp, kp, vp, bt, slp, num_splits=4)
    torch.cuda.synchronize()
    assert float((o1.float() - o2.float()).abs().max()) <= O_TOL
    assert float((l1 - l2).abs().max()) <= LSE_TOL


def test_full_size_workload_every_sequence():
    """The decode workload (B=64, Hq=32, Hkv=8, d=128, L ~ U{4096..16384}) in
    16-key pages, launched as the bench launches it; every sequence and head
    against the oracle on the gathered pages."""
    c = CONFIGS["decode_b64_splitkv_d128"]
    q, kp, vp, bt, sl = paged_decode_inputs(c.B, c.Hq, c.Hkv, c.Lmin, c.Lmax, c.d, c.seed,
                                            page_size=16, device="cuda")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n = fa.decode_default_splits(c.B, c.Hkv, c.Lmax, sms)
    op, lp, o, lse = run_paged(q, kp, vp, bt, sl, c.scale, n)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    for b in range(c.B):
        L = int(sl[b])
        pages = bt[b, :(L + 15) // 16].long()
        kg = kp[pages].permute(1, 0, 2, 3).reshape(c.Hkv, -1, c.d)[:, :L].cpu()
        vg = vp[pages].permute(1, 0, 2, 3).reshape(c.Hkv, -1, c.d)[:, :L].cpu()
        o_ref, lse_ref = oracle.decode(q[b:b + 1].cpu(), kg[None], vg[None],
                                       np.array([L], dtype=np.int32), c.scale)
        cmp(o[b:b + 1].float().cpu().numpy(), o_ref, O_TOL, "O b=%d" % b)
        cmp(lse[b:b + 1].cpu().numpy(), lse_ref, LSE_TOL, "LSE b=%d" % b)
