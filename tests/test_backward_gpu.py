"""fa_bwd (through the C ABI) against the fp64 oracle's exact gradients on a
B200.  The kernel gets the forward's own O and LSE (from fa_fwd), as a
training step would; the oracle recomputes everything from q, k, v and dO.

Tolerance.  P and dS enter the tensor-core products as bf16 (relative
rounding 2^-9 each), D = dO . O uses the bf16-rounded forward output, and
dq, dk, dv are rounded to bf16 (2^-9 relative); sums over up to Sq or Skv
terms accumulate in fp32.  Errors are therefore relative to each gradient's
scale: max |d - ref| <= GRAD_TOL * max |ref| for each of dq, dk, dv, with
GRAD_TOL = 2e-2 (a few 2^-9 roundings, with margin for the cancellation in
dP - D), and the Frobenius norm of the error within 1e-2 of the reference's.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_flashattention_b200 import fa
from io_aware_exact_flashattention_b200.inputs import (CONFIGS, grad_output, prefill_inputs,
                                                       prefill_inputs_for)

pytestmark = pytest.mark.gpu

GRAD_TOL = 2e-2
FRO_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.lib()


def run_bwd(B, Hq, Hkv, Sq, Skv, d, causal, seed, q_mult=1.0, scale=None):
    q, k, v = prefill_inputs(B, Hq, Hkv, Sq, Skv, d, seed, q_mult)
    d_o = grad_output((B, Hq, Sq, d), seed)
    scale = scale if scale is not None else 1.0 / math.sqrt(d)
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, d_o))
    o = torch.empty_like(qc)
    lse = torch.empty((B, Hq, Sq), device="cuda", dtype=torch.float32)
    fa.fa_fwd(qc, kc, vc, o, lse, causal, scale)
    dq, dk, dv = fa.attention_backward(qc, kc, vc, o, lse, doc, causal, scale)
    torch.cuda.synchronize()
    ref = oracle.attn_bwd(q, k, v, d_o, causal, scale)
    errs = {}
    for name, got, want in (("dq", dq, ref[0]), ("dk", dk, ref[1]), ("dv", dv, ref[2])):
        g = got.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all(), name + ": non-finite"
        scale_ref = max(float(np.abs(want).max()), 1e-30)
        e_max = float(np.abs(g - want).max()) / scale_ref if g.size else 0.0
        e_fro = (float(np.linalg.norm(g - want)) / max(float(np.linalg.norm(want)), 1e-30)
                 if g.size else 0.0)
        errs[name] = (e_max, e_fro)
    return errs


def check(errs):
    for name, (e_max, e_fro) in errs.items():
        assert e_max <= GRAD_TOL and e_fro <= FRO_TOL, "%s: max %.3e fro %.3e (%s)" % (
            name, e_max, e_fro, errs)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_square(d, causal):
    check(run_bwd(1, 2, 2, 300, 300, d, causal, seed=40 + d + causal))


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 1)])
def test_gqa(Hq, Hkv):
    check(run_bwd(2, Hq, Hkv, 257, 257, 128, True, seed=50 + Hq))


@pytest.mark.parametrize("Sq,Skv", [(150, 400), (400, 150), (128, 384)])
def test_rectangular_causal(Sq, Skv):
    # Sq > Skv: the first Sq - Skv query rows see no key (zero gradients there)
    check(run_bwd(1, 4, 2, Sq, Skv, 128, True, seed=60 + Sq))


def test_large_logits_q_times_8():
    check(run_bwd(1, 2, 2, 512, 512, 128, True, seed=70, q_mult=8.0))


def test_headline_shape_eight_heads():
    """The bench's extras workload (causal MHA B=4 H=16 S=2048 d=128, Q*8),
    forward and backward launched on the whole problem as the bench launches
    them; the gradients of 8 heads (two per batch) against the oracle, which
    differentiates one head at a time."""
    c = CONFIGS["causal_mha_s2048_d128_qx8"]
    q, k, v = prefill_inputs_for(c)
    d_o = grad_output(q.shape, c.seed)
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, d_o))
    o = torch.empty_like(qc)
    lse = torch.empty((c.B, c.Hq, c.Sq), device="cuda", dtype=torch.float32)
    fa.fa_fwd(qc, kc, vc, o, lse, c.causal, c.scale)
    dq, dk, dv = fa.attention_backward(qc, kc, vc, o, lse, doc, c.causal, c.scale)
    torch.cuda.synchronize()
    for b in range(c.B):
        for h in (b, c.Hq - 1 - 2 * b):
            sl = (slice(b, b + 1), slice(h, h + 1))
            ref = oracle.attn_bwd(q[sl], k[sl], v[sl], d_o[sl], c.causal, c.scale)
            errs = {}
            for name, got, want in (("dq", dq, ref[0]), ("dk", dk, ref[1]), ("dv", dv, ref[2])):
                g = got[sl].float().cpu().numpy().astype(np.float64)
                assert np.isfinite(g).all(), name + ": non-finite"
                errs[name] = (float(np.abs(g - want).max()) / max(float(np.abs(want).max()), 1e-30),
                              float(np.linalg.norm(g - want)) / max(float(np.linalg.norm(want)), 1e-30))
            check(errs)


def test_rectangular_full():
    # no mask, more key tiles than query tiles and ragged on both sides
    check(run_bwd(1, 4, 2, 200, 650, 128, False, seed=80))


def test_no_keys_gives_zero_dq():
    """Skv = 0: the dQ kernel sees no key tile and writes zeros."""
    B, Hq, Hkv, Sq, d = 1, 2, 1, 200, 128
    q = torch.randn(B, Hq, Sq, d, device="cuda").to(torch.bfloat16)
    k = torch.empty(B, Hkv, 0, d, device="cuda", dtype=torch.bfloat16)
    v = torch.empty_like(k)
    o = torch.zeros_like(q)
    lse = torch.full((B, Hq, Sq), -math.inf, device="cuda")
    d_o = torch.randn_like(q)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, d_o, True, 0.088)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dq).item() == 0
    assert dk.numel() == 0 and dv.numel() == 0


def test_repeat_calls_bit_identical():
    """Each gradient is accumulated in one CTA's tensor memory and written
    once, so two calls give the same bits."""
    q, k, v = prefill_inputs(2, 4, 2, 520, 520, 128, 90, 1.0)
    d_o = grad_output((2, 4, 520, 128), 90)
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, d_o))
    o = torch.empty_like(qc)
    lse = torch.empty((2, 4, 520), device="cuda", dtype=torch.float32)
    fa.fa_fwd(qc, kc, vc, o, lse, True, 0.088)
    first = fa.attention_backward(qc, kc, vc, o, lse, doc, True, 0.088)
    second = fa.attention_backward(qc, kc, vc, o, lse, doc, True, 0.088)
    torch.cuda.synchronize()
    for a, b in zip(first, second):
        assert torch.equal(a, b)


def test_gqa_long_dkdv_ctas_order_by_role():
    """GQA with four query heads per kv head at S = 4096: each dK/dV CTA is long,
    so the launch takes the by-role CTA order (all dK/dV CTAs, then the dQ
    ones).  The whole problem is launched; kv head 7 and its four query heads
    are checked against the oracle."""
    B, Hq, Hkv, S, d = 1, 32, 8, 4096, 128
    q, k, v = prefill_inputs(B, Hq, Hkv, S, S, d, 95, 1.0)
    d_o = grad_output((B, Hq, S, d), 95)
    scale = 1.0 / math.sqrt(d)
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, d_o))
    o = torch.empty_like(qc)
    lse = torch.empty((B, Hq, S), device="cuda", dtype=torch.float32)
    fa.fa_fwd(qc, kc, vc, o, lse, True, scale)
    dq, dk, dv = fa.attention_backward(qc, kc, vc, o, lse, doc, True, scale)
    torch.cuda.synchronize()
    hq, hk = slice(28, 32), slice(7, 8)
    ref = oracle.attn_bwd(q[:, hq], k[:, hk], v[:, hk], d_o[:, hq], True, scale)
    errs = {}
    for name, got, want in (("dq", dq[:, hq], ref[0]), ("dk", dk[:, hk], ref[1]),
                            ("dv", dv[:, hk], ref[2])):
        g = got.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all(), name + ": non-finite"
        errs[name] = (float(np.abs(g - want).max()) / max(float(np.abs(want).max()), 1e-30),
                      float(np.linalg.norm(g - want)) / max(float(np.linalg.norm(want)), 1e-30))
    check(errs)


def test_inputs_written_just_before_the_call():
    """The main backward kernel is a programmatic dependent of the D kernel:
    its K, V, Q and dO loads may start before the D kernel ends, and only its
    reads of the D kernel's output wait.  Inputs written by a kernel enqueued
    right before the call (here: dO, o and lse rewritten in place on the same
    stream, no synchronisation) must still be seen, and a following call's D
    kernel must not overwrite the workspace under a running main kernel: the
    result equals a call made after a full synchronisation, bit for bit."""
    B, Hq, Hkv, S, d = 2, 8, 2, 1000, 128
    q, k, v = prefill_inputs(B, Hq, Hkv, S, S, d, 91, 1.0)
    d_o = grad_output((B, Hq, S, d), 91)
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, d_o))
    o = torch.empty_like(qc)
    lse = torch.empty((B, Hq, S), device="cuda", dtype=torch.float32)
    fa.fa_fwd(qc, kc, vc, o, lse, True, 0.088)
    torch.cuda.synchronize()
    ref = [t.clone() for t in fa.attention_backward(qc, kc, vc, o, lse, doc, True, 0.088)]
    torch.cuda.synchronize()
    # scramble the inputs, then restore them with kernels on the compute
    # stream immediately before each call
    saved = [t.clone() for t in (o, lse, doc)]
    for _ in range(3):
        for t in (o, lse, doc):
            t.fill_(7.0)
        for t, s in zip((o, lse, doc), saved):
            t.copy_(s)
        got = fa.attention_backward(qc, kc, vc, o, lse, doc, True, 0.088)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
