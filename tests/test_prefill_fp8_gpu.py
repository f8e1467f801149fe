"""fa_fwd_fp8 (through the C ABI) against the fp64 oracle on a B200.

The oracle dequantises the E4M3 codes with their per-(batch, key/value head)
factors and computes exact attention of the real values.  The tolerances
follow from the kernel's arithmetic:

  LSE: <= 1e-3, as for bf16 inputs.  Products of two E4M3 values are exact
  in fp32, the scores are summed in fp32, and l sums unquantised fp32 weights.

  O, per element i:  2^-4 * A_i + n * 2^-16 * max|v| + 2^-8 * |O_i| + 1e-4
    A_i = sum_j w_ij |v_j| (the attention of |V|, from the oracle).  The
      weights fed to P.V are rounded to E4M3, whose 3 mantissa bits give a
      relative error of at most 2^-4 on normal values.
    n * 2^-16 * max|v| (n keys).  E4M3 subnormals round with an absolute
      error of at most 2^-10, and the weights are stored as p * 2^6 with the
      row's largest >= 2^6, so each key adds at most 2^-16 of l.
    2^-8 * |O_i|: the bf16 rounding of O (half an ulp is 2^-9 relative) and
      the fp32 accumulation.

Large-logit inputs (queries x 8) make the attention peaky, so a key placed in
the wrong slot of P would move O by about |v|, far outside the bound.  When
all keys of a head are equal, every weight is exactly 2^6, so O is the mean of
V to bf16 rounding; that case checks the V operand and its factor sharply.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_flashattention_b200 import fa
from io_aware_exact_flashattention_b200.inputs import (CONFIGS, fp8_prefill_inputs,
                                                       fp8_prefill_inputs_for)

pytestmark = pytest.mark.gpu

LSE_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.lib()


def _cpu(t):
    return None if t is None else t.cpu()


def run_fp8(q8, k8, v8, dq, dk, dv, causal, scale):
    B, Hq, Sq, d = q8.shape
    o = torch.empty((B, Hq, Sq, d), device=q8.device, dtype=torch.bfloat16)
    lse = torch.empty((B, Hq, Sq), device=q8.device, dtype=torch.float32)
    fa.fa_fwd_fp8(q8, k8, v8, dq, dk, dv, o, lse, causal, scale)
    torch.cuda.synchronize()
    return o, lse


def dequantised(q8, k8, v8, dq, dk, dv):
    Hkv = int(k8.shape[1])
    return (oracle.dequant_heads(q8.cpu(), _cpu(dq), Hkv),
            oracle.dequant_heads(k8.cpu(), _cpu(dk), Hkv),
            oracle.dequant_heads(v8.cpu(), _cpu(dv), Hkv))


def o_bound(o_ref, a_abs, n_keys, vmax):
    return (2.0 ** -4) * a_abs + n_keys * (2.0 ** -16) * vmax + (2.0 ** -8) * np.abs(o_ref) + 1e-4


def compare(o, lse, o_ref, lse_ref, tol):
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    assert np.isfinite(o).all(), "non-finite O"
    ninf = np.isneginf(lse_ref)
    assert (np.isneginf(lse) == ninf).all(), "LSE -inf pattern differs"
    if o.size:
        ratio = np.abs(o - o_ref) / tol
        worst = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        assert ratio.max() <= 1.0, ("O error over bound", worst, float(ratio.max()),
                                    float(o[worst]), float(o_ref[worst]))
    if lse.size:
        el = float(np.abs(np.where(ninf, 0, lse) - np.where(ninf, 0, lse_ref)).max())
        assert el <= LSE_TOL, el


def check_full(B, Hq, Hkv, Sq, Skv, causal, seed, q_mult=1.0, d=128, descales=True,
               scale=None):
    q8, k8, v8, dq, dk, dv = fp8_prefill_inputs(B, Hq, Hkv, Sq, Skv, d, seed, q_mult,
                                                device="cuda")
    if not descales:
        dq = dk = dv = None
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o, lse = run_fp8(q8, k8, v8, dq, dk, dv, causal, scale)
    qd, kd, vd = dequantised(q8, k8, v8, dq, dk, dv)
    o_ref, lse_ref = oracle.attn_fwd(qd, kd, vd, causal, scale)
    a_abs, _ = oracle.attn_fwd(qd, kd, np.abs(vd), causal, scale)
    vmax = float(np.abs(vd).max()) if vd.size else 0.0
    compare(o, lse, o_ref, lse_ref, o_bound(o_ref, a_abs, Skv, vmax))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", [1, 127, 128, 129, 255, 300, 513])
def test_square_shapes(S, causal):
    check_full(1, 2, 2, S, S, causal, seed=200 + S)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (8, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_groups(Hq, Hkv, causal):
    check_full(2, Hq, Hkv, 384, 384, causal, seed=11 * Hq + Hkv)


@pytest.mark.parametrize("Sq,Skv", [(200, 513), (513, 200), (1, 700), (128, 0), (300, 129)])
@pytest.mark.parametrize("causal", [False, True])
def test_rectangular(Sq, Skv, causal):
    check_full(1, 4, 2, Sq, Skv, causal, seed=Sq * 7 + Skv)


@pytest.mark.parametrize("causal", [False, True])
def test_large_logits(causal):
    check_full(2, 4, 4, 512, 512, causal, seed=17, q_mult=8.0)


def test_null_factors_mean_one():
    q8, k8, v8, dq, dk, dv = fp8_prefill_inputs(1, 4, 2, 300, 300, 128, 5, device="cuda")
    ones = torch.ones_like(dq)
    o1, l1 = run_fp8(q8, k8, v8, None, None, None, True, 0.1)
    o2, l2 = run_fp8(q8, k8, v8, ones, ones, ones, True, 0.1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # Without factors the inputs are the raw codes (up to 448): a small scale
    # keeps the logits near those of the other tests, where an fp32 LSE can
    # meet 1e-3 (at |LSE| ~ 1e4 one fp32 ulp is already 1e-3).
    check_full(1, 4, 2, 300, 300, True, seed=5, descales=False, scale=5e-5)


def test_factor_placement_is_exact():
    """A power of two moved from the key factor to the query factor changes
    nothing; doubling the value factor doubles O exactly."""
    q8, k8, v8, dq, dk, dv = fp8_prefill_inputs(2, 8, 2, 256, 256, 128, 6, device="cuda")
    o1, l1 = run_fp8(q8, k8, v8, dq, dk, dv, True, 0.1)
    o2, l2 = run_fp8(q8, k8, v8, dq * 2, dk / 2, dv, True, 0.1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o3, l3 = run_fp8(q8, k8, v8, dq, dk, dv * 2, True, 0.1)
    assert torch.equal(o3.float(), 2 * o1.float()) and torch.equal(l3, l1)


def test_factors_differ_per_batch_and_group():
    """Distinct factors for every (batch, key/value head) land on the right heads."""
    g = torch.Generator().manual_seed(9)
    q8, k8, v8, _, _, _ = fp8_prefill_inputs(2, 8, 4, 200, 200, 128, 9, device="cuda")
    dq, dk, dv = (torch.rand((2, 4), generator=g).add_(0.25).cuda() for _ in range(3))
    scale = 5e-5  # the codes reach 448: logits of a few units, as in the other tests
    o, lse = run_fp8(q8, k8, v8, dq, dk, dv, False, scale)
    qd, kd, vd = dequantised(q8, k8, v8, dq, dk, dv)
    o_ref, lse_ref = oracle.attn_fwd(qd, kd, vd, False, scale)
    a_abs, _ = oracle.attn_fwd(qd, kd, np.abs(vd), False, scale)
    compare(o, lse, o_ref, lse_ref, o_bound(o_ref, a_abs, 200, float(np.abs(vd).max())))


@pytest.mark.parametrize("causal", [False, True])
def test_equal_keys_give_mean_of_values(causal):
    """Every weight is exactly 2^6 in E4M3: O = mean of the visible V rows."""
    B, Hq, Hkv, S, d = 1, 4, 2, 333, 128
    q8, k8, v8, dq, dk, dv = fp8_prefill_inputs(B, Hq, Hkv, S, S, d, 21, device="cuda")
    k8 = k8[:, :, :1].expand(B, Hkv, S, d).contiguous()
    o, lse = run_fp8(q8, k8, v8, dq, dk, dv, causal, 1.0 / math.sqrt(d))
    qd, kd, vd = dequantised(q8, k8, v8, dq, dk, dv)
    o_ref, lse_ref = oracle.attn_fwd(qd, kd, vd, causal, 1.0 / math.sqrt(d))
    tol = (2.0 ** -8) * np.abs(o_ref) + 1e-5 * float(np.abs(vd).max())
    compare(o, lse, o_ref, lse_ref, tol)


def test_headline_shape_every_row():
    """The bench's extras workload in E4M3 (B=4, H=16, S=2048, d=128, causal,
    queries x 8), the launch the bench times; every row of every head against
    the oracle within the derived per-element bound."""
    c = CONFIGS["causal_mha_s2048_d128_qx8"]
    q8, k8, v8, dq, dk, dv = fp8_prefill_inputs_for(c, device="cuda")
    o, lse = run_fp8(q8, k8, v8, dq, dk, dv, c.causal, c.scale)
    qd, kd, vd = dequantised(q8, k8, v8, dq, dk, dv)
    o_ref, lse_ref = oracle.attn_fwd(qd, kd, vd, c.causal, c.scale)
    a_abs, _ = oracle.attn_fwd(qd, kd, np.abs(vd), c.causal, c.scale)
    compare(o, lse, o_ref, lse_ref, o_bound(o_ref, a_abs, c.Skv, float(np.abs(vd).max())))
