"""The seeded input generators on the CPU: determinism, the documented
distributions' basic shape, and the paged layout checked against the
oracle's independent block-table gather."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_flashattention_b200.inputs import (decode_inputs, fp8_prefill_inputs,
                                                       grad_output, paginate,
                                                       paged_decode_inputs, prefill_inputs,
                                                       quantize_e4m3)


def test_prefill_inputs_deterministic_and_scaled():
    a = prefill_inputs(1, 2, 1, 40, 50, 64, seed=3, q_mult=8.0)
    b = prefill_inputs(1, 2, 1, 40, 50, 64, seed=3, q_mult=8.0)
    c = prefill_inputs(1, 2, 1, 40, 50, 64, seed=3, q_mult=1.0)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert all(t.dtype == torch.bfloat16 and t.is_contiguous() for t in a)
    # Q x 8 is exact in bf16 (a power of two); K and V do not depend on it
    assert torch.equal(a[0].float(), c[0].float() * 8)
    assert torch.equal(a[1], c[1]) and torch.equal(a[2], c[2])


def test_grad_output_seeded():
    x = grad_output((2, 3, 5, 8), seed=9)
    assert torch.equal(x, grad_output((2, 3, 5, 8), seed=9))
    assert not torch.equal(x, grad_output((2, 3, 5, 8), seed=10))
    assert x.dtype == torch.bfloat16


@pytest.mark.parametrize("P", [16, 32, 128, 256])
def test_paginate_matches_oracle_gather(P):
    q, kc, vc, sl = decode_inputs(4, 8, 2, 1, 600, 64, seed=P)
    kp, vp, bt = paginate(kc, vc, sl, P, seed=P)
    # pool holds exactly the used pages; every used page appears once
    counts = [(int(L) + P - 1) // P for L in sl.tolist()]
    assert kp.shape[0] == max(1, sum(counts))
    used = bt[bt >= 0].tolist()
    assert sorted(used) == list(range(sum(counts)))
    for b, n in enumerate(counts):
        assert (bt[b, :n] >= 0).all() and (bt[b, n:] == -1).all()
    kg, vg = oracle.paged_gather(kp, vp, bt, sl)
    for b in range(4):
        L = int(sl[b])
        assert np.array_equal(kg[b, :, :L], kc[b, :, :L].double().numpy())
        assert np.array_equal(vg[b, :, :L], vc[b, :, :L].double().numpy())
        n = counts[b]
        if n and L % P:
            last = int(bt[b, n - 1])
            assert torch.isnan(kp[last, :, L % P:].float()).all(), "rows past L_b must be poison"


def test_paged_decode_inputs_match_decode_inputs():
    q, kp, vp, bt, sl = paged_decode_inputs(3, 4, 2, 1, 300, 64, seed=8, page_size=32)
    q2, kc, vc, sl2 = decode_inputs(3, 4, 2, 1, 300, 64, seed=8)
    assert torch.equal(q, q2) and torch.equal(sl, sl2)
    o, lse = oracle.decode_paged(q, kp, vp, bt, sl, 0.125)
    o2, lse2 = oracle.decode(q2, kc, vc, sl2, 0.125)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_quantiser_round_trip():
    """quantize_e4m3's codes dequantise (through the oracle) to within E4M3
    rounding of the input: 2^-4 relative for normal codes, 2^-10 of the
    factor for subnormal ones; each group's largest magnitude maps to 448."""
    x = torch.randn((2, 4, 64, 128), generator=torch.Generator().manual_seed(3))
    x8, ds = quantize_e4m3(x, 2)
    assert x8.dtype == torch.float8_e4m3fn and tuple(ds.shape) == (2, 2)
    back = oracle.dequant_heads(x8, ds, 2)
    per_head = ds.repeat_interleave(2, dim=1)[:, :, None, None].double().numpy()
    xd = x.double().numpy()
    assert (np.abs(back - xd) <= np.abs(xd) * 2.0 ** -4 + 2.0 ** -10 * per_head).all()
    codes = x8.float().abs().reshape(2, 2, -1).amax(dim=2)
    assert torch.equal(codes, torch.full((2, 2), 448.0))


def test_fp8_inputs_deterministic():
    a = fp8_prefill_inputs(1, 4, 2, 30, 40, 128, seed=8, q_mult=8.0)
    b = fp8_prefill_inputs(1, 4, 2, 30, 40, 128, seed=8, q_mult=8.0)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8) if x.element_size() == 1 else x,
                           y.view(torch.uint8) if y.element_size() == 1 else y)
    q8, k8, v8, dq, dk, dv = a
    assert q8.shape == (1, 4, 30, 128) and k8.shape == (1, 2, 40, 128)
    assert dq.shape == dk.shape == dv.shape == (1, 2)


def test_quantiser_empty_sequence():
    x8, ds = quantize_e4m3(torch.zeros((2, 4, 0, 128)), 2)
    assert x8.shape == (2, 4, 0, 128) and torch.equal(ds, torch.ones((2, 2)))
