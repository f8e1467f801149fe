"""The seeded input generators on the CPU: determinism, the documented
distributions' basic shape, and the paged layout checked against the
oracle's independent block-table gather."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_flashattention_b200.inputs import (decode_inputs, grad_output, paginate,
                                                       paged_decode_inputs, prefill_inputs)


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
