"""The polynomial 2^x used for part of the softmax weights (the FP8 prefill
and the backward's dK/dV kernel).

CPU: the fit is re-derived from its definition (exp2_poly_fit.py, a Remez
exchange for minimal relative error of a cubic on [-1/2, 1/2]); the kernel's
constants must be that fit rounded to fp32, and the kernel's fp32 evaluation
sequence, emulated in numpy, must stay within the fit's error bound.
GPU: the device evaluation (through the test hook) must equal the numpy
emulation bit for bit and agree with torch.exp2 within the bound.
"""
import os
import re
import sys

import numpy as np
import pytest
import torch

from io_aware_exact_flashattention_b200 import build as fabuild
from io_aware_exact_flashattention_b200 import fa

sys.path.insert(0, fabuild.CSRC)
import exp2_poly_fit  # noqa: E402

BOUND = 8e-5  # the fit's max relative error is 7.48e-5; fp32 evaluation adds < 1e-6


def kernel_constants():
    text = open(os.path.join(fabuild.CSRC, "sm100.cuh")).read()
    return [float(re.search(r"kExp2C%d = ([0-9.eE+-]+)f;" % i, text).group(1)) for i in range(4)]


def emulate(x):
    """The kernel's fp32 sequence: clamp, round via 1.5*2^23, cubic in f, add n
    to the exponent field."""
    c = [np.float32(v) for v in kernel_constants()]
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    big = np.float32(12582912.0)
    t = (x + big).astype(np.float32)
    n = (t - big).astype(np.float32)
    f = (x.astype(np.float64) - n).astype(np.float32)  # one fma(n, -1, x)

    def fma(a, b, d):
        return (a.astype(np.float64) * b + d).astype(np.float32)

    q = fma(f, c[3], c[2])
    q = fma(q, f, c[1])
    q = fma(q, f, c[0])
    bits = (q.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23)
                                                   & 0xFFFFFFFF)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_constants_are_the_fit():
    fit, err = exp2_poly_fit.coefficients_fp32()
    assert err < 7.6e-5
    for a, b in zip(kernel_constants(), fit):
        assert np.float32(a) == np.float32(b), (a, b)


def test_fit_is_equioscillating():
    """A minimax fit's error reaches its maximum with alternating signs at
    degree + 2 points (Chebyshev alternation)."""
    c, err = exp2_poly_fit.remez_relative()
    f = np.linspace(-0.5, 0.5, 200001)
    e = np.polyval(c[::-1], f) / 2.0 ** f - 1.0
    peaks = [i for i in range(1, len(f) - 1) if abs(e[i]) >= abs(e[i - 1]) and abs(e[i]) >= abs(e[i + 1])]
    peaks = [0] + peaks + [len(f) - 1]
    big = [i for i in peaks if abs(e[i]) > 0.99 * err]
    assert len(big) >= exp2_poly_fit.DEGREE + 2
    signs = np.sign(e[big])
    assert (signs[1:] != signs[:-1]).all()


def test_emulated_sequence_within_bound():
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    y = emulate(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < BOUND
    # integers are scaled exactly from p(0) = c0
    k = np.arange(-120, 9, dtype=np.float32)
    assert np.all(np.abs(emulate(k) / np.exp2(k.astype(np.float64)) - 1) < BOUND)
    # very negative arguments give (almost) nothing, never garbage
    tiny = emulate(np.array([-126.0, -200.0, -1e30], np.float32))
    assert np.all((tiny >= 0) & (tiny < 2e-38))


def test_hook_rejects_bad_args():
    fabuild.build()
    assert fa.lib().fa_debug_exp2_poly(None, None, -1, None) == 1
    assert fa.lib().fa_debug_exp2_poly(None, None, 0, None) == 0
    assert fa.lib().fa_debug_exp2_poly(256 + 4, 256, 8, None) == 3


@pytest.mark.gpu
def test_device_matches_emulation_and_exp2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.rand(1_000_000, generator=g) * 133.0 - 125.0,
                   torch.tensor([0.0, 1.0, -1.0, 0.5, -0.5, 8.0, -126.0, -300.0])])
    y = fa.debug_exp2_poly(x.cuda()).cpu().numpy()
    assert np.array_equal(y.view(np.uint32), emulate(x.numpy()).view(np.uint32))
    ref = torch.exp2(x.double()).numpy()
    ok = x.numpy() > -125.0
    assert np.abs(y[ok] / ref[ok] - 1.0).max() < BOUND
