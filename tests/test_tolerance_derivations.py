"""The tolerances derived from the arithmetic, checked against emulations of
that arithmetic (CPU only).

The FP8 forward and the feed-forward network have no tolerance fixed by the
workload; their GPU tests use bounds derived from how the kernels round.  Here
numpy reproduces those rounding schemes (not the kernels' code, which these
tests never touch) and the emulated results must stay within the same bounds
against the fp64 oracle.  A derivation that forgot a rounding step, or a
bound written too tight, fails here before any GPU run.
"""
import math

import numpy as np
import torch

import oracle
from io_aware_exact_flashattention_b200.inputs import ffn_inputs, fp8_prefill_inputs


def e4m3(x):
    """Round to E4M3, nearest even, saturating at 448 (torch's conversion)."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).clamp(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).double().numpy()


def bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def emulate_fp8_forward(q_codes, k_codes, v_codes, dq, dk, dv, causal, scale, Hkv):
    """The E4M3 forward's rounding: per 128-key tile, a reference max that
    moves only when the row max grows by more than 2^2 (in exponent units),
    weights p * 2^6 rounded to E4M3 for P.V, l summed from the unrounded
    weights, O = acc * dv / l rounded to bf16."""
    B, Hq, Sq, d = q_codes.shape
    Skv = k_codes.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, Sq, d))
    rows = np.arange(Sq)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            c = scale * math.log2(math.e) * dq[b, g] * dk[b, g]
            s_all = q_codes[b, h] @ k_codes[b, g].T
            last = rows + (Skv - Sq) if causal else np.full(Sq, Skv - 1)
            m = np.full(Sq, -np.inf)
            l = np.zeros(Sq)
            acc = np.zeros((Sq, d))
            for j0 in range(0, Skv, 128):
                s = s_all[:, j0:j0 + 128].copy()
                keys = np.arange(j0, j0 + s.shape[1])
                s[keys[None, :] > last[:, None]] = -np.inf
                m_new = np.maximum(m, s.max(axis=1))
                with np.errstate(invalid="ignore"):
                    move = (m_new - m) * c > 2.0
                alpha = np.where(move, np.exp2(np.where(np.isinf(m), -np.inf, (m - m_new) * c)), 1.0)
                l *= alpha
                acc *= alpha[:, None]
                m = np.where(move, m_new, m)
                mc = np.where(np.isinf(m), 0.0, m * c)
                p = np.exp2(s * c - mc[:, None] + 6.0)
                l += p.sum(axis=1)
                acc += e4m3(p) @ v_codes[b, g, j0:j0 + s.shape[1]]
            with np.errstate(invalid="ignore", divide="ignore"):
                out[b, h] = np.where(l[:, None] > 0, acc * dv[b, g] / l[:, None], 0.0)
    return bf16(out)


def test_fp8_bound_holds_for_its_rounding():
    for (B, Hq, Hkv, S, q_mult, causal, seed) in ((1, 2, 2, 300, 8.0, True, 1),
                                                  (1, 4, 2, 256, 1.0, False, 2),
                                                  (1, 2, 1, 260, 8.0, False, 3)):
        q8, k8, v8, dq, dk, dv = fp8_prefill_inputs(B, Hq, Hkv, S, S, 128, seed, q_mult)
        codes = [oracle.dequant_heads(x, None, Hkv) for x in (q8, k8, v8)]
        f = [x.double().numpy() for x in (dq, dk, dv)]
        scale = 1.0 / math.sqrt(128)
        got = emulate_fp8_forward(*codes, *f, causal, scale, Hkv)
        qr, kr, vr = (oracle.dequant_heads(x, fx, Hkv) for x, fx in ((q8, dq), (k8, dk), (v8, dv)))
        o_ref, _ = oracle.attn_fwd(qr, kr, vr, causal, scale)
        a_abs, _ = oracle.attn_fwd(qr, kr, np.abs(vr), causal, scale)
        bound = (2.0 ** -4 * a_abs + S * 2.0 ** -16 * float(np.abs(vr).max())
                 + 2.0 ** -8 * np.abs(o_ref) + 1e-4)
        ratio = float((np.abs(got - o_ref) / bound).max())
        assert ratio <= 1.0, ratio
        # and the bound is not vacuous: the rounding of P shows
        assert float(np.abs(got - o_ref).max()) > 1e-3


def test_ffn_bound_holds_for_its_rounding():
    for (B, Hq, S, d, F, seed) in ((1, 2, 300, 128, 512, 1), (2, 4, 200, 64, 256, 2)):
        o, w1, w2 = ffn_inputs(B, Hq, S, d, F, seed)
        x = oracle.heads_to_tokens(o).reshape(B * S, Hq * d)
        w1n, w2n = w1.double().numpy(), w2.double().numpy()
        h32 = x.astype(np.float32) @ w1n.T.astype(np.float32)
        h32 = 0.5 * h32 * (1.0 + torch.erf(torch.from_numpy(h32) / math.sqrt(2.0)).numpy())
        y = bf16(bf16(h32).astype(np.float32) @ w2n.T.astype(np.float32))
        h_ref = oracle.ffn_hidden(x, w1n)
        y_ref = oracle.ffn(x, w1n, w2n)
        K = Hq * d
        bound = ((2.0 ** -8 + F * 2.0 ** -24) * (np.abs(h_ref) @ np.abs(w2n).T)
                 + 1.13 * K * 2.0 ** -24 * ((np.abs(x) @ np.abs(w1n).T) @ np.abs(w2n).T)
                 + 2.0 ** -8 * np.abs(y_ref) + 1e-6)
        ratio = float((np.abs(y - y_ref) / bound).max())
        assert ratio <= 1.0, ratio
        assert float(np.abs(y - y_ref).max()) > 0.0
