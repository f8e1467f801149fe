"""fa_bpt_ffn (through the C ABI) against the fp64 oracle on a B200.

The network's input is a seeded bf16 stand-in for an attention output, so the
oracle's inputs never come from the CUDA path.  Per output element the bound
follows from the arithmetic (bf16 inputs, fp32 accumulation, H and y rounded
to bf16 once each):

  2^-8 * (|H| |W2|^T)        H rounded to bf16 (half an ulp is 2^-9 relative)
  + F * 2^-24 * (|H| |W2|^T)  fp32 accumulation of the second product
  + 1.13 * K * 2^-24 * ((|x| |W1|^T) |W2|^T)
                              fp32 accumulation of the first product, through
                              GELU (slope at most 1.13) and W2
  + 2^-8 * |y|                y rounded to bf16
  + 1e-6

with H the oracle's hidden activations.  Any misplaced head, token, column or
chunk row moves y by about |y| and falls far outside it.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_flashattention_b200 import fa
from io_aware_exact_flashattention_b200.inputs import ffn_inputs, prefill_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.lib()


def ffn_bound(x, w1, w2, h_ref, y_ref):
    a1, a2 = np.abs(w1), np.abs(w2)
    K, F = w1.shape[1], w1.shape[0]
    hw = np.abs(h_ref) @ a2.T
    return ((2.0 ** -8 + F * 2.0 ** -24) * hw
            + 1.13 * K * 2.0 ** -24 * ((np.abs(x) @ a1.T) @ a2.T)
            + 2.0 ** -8 * np.abs(y_ref) + 1e-6)


def check_rows(y_got, x, w1, w2):
    """y_got [n, D] (torch, any device) against the oracle on token rows x [n, D]."""
    w1n, w2n = (w.double().numpy() for w in (w1, w2))
    h_ref = oracle.ffn_hidden(x, w1n)
    y_ref = oracle.ffn(x, w1n, w2n)
    tol = ffn_bound(x, w1n, w2n, h_ref, y_ref)
    got = y_got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all(), "non-finite y"
    ratio = np.abs(got - y_ref) / tol
    worst = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
    assert ratio.max() <= 1.0, ("y error over bound", worst, float(ratio.max()),
                                float(got[worst]), float(y_ref[worst]))


@pytest.mark.parametrize("B,Hq,S,d,F,chunk", [
    (1, 2, 300, 128, 512, 2),     # ragged last tile, two chunks
    (2, 4, 200, 64, 256, 1),      # two sequences, one tile per chunk
    (1, 4, 128, 128, 768, 8),     # one full tile, F = 3 column tiles
    (3, 2, 130, 128, 256, 3),     # tiles of three sequences in one chunk
])
def test_ffn_matches_oracle(B, Hq, S, d, F, chunk):
    o, w1, w2 = ffn_inputs(B, Hq, S, d, F, seed=B * 100 + S)
    y = fa.bpt_ffn(o.cuda(), w1.cuda(), w2.cuda(), chunk_tiles=chunk)
    torch.cuda.synchronize()
    x = oracle.heads_to_tokens(o).reshape(B * S, Hq * d)
    check_rows(y.reshape(B * S, Hq * d), x, w1, w2)


def test_chunking_changes_nothing():
    """Each tile is computed the same way whatever chunk it falls in."""
    o, w1, w2 = ffn_inputs(2, 2, 333, 128, 512, seed=7)
    oc, w1c, w2c = o.cuda(), w1.cuda(), w2.cuda()
    ys = [fa.bpt_ffn(oc, w1c, w2c, chunk_tiles=c) for c in (1, 2, 3, 100)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


@pytest.mark.parametrize("B,Hq,Hkv,S,d,causal", [(1, 2, 1, 300, 128, True),
                                                (2, 4, 2, 700, 64, True),
                                                (1, 2, 2, 520, 128, False)])
def test_layer_is_attention_then_ffn(B, Hq, Hkv, S, d, causal):
    """bpt_layer runs attention and the network chunk by chunk; its y equals
    the network on fa_fwd's whole output and its LSE equals fa_fwd's, bit for
    bit, for chunkings that split query-tile pairs (1, 3) or not (2) and one
    chunk (100); and y is checked against the oracle's layer.  The bound adds
    the attention's own error (|dO| <= 2e-2, the forward's tolerance) carried
    through GELU and both maps."""
    F = 512
    q, k, v = prefill_inputs(B, Hq, Hkv, S, S, d, seed=9 + S)
    _, w1, w2 = ffn_inputs(B, Hq, S, d, F, seed=9)
    scale = 1.0 / math.sqrt(d)
    qc, kc, vc, w1c, w2c = q.cuda(), k.cuda(), v.cuda(), w1.cuda(), w2.cuda()
    o = torch.empty_like(qc)
    lse = torch.empty((B, Hq, S), device="cuda")
    fa.fa_fwd(qc, kc, vc, o, lse, causal, scale)
    y_two_pass = fa.bpt_ffn(o, w1c, w2c, chunk_tiles=2)
    for chunk in (1, 2, 3, 100):
        y, lse_l = fa.bpt_layer(qc, kc, vc, w1c, w2c, causal=causal, scale=scale,
                                chunk_tiles=chunk)
        torch.cuda.synchronize()
        assert torch.equal(y, y_two_pass), chunk
        assert torch.equal(lse_l, lse), chunk
    y_ref, o_ref, _ = oracle.bpt_layer(q, k, v, w1, w2, causal, scale)
    x_ref = oracle.heads_to_tokens(o_ref).reshape(B * S, Hq * d)
    w1n, w2n = (w.double().numpy() for w in (w1, w2))
    tol = ffn_bound(x_ref, w1n, w2n, oracle.ffn_hidden(x_ref, w1n), y_ref.reshape(B * S, -1))
    tol = tol + 1.13 * 2e-2 * (np.abs(w2n) @ (np.abs(w1n) @ np.ones(Hq * d)))[None, :]
    got = y.reshape(B * S, -1).float().cpu().numpy()
    assert (np.abs(got - y_ref.reshape(B * S, -1)) <= tol).all()


def test_layer_workspace_is_one_chunk():
    """The layer's scratch holds one chunk's attention output and hidden
    activations, not the sequence's."""
    B, Hq, d, F, chunk = 4, 16, 128, 8192, 2
    got = fa.bpt_layer_workspace_bytes(B, Hq, d, F, chunk)
    rows = chunk * 128
    assert got == B * Hq * rows * d * 2 + B * rows * F * 2
    assert got * 8 == B * 2048 * Hq * d * 2 + B * 2048 * F * 2  # S = 2048: 8 chunks


def test_headline_shape_every_tile():
    """The bench's configuration: the causal S=2048 workload's attention
    output shape (B=4, H=16, d=128: D=2048), F = 4 D = 8192, 16 query tiles
    per chunk; the first, the last and two random tokens of every 128-token
    tile (so every tile of every chunk) against the oracle."""
    B, Hq, S, d, F = 4, 16, 2048, 128, 8192
    o, w1, w2 = ffn_inputs(B, Hq, S, d, F, seed=2)
    y = fa.bpt_ffn(o.cuda(), w1.cuda(), w2.cuda(), chunk_tiles=16)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    toks = set()
    for t0 in range(0, B * S, 128):
        toks.update({t0, t0 + 127})
        toks.update(int(x) for x in rng.integers(t0, t0 + 128, 2))
    toks = sorted(toks)
    x_all = oracle.heads_to_tokens(o).reshape(B * S, Hq * d)
    check_rows(y.reshape(B * S, -1)[toks], x_all[toks], w1, w2)


def test_inputs_written_just_before_the_call():
    """Each network launch is a programmatic dependent of the kernel before it:
    its setup may overlap that kernel, its first load waits for it.  The input
    o and the weights rewritten in place on the same stream right before the
    call (no synchronisation), and several calls in flight back to back (the
    next chunk's first product reuses the buffer the previous second product
    reads), still give the synchronised result bit for bit."""
    o, w1, w2 = ffn_inputs(2, 4, 700, 128, 1024, seed=13)
    oc, w1c, w2c = o.cuda(), w1.cuda(), w2.cuda()
    ref = fa.bpt_ffn(oc, w1c, w2c, chunk_tiles=2).clone()
    torch.cuda.synchronize()
    saved = [t.clone() for t in (oc, w1c, w2c)]
    outs = []
    for _ in range(3):
        for t in (oc, w1c, w2c):
            t.fill_(3.0)
        for t, s in zip((oc, w1c, w2c), saved):
            t.copy_(s)
        outs.append(fa.bpt_ffn(oc, w1c, w2c, chunk_tiles=2))
    torch.cuda.synchronize()
    for y in outs:
        assert torch.equal(y, ref)
