"""fa_fwd (through the C ABI) against the fp64 oracle on a B200.

Tolerances: max |dO| <= 2e-2 and max |dLSE| <= 1e-3 for bf16 inputs with
fp32 accumulation.  The bf16 rounding of O alone costs up to half an ulp of
|O| (0.0156 for |O| in [4, 8)), so the O bound leaves room for the bf16
rounding of the probabilities fed to the P.V product; the LSE is formed in
fp32 from an fp32 running sum and has no bf16 step.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_flashattention_b200 import fa
from io_aware_exact_flashattention_b200.inputs import CONFIGS, prefill_inputs, prefill_inputs_for

pytestmark = pytest.mark.gpu

O_TOL = 2e-2
LSE_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fa.lib()
    torch.manual_seed(0)


def run_fa(q, k, v, causal, scale, stream=None):
    B, Hq, Sq, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Sq), device=q.device, dtype=torch.float32)
    fa.fa_fwd(q, k, v, o, lse, causal, scale, stream=stream)
    return o, lse


def errors(o, lse, o_ref, lse_ref):
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    assert np.isfinite(o).all(), "non-finite O"
    ninf = np.isneginf(lse_ref)
    assert (np.isneginf(lse) == ninf).all(), "LSE -inf pattern differs"
    eo = float(np.abs(o - o_ref).max()) if o.size else 0.0
    el = float(np.abs(np.where(ninf, 0, lse) - np.where(ninf, 0, lse_ref)).max()) if lse.size else 0.0
    return eo, el


def check_full(B, Hq, Hkv, Sq, Skv, d, causal, seed, q_mult=1.0, scale=None):
    q, k, v = prefill_inputs(B, Hq, Hkv, Sq, Skv, d, seed, q_mult, device="cuda")
    scale = scale if scale is not None else 1.0 / math.sqrt(d)
    o, lse = run_fa(q, k, v, causal, scale)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal, scale)
    eo, el = errors(o, lse, o_ref, lse_ref)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)
    return eo, el


def test_config_mha_s512_d64():
    c = CONFIGS["mha_s512_d64"]
    check_full(c.B, c.Hq, c.Hkv, c.Sq, c.Skv, c.d, c.causal, c.seed, c.q_mult)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S", [1, 127, 128, 129, 255, 256, 300, 513])
def test_square_shapes(S, causal, d):
    check_full(1, 2, 2, S, S, d, causal, seed=100 + S)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (8, 2), (8, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_groups(Hq, Hkv, causal):
    check_full(2, Hq, Hkv, 384, 384, 128, causal, seed=7 * Hq + Hkv)


@pytest.mark.parametrize("Sq,Skv", [(100, 700), (384, 1000), (1, 900), (700, 300), (260, 129), (128, 0)])
@pytest.mark.parametrize("causal", [False, True])
def test_rectangular(Sq, Skv, causal):
    # causal with Sq > Skv leaves leading rows with no visible key: O = 0, LSE = -inf
    check_full(1, 2, 1, Sq, Skv, 128, causal, seed=Sq + 3 * Skv)


def test_large_logits_q_times_8():
    # the config-2 distribution (Q ~ N(0,1)*8) on a smaller, fully checked shape
    check_full(1, 4, 4, 640, 640, 128, True, seed=22, q_mult=8.0)


def test_overflow_stress_q_times_1024():
    """Scores of order 1e3-1e4: exp would overflow fp32 without the running
    max.  O must match; the LSE is compared relative to its magnitude (fp32
    scores of size ~1e4 carry ~1e-3 absolute rounding)."""
    q, k, v = prefill_inputs(1, 2, 2, 256, 256, 64, 31, 1024.0, device="cuda")
    scale = 0.125
    o, lse = run_fa(q, k, v, True, scale)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, scale)
    o_np = o.float().cpu().numpy()
    assert np.isfinite(o_np).all() and torch.isfinite(lse).all()
    assert float(np.abs(o_np - o_ref).max()) <= O_TOL
    rel = np.abs(lse.cpu().numpy() - lse_ref) / np.maximum(1.0, np.abs(lse_ref))
    assert float(rel.max()) <= 2e-6


def test_empty_and_keyless():
    q, k, v = prefill_inputs(1, 2, 2, 0, 64, 64, 1, device="cuda")
    o, lse = run_fa(q, k, v, False, 0.1)  # Sq = 0: no-op
    assert o.numel() == 0
    # Skv = 0: every row sees no key
    q = torch.randn(1, 2, 70, 64, device="cuda").bfloat16()
    kv = torch.empty(1, 2, 0, 64, device="cuda", dtype=torch.bfloat16)
    k0 = torch.empty(1, 2, 8, 64, device="cuda", dtype=torch.bfloat16)  # a valid base pointer
    o = torch.full_like(q, 7.0)
    lse = torch.zeros(1, 2, 70, device="cuda")
    assert fa.lib().fa_fwd(q.data_ptr(), k0.data_ptr(), k0.data_ptr(), o.data_ptr(),
                           lse.data_ptr(), 1, 2, 2, 70, 0, 64, 0, 0.1, None) == 0
    torch.cuda.synchronize()
    assert (o == 0).all() and torch.isneginf(lse).all()
    del kv


def test_guard_bytes_untouched_and_deterministic():
    q, k, v = prefill_inputs(1, 4, 2, 300, 300, 128, 5, device="cuda")
    B, Hq, Sq, d = q.shape
    n = q.numel()
    guard = 4096
    obuf = torch.full((n + 2 * guard,), 3.0, device="cuda", dtype=torch.bfloat16)
    lbuf = torch.full((B * Hq * Sq + 2 * guard,), 5.0, device="cuda")
    o = obuf[guard:guard + n].view(q.shape)
    lse = lbuf[guard:guard + B * Hq * Sq].view(B, Hq, Sq)
    fa.fa_fwd(q, k, v, o, lse, True, 0.088)
    o1, l1 = o.clone(), lse.clone()
    fa.fa_fwd(q, k, v, o, lse, True, 0.088)
    torch.cuda.synchronize()
    assert (obuf[:guard] == 3.0).all() and (obuf[guard + n:] == 3.0).all()
    assert (lbuf[:guard] == 5.0).all() and (lbuf[guard + B * Hq * Sq:] == 5.0).all()
    assert torch.equal(o1, o) and torch.equal(l1, lse), "two runs differ"


@pytest.mark.parametrize("d", [64, 128])
def test_output_only_16_byte_aligned(d):
    """O rows are written with 32-byte stores when o is 32-byte aligned and
    with 16-byte stores otherwise; both give the same bytes and stay inside
    the output."""
    q, k, v = prefill_inputs(1, 4, 2, 300, 300, d, 15, device="cuda")
    n = q.numel()
    guard = 4096
    o32, l32 = run_fa(q, k, v, True, 0.1)
    obuf = torch.full((n + 2 * guard,), 3.0, device="cuda", dtype=torch.bfloat16)
    o16 = obuf[guard + 8:guard + 8 + n].view(q.shape)  # 16 bytes past a 32-byte boundary
    assert o16.data_ptr() % 32 == 16
    l16 = torch.empty_like(l32)
    fa.fa_fwd(q, k, v, o16, l16, True, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(o32, o16) and torch.equal(l32, l16)
    assert (obuf[:guard + 8] == 3.0).all() and (obuf[guard + 8 + n:] == 3.0).all()


def test_non_default_stream():
    q, k, v = prefill_inputs(2, 4, 4, 256, 256, 64, 9, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, lse = run_fa(q, k, v, False, 0.125, stream=s)
    s.synchronize()
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, False, 0.125)
    eo, el = errors(o, lse, o_ref, lse_ref)
    assert eo <= O_TOL and el <= LSE_TOL


def test_host_buffers_round_trip():
    """The user-level call with host (pinned) tensors copies in and out."""
    q, k, v = prefill_inputs(1, 2, 2, 200, 200, 128, 12)
    q, k, v = (t.pin_memory() for t in (q, k, v))
    o, lse = fa.flash_attention(q, k, v, causal=True)
    assert not o.is_cuda
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, 1.0 / math.sqrt(128))
    eo, el = errors(o, lse, o_ref, lse_ref)
    assert eo <= O_TOL and el <= LSE_TOL


@pytest.mark.parametrize("chunks", [2, 3, 5])
def test_host_buffers_in_chunks_equal_device_call(chunks):
    """Host inputs are cut into groups of key/value heads that are copied in,
    computed and copied out on overlapping streams; every group is its own
    launch, and the result is bit-identical to one launch on device tensors
    (a query tile's computation does not depend on which launch holds it)."""
    q, k, v = prefill_inputs(2, 8, 2, 333, 333, 128, 14)  # 4 key/value heads, G=4
    o_dev, lse_dev = run_fa(q.cuda(), k.cuda(), v.cuda(), True, 0.09)
    torch.cuda.synchronize()
    q, k, v = (t.pin_memory() for t in (q, k, v))
    o_h, lse_h = fa.flash_attention(q, k, v, causal=True, scale=0.09, chunks=chunks)
    assert not o_h.is_cuda
    assert torch.equal(o_h, o_dev.cpu()) and torch.equal(lse_h, lse_dev.cpu())


def tile_rows(Sq, per_tile, rng):
    """`per_tile` query rows drawn from every 128-row tile (the tile's first
    and last rows always among them), so every tile of a head is checked."""
    rows = set()
    for t0 in range(0, Sq, 128):
        t1 = min(Sq, t0 + 128)
        rows.update({t0, t1 - 1})
        rows.update(int(x) for x in rng.integers(t0, t1, max(0, per_tile - 2)))
    return sorted(rows)


def full_size_run(name):
    """The full-size workload in the launch the benchmark times, with the
    properties that hold at any size checked on every row: finite, and each O
    row inside the value range of its head."""
    c = CONFIGS[name]
    q, k, v = prefill_inputs_for(c, device="cuda")
    o, lse = run_fa(q, k, v, c.causal, c.scale)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    grp = c.Hq // c.Hkv
    vmax = v.float().amax(dim=2).repeat_interleave(grp, dim=1)  # [B,Hq,d]
    vmin = v.float().amin(dim=2).repeat_interleave(grp, dim=1)
    of = o.float()
    assert (of <= vmax[:, :, None, :] + O_TOL).all() and (of >= vmin[:, :, None, :] - O_TOL).all()
    return c, q, k, v, o, lse


def check_whole_head(c, q, k, v, o, lse, b, h):
    g = h // (c.Hq // c.Hkv)
    o_ref, lse_ref = oracle.attn_fwd(q[b:b + 1, h:h + 1].cpu(), k[b:b + 1, g:g + 1].cpu(),
                                     v[b:b + 1, g:g + 1].cpu(), c.causal, c.scale)
    eo, el = errors(o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], o_ref, lse_ref)
    assert eo <= O_TOL and el <= LSE_TOL, ("head", b, h, eo, el)


def check_tile_rows(c, q, k, v, o, lse, per_tile, seed):
    """`per_tile` rows of every 128-row tile of every (b, head), one oracle
    call per key/value head (the oracle reads only that head's keys)."""
    rng = np.random.default_rng(seed)
    grp = c.Hq // c.Hkv
    for b in range(c.B):
        for g in range(c.Hkv):
            kb, vb = k[b:b + 1, g:g + 1].cpu(), v[b:b + 1, g:g + 1].cpu()
            rows = [(0, j, i) for j in range(grp) for i in tile_rows(c.Sq, per_tile, rng)]
            hs = torch.tensor([g * grp + j for (_, j, _) in rows], device=q.device)
            ii = torch.tensor([i for (_, _, i) in rows], device=q.device)
            qr = q[b][hs, ii].cpu()
            o_ref, lse_ref = oracle.attn_rows(qr, kb, vb, rows, grp, c.Sq, c.causal, c.scale)
            o_got = o[b][hs, ii].float().cpu()
            l_got = lse[b][hs, ii].cpu()
            eo = float(np.abs(o_got.numpy() - o_ref).max())
            el = float(np.abs(l_got.numpy() - lse_ref).max())
            assert eo <= O_TOL and el <= LSE_TOL, ("tile rows", b, g, eo, el)


def test_full_size_causal_mha_s2048_every_row():
    """Causal MHA B=4 H=16 S=2048 d=128, Q ~ N(0,1)*8: every row of every head
    against the oracle (about a second of fp64 work on the host)."""
    c, q, k, v, o, lse = full_size_run("causal_mha_s2048_d128_qx8")
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, c.causal, c.scale)
    eo, el = errors(o, lse, o_ref, lse_ref)
    assert eo <= O_TOL and el <= LSE_TOL, (eo, el)


def test_full_size_causal_gqa_s8192():
    """Causal GQA B=2 Hq=32 Hkv=8 S=8192 d=128: one whole query head of every
    (batch, key/value head) pair, and 4 rows of every 128-row tile of every
    query head."""
    c, q, k, v, o, lse = full_size_run("causal_gqa_s8192_d128")
    grp = c.Hq // c.Hkv
    for b in range(c.B):
        for g in range(c.Hkv):
            check_whole_head(c, q, k, v, o, lse, b, g * grp + (g + b) % grp)
    check_tile_rows(c, q, k, v, o, lse, 4, seed=c.seed)


def test_full_size_causal_gqa_s32768():
    """Causal GQA B=1 Hq=32 Hkv=8 S=32768 d=128 (the persistent scheduler's
    last round of items holds the first query tiles of the last heads): the
    first query head of key/value head 0 and the last query head of key/value
    head 7 whole, and 4 rows of every 128-row tile of every query head."""
    c, q, k, v, o, lse = full_size_run("causal_gqa_s32768_d128")
    check_whole_head(c, q, k, v, o, lse, 0, 0)
    check_whole_head(c, q, k, v, o, lse, 0, c.Hq - 1)
    check_tile_rows(c, q, k, v, o, lse, 4, seed=c.seed)


def test_timeout_probe_reports_and_context_survives():
    """A bounded wait that nothing completes gives up, records the timeout
    status, and leaves the context usable."""
    assert fa.get_device_status() == 0
    fa.debug_timeout_probe(2000)
    assert fa.get_device_status() == 5
    assert fa.get_device_status() == 0  # read-and-clear
    check_full(1, 2, 2, 130, 130, 64, True, seed=77)
    assert fa.get_device_status() == 0
