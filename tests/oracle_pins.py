"""Checks that pin the fp64 oracle to facts other than itself.

Each ``pin_*`` function takes a loaded oracle library (the real one, or a
mutant built by tests/test_oracle_mutants.py) and raises AssertionError when the
oracle disagrees with:
  * hand-derived closed forms (tests/golden/closed_forms.json);
  * an independent block-wise online-softmax recurrence written here from the
    description in "FlashAttention & IO-aware attention", section "Direct
    answer" (running max m, normaliser l and accumulator O, rescaled by
    e^(m - m_new) whenever the max grows) -- that page states the streamed
    result equals the one-shot softmax;
  * invariants of softmax attention;
  * torch's fp64 scaled_dot_product_attention (an independent implementation);
  * reductions: GQA == MHA with repeated K/V, decode == prefill with one query,
    split + combine == unsplit;
  * for E4M3 inputs: code values derived by hand (tests/golden/e4m3_codes.json),
    torch's float8_e4m3fn decoding, and a one-key closed form per head;
  * for the feed-forward network after attention: textbook values of the normal
    CDF, torch's fp64 GELU network, token independence (blockwise == full) and
    the head-to-token concatenation by hand.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "closed_forms.json")

_MATH_NAMES = {"log": math.log, "exp": math.exp, "inf": math.inf}


def _ev(x):
    """Evaluate a golden expression string ("log(4)", "-inf", "7") with math."""
    if isinstance(x, (int, float)):
        return float(x)
    return float(eval(x, {"__builtins__": {}}, _MATH_NAMES))


def _evarr(a):
    return np.vectorize(_ev, otypes=[np.float64])(np.asarray(a, dtype=object))


def _close(got, want, tol, what):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, f"{what}: shape {got.shape} != {want.shape}"
    both_inf = np.isinf(got) & np.isinf(want) & (np.sign(got) == np.sign(want))
    with np.errstate(invalid="ignore"):
        diff = np.where(both_inf, 0.0, np.abs(got - want))
    diff = np.where(np.isnan(diff), np.inf, diff)
    err = float(diff.max()) if diff.size else 0.0
    assert err <= tol, f"{what}: max abs error {err:.3e} > {tol:.1e}"


def _rand(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


# --------------------------------------------------------------------------
# Independent reference algorithms written for the pins
# --------------------------------------------------------------------------

def online_softmax_attention(q, k, v, causal, scale, block):
    """Block-wise streaming softmax attention in fp64 (per query row, keys in
    blocks of `block`, left to right).  Independent of the C oracle."""
    B, Hq, Sq, d = q.shape
    _, Hkv, Skv, _ = k.shape
    grp = Hq // Hkv
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            kh, vh = k[b, h // grp], v[b, h // grp]
            for i in range(Sq):
                n_vis = Skv if not causal else max(0, min(Skv, i + Skv - Sq + 1))
                m, l = -math.inf, 0.0
                acc = np.zeros(d)
                for j0 in range(0, n_vis, block):
                    j1 = min(n_vis, j0 + block)
                    s = scale * (kh[j0:j1] @ q[b, h, i])
                    m_new = max(m, float(s.max()))
                    shrink = 0.0 if m == -math.inf else math.exp(m - m_new)
                    p = np.exp(s - m_new)
                    l = l * shrink + float(p.sum())
                    acc = acc * shrink + p @ vh[j0:j1]
                    m = m_new
                if n_vis == 0:
                    o[b, h, i] = 0.0
                    lse[b, h, i] = -math.inf
                else:
                    o[b, h, i] = acc / l
                    lse[b, h, i] = m + math.log(l)
    return o, lse


def torch_sdpa_fp64(q, k, v, causal, scale):
    """torch's fp64 CPU scaled_dot_product_attention with K/V repeated per
    query group, a bottom-right causal boolean mask, and LSE from logsumexp."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    grp = tq.shape[1] // tk.shape[1]
    tk = tk.repeat_interleave(grp, dim=1)
    tv = tv.repeat_interleave(grp, dim=1)
    Sq, Skv = tq.shape[2], tk.shape[2]
    mask = None
    if causal:
        i = torch.arange(Sq).unsqueeze(1)
        j = torch.arange(Skv).unsqueeze(0)
        mask = j <= i + (Skv - Sq)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask,
                                                         scale=scale)
    s = (tq @ tk.transpose(-1, -2)) * scale
    if mask is not None:
        s = s.masked_fill(~mask, -math.inf)
    lse = torch.logsumexp(s, dim=-1)
    return o.numpy(), lse.numpy()


# --------------------------------------------------------------------------
# Pins
# --------------------------------------------------------------------------

def pin_golden_prefill(lib):
    cases = json.load(open(GOLDEN))["prefill"]
    for c in cases:
        q, k, v = (np.asarray(c[x], dtype=np.float64) for x in ("q", "k", "v"))
        scale = _ev(c["scale_expr"]) if "scale_expr" in c else float(c["scale"])
        o, lse = oracle.attn_fwd(q, k, v, c["causal"], scale, lib=lib)
        _close(o, _evarr(c["o"]), 1e-12, c["name"] + " O")
        _close(lse, _evarr(c["lse"]), 1e-12, c["name"] + " LSE")


def pin_golden_combine(lib):
    for c in json.load(open(GOLDEN))["combine"]:
        o, lse = oracle.combine(_evarr(c["o_part"]), _evarr(c["lse_part"]), lib=lib)
        _close(o, _evarr(c["o"]), 1e-12, c["name"] + " O")
        _close(lse, _evarr(c["lse"]), 1e-12, c["name"] + " LSE")


def pin_online_equals_one_shot(lib):
    rng = np.random.default_rng(11)
    shapes = [  # B, Hq, Hkv, Sq, Skv, d, causal
        (1, 2, 2, 5, 9, 4, False),
        (2, 4, 2, 7, 7, 3, True),
        (1, 3, 1, 9, 4, 5, True),   # Sq > Skv: leading rows see no key
        (1, 2, 1, 3, 11, 2, True),  # Sq < Skv
    ]
    for (B, Hq, Hkv, Sq, Skv, d, causal) in shapes:
        q = _rand((B, Hq, Sq, d), rng, 2.0)
        k = _rand((B, Hkv, Skv, d), rng)
        v = _rand((B, Hkv, Skv, d), rng)
        scale = 1.0 / math.sqrt(d)
        o, lse = oracle.attn_fwd(q, k, v, causal, scale, lib=lib)
        for blk in (1, 2, 3, 7, 128):
            o2, lse2 = online_softmax_attention(q, k, v, causal, scale, blk)
            _close(o, o2, 1e-12, f"online block={blk} O {B,Hq,Hkv,Sq,Skv,d,causal}")
            _close(lse, lse2, 1e-12, f"online block={blk} LSE")


def pin_invariants(lib):
    rng = np.random.default_rng(12)
    B, Hq, Hkv, S, d = 1, 2, 2, 6, 6
    scale = 0.37
    q = _rand((B, Hq, S, d), rng)
    k = _rand((B, Hkv, S, d), rng)
    # constant V rows -> that row
    row = _rand((d,), rng)
    v = np.broadcast_to(row, (B, Hkv, S, d)).copy()
    for causal in (False, True):
        o, _ = oracle.attn_fwd(q, k, v, causal, scale, lib=lib)
        _close(o, np.broadcast_to(row, o.shape), 1e-12, "constant V rows")
    # identical keys -> mean of V, LSE = s + ln n
    k1 = np.broadcast_to(_rand((d,), rng), (B, Hkv, S, d)).copy()
    v = _rand((B, Hkv, S, d), rng)
    o, lse = oracle.attn_fwd(q, k1, v, False, scale, lib=lib)
    _close(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), 1e-12, "identical keys O")
    s = scale * np.einsum("bhsd,d->bhs", q, k1[0, 0, 0])
    _close(lse, s + math.log(S), 1e-12, "identical keys LSE")
    # V = identity (Skv = d): O rows are the probability rows: >= 0, sum to 1
    eye = np.broadcast_to(np.eye(S), (B, Hkv, S, S)).copy()
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, eye, causal, scale, lib=lib)
        assert (o >= 0).all(), "softmax weights must be non-negative"
        _close(o.sum(-1), np.ones((B, Hq, S)), 1e-12, "softmax rows sum to 1")
        # the weights are exp(s - LSE): check against the scores directly
        sc = scale * np.einsum("bhid,bhjd->bhij", q, k)
        if causal:
            sc = np.where(np.tril(np.ones((S, S), bool)), sc, -np.inf)
        _close(o, np.exp(sc - lse[..., None]), 1e-12, "weights = exp(s - LSE)")
        if causal:
            # masked weights are exactly zero
            assert (o[..., np.triu(np.ones((S, S), bool), 1)] == 0).all()
    # shifting every key by u: LSE shifts by scale*q.u, O unchanged
    u = _rand((d,), rng)
    v = _rand((B, Hkv, S, d), rng)
    o, lse = oracle.attn_fwd(q, k, v, True, scale, lib=lib)
    o2, lse2 = oracle.attn_fwd(q, k + u, v, True, scale, lib=lib)
    _close(o2, o, 1e-12, "key shift O")
    _close(lse2, lse + scale * (q @ u), 1e-12, "key shift LSE")
    # jointly permuting keys and values (no mask) leaves the result unchanged
    perm = rng.permutation(S)
    o, lse = oracle.attn_fwd(q, k, v, False, scale, lib=lib)
    o2, lse2 = oracle.attn_fwd(q, k[:, :, perm], v[:, :, perm], False, scale, lib=lib)
    _close(o2, o, 1e-12, "permutation O")
    _close(lse2, lse, 1e-12, "permutation LSE")
    # causal first row sees key 0 only: O = v_0, LSE = its score
    o, lse = oracle.attn_fwd(q, k, v, True, scale, lib=lib)
    _close(o[:, :, 0], v[:, :, 0], 1e-12, "causal row 0 O")
    _close(lse[:, :, 0], scale * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]), 1e-12,
           "causal row 0 LSE")


def pin_large_logits(lib):
    """Scores of order 1e3..1e4 (Q x 1024): no overflow, and the softmax is
    one-hot on the arg-max key (the gaps between scores are >> 40)."""
    rng = np.random.default_rng(13)
    B, H, S, d = 1, 2, 16, 8
    q = np.round(_rand((B, H, S, d), rng) * 4) * 1024.0
    k = np.round(_rand((B, H, S, d), rng) * 4)
    v = _rand((B, H, S, d), rng)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attn_fwd(q, k, v, False, scale, lib=lib)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), "overflow at large logits"
    s = scale * np.einsum("bhid,bhjd->bhij", q, k)
    srt = np.sort(s, axis=-1)
    gap = srt[..., -1] - srt[..., -2]
    top = s.argmax(-1)
    one_hot = np.take_along_axis(v, top[..., None], axis=2)
    ok = gap > 50.0  # exp(-50) ~ 2e-22: below fp64 resolution of O
    assert ok.any(), "test case lost its large gaps"
    _close(np.where(ok[..., None], o, 0), np.where(ok[..., None], one_hot, 0), 1e-12,
           "one-hot limit O")
    _close(np.where(ok, lse, 0), np.where(ok, srt[..., -1], 0), 1e-9, "one-hot limit LSE")


def pin_torch_sdpa(lib):
    rng = np.random.default_rng(14)
    shapes = [  # B, Hq, Hkv, Sq, Skv, d, causal
        (2, 4, 4, 33, 33, 16, False),
        (2, 4, 4, 33, 33, 16, True),
        (1, 8, 2, 20, 20, 8, True),
        (1, 4, 1, 7, 19, 8, True),
        (1, 4, 2, 19, 7, 8, True),
        (1, 2, 2, 12, 40, 32, False),
    ]
    for (B, Hq, Hkv, Sq, Skv, d, causal) in shapes:
        q = _rand((B, Hq, Sq, d), rng, 3.0)
        k = _rand((B, Hkv, Skv, d), rng)
        v = _rand((B, Hkv, Skv, d), rng)
        scale = 1.0 / math.sqrt(d)
        o, lse = oracle.attn_fwd(q, k, v, causal, scale, lib=lib)
        o2, lse2 = torch_sdpa_fp64(q, k, v, causal, scale)
        # torch returns NaN for rows with no visible key; the oracle's reading
        # is O = 0, LSE = -inf for them.
        empty = np.isneginf(lse2)
        o2 = np.where(empty[..., None], 0.0, o2)
        _close(o, o2, 1e-12, f"sdpa O {B,Hq,Hkv,Sq,Skv,d,causal}")
        _close(lse, lse2, 1e-12, f"sdpa LSE {B,Hq,Hkv,Sq,Skv,d,causal}")


def pin_rows_match_full(lib):
    rng = np.random.default_rng(15)
    B, Hq, Hkv, Sq, Skv, d = 2, 4, 2, 13, 17, 8
    q = _rand((B, Hq, Sq, d), rng)
    k = _rand((B, Hkv, Skv, d), rng)
    v = _rand((B, Hkv, Skv, d), rng)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, causal, 0.3, lib=lib)
        rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in (0, 5, Sq - 1)]
        qr = np.stack([q[b, h, i] for (b, h, i) in rows])
        o2, lse2 = oracle.attn_rows(qr, k, v, rows, Hq, Sq, causal, 0.3, lib=lib)
        _close(o2, np.stack([o[r] for r in rows]), 0.0, "rows O")
        _close(lse2, np.array([lse[r] for r in rows]), 0.0, "rows LSE")


def pin_gqa_equals_repeated_mha(lib):
    rng = np.random.default_rng(16)
    B, Hq, Hkv, S, d = 2, 8, 2, 9, 4
    q = _rand((B, Hq, S, d), rng)
    k = _rand((B, Hkv, S, d), rng)
    v = _rand((B, Hkv, S, d), rng)
    rep_k = np.repeat(k, Hq // Hkv, axis=1)
    rep_v = np.repeat(v, Hq // Hkv, axis=1)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, causal, 0.5, lib=lib)
        o2, lse2 = oracle.attn_fwd(q, rep_k, rep_v, causal, 0.5, lib=lib)
        _close(o, o2, 0.0, "GQA O")
        _close(lse, lse2, 0.0, "GQA LSE")
        # and each query head against its own explicit kv head
        for h in range(Hq):
            o3, _ = oracle.attn_fwd(q[:, h:h + 1], k[:, h // (Hq // Hkv)][:, None],
                                    v[:, h // (Hq // Hkv)][:, None], causal, 0.5, lib=lib)
            _close(o[:, h:h + 1], o3, 0.0, f"GQA head {h}")


def _decode_case(rng, B=3, Hq=4, Hkv=2, Lmax=23, d=8, lens=(23, 1, 10)):
    q = _rand((B, Hq, d), rng)
    kc = _rand((B, Hkv, Lmax, d), rng)
    vc = _rand((B, Hkv, Lmax, d), rng)
    sl = np.asarray(lens, dtype=np.int32)
    return q, kc, vc, sl


def pin_decode_equals_prefill(lib):
    rng = np.random.default_rng(17)
    q, kc, vc, sl = _decode_case(rng)
    # cache positions beyond a sequence's length must never be read
    for b, L in enumerate(sl):
        kc[b, :, L:] = np.nan
        vc[b, :, L:] = np.nan
    o, lse = oracle.decode(q, kc, vc, sl, 0.25, lib=lib)
    for b, L in enumerate(sl):
        o2, lse2 = oracle.attn_fwd(q[b:b + 1, :, None], kc[b:b + 1, :, :L], vc[b:b + 1, :, :L],
                                   False, 0.25, lib=lib)
        _close(o[b], o2[0, :, 0], 0.0, f"decode O b={b}")
        _close(lse[b], lse2[0, :, 0], 0.0, f"decode LSE b={b}")


def pin_split_combine_equals_unsplit(lib):
    rng = np.random.default_rng(18)
    q, kc, vc, sl = _decode_case(rng, lens=(23, 1, 10))
    o, lse = oracle.decode(q, kc, vc, sl, 0.25, lib=lib)
    for n in (1, 2, 3, 5, 7, 30):  # 30 > every length: empty chunks occur
        op, lp = oracle.split_partials(q, kc, vc, sl, n, 0.25, lib=lib)
        o2, lse2 = oracle.combine(op, lp, lib=lib)
        _close(o2, o, 1e-12, f"split {n} O")
        _close(lse2, lse, 1e-12, f"split {n} LSE")
        # chunk c of sequence b covers [c*cs, min(L,(c+1)*cs)), cs = ceil(L/n)
        for b, L in enumerate(sl):
            cs = -(-int(L) // n)
            for c in range(n):
                lo, hi = min(L, c * cs), min(L, (c + 1) * cs)
                if hi <= lo:
                    assert np.isneginf(lp[b, :, c]).all() and (op[b, :, c] == 0).all(), \
                        "empty chunk must give lse=-inf, o=0"
                else:
                    o3, l3 = oracle.attn_fwd(q[b:b + 1, :, None], kc[b:b + 1, :, lo:hi],
                                             vc[b:b + 1, :, lo:hi], False, 0.25, lib=lib)
                    _close(op[b, :, c], o3[0, :, 0], 1e-12, f"chunk {b},{c} O")
                    _close(lp[b, :, c], l3[0, :, 0], 1e-12, f"chunk {b},{c} LSE")


def pin_paged_gather_by_hand(lib):
    """Block-table indirection on a case worked by hand: page size 2, three
    physical pages, one sequence of 5 keys whose logical pages are physical
    pages 2, 0, 1."""
    kp = np.zeros((3, 1, 2, 1))
    vp = np.zeros((3, 1, 2, 1))
    for page in range(3):
        for row in range(2):
            kp[page, 0, row, 0] = 10 * page + row      # key value names its page and row
            vp[page, 0, row, 0] = -(10 * page + row)
    bt = np.array([[2, 0, 1]])
    kc, vc = oracle.paged_gather(kp, vp, bt, np.array([5]))
    # logical keys 0,1 <- page 2 rows 0,1; keys 2,3 <- page 0; key 4 <- page 1 row 0
    assert kc[0, 0, :5, 0].tolist() == [20, 21, 0, 1, 10], kc[0, 0, :, 0]
    assert vc[0, 0, :5, 0].tolist() == [-20, -21, 0, -1, -10]
    assert np.isnan(kc[0, 0, 5:]).all(), "rows past the sequence must stay unread (NaN)"


def pin_paged_decode_equals_contiguous(lib):
    """A contiguous cache cut into pages, scattered by a random permutation and
    read back through the block table, decodes exactly as the contiguous one."""
    rng = np.random.default_rng(19)
    B, Hq, Hkv, P, d = 3, 4, 2, 4, 8
    max_pages = 6
    q = _rand((B, Hq, d), rng)
    kc = _rand((B, Hkv, max_pages * P, d), rng)
    vc = _rand((B, Hkv, max_pages * P, d), rng)
    sl = np.array([24, 1, 13], dtype=np.int32)
    perm = rng.permutation(B * max_pages)
    kp = np.zeros((B * max_pages, Hkv, P, d))
    vp = np.zeros((B * max_pages, Hkv, P, d))
    bt = np.zeros((B, max_pages), dtype=np.int32)
    for b in range(B):
        for j in range(max_pages):
            phys = int(perm[b * max_pages + j])
            bt[b, j] = phys
            kp[phys] = kc[b, :, j * P:(j + 1) * P]
            vp[phys] = vc[b, :, j * P:(j + 1) * P]
    o, lse = oracle.decode(q, kc, vc, sl, 0.3, lib=lib)
    o2, lse2 = oracle.decode_paged(q, kp, vp, bt, sl, 0.3, lib=lib)
    _close(o2, o, 0.0, "paged O")
    _close(lse2, lse, 0.0, "paged LSE")


def pin_aligned_split(lib):
    """Chunk sizes rounded up to a multiple of align: partials merge to the
    unsplit decode, every chunk is the one-shot softmax over its own keys,
    and align = 1 is the plain split rule."""
    rng = np.random.default_rng(20)
    q, kc, vc, sl = _decode_case(rng, Lmax=40, lens=(40, 3, 17))
    o, lse = oracle.decode(q, kc, vc, sl, 0.25, lib=lib)
    for n in (1, 2, 3, 7):
        a1 = oracle.split_partials_aligned(q, kc, vc, sl, n, 1, 0.25, lib=lib)
        a0 = oracle.split_partials(q, kc, vc, sl, n, 0.25, lib=lib)
        _close(a1[0], a0[0], 0.0, "align 1 O")
        _close(a1[1], a0[1], 0.0, "align 1 LSE")
        for align in (4, 8, 16):
            op, lp = oracle.split_partials_aligned(q, kc, vc, sl, n, align, 0.25, lib=lib)
            o2, lse2 = oracle.combine(op, lp, lib=lib)
            _close(o2, o, 1e-12, f"aligned split {n}/{align} O")
            _close(lse2, lse, 1e-12, f"aligned split {n}/{align} LSE")
            for b, L in enumerate(sl):
                cs = -(-(-(-int(L) // n)) // align) * align
                assert cs % align == 0
                for c in range(n):
                    lo, hi = min(L, c * cs), min(L, (c + 1) * cs)
                    if hi <= lo:
                        assert np.isneginf(lp[b, :, c]).all() and (op[b, :, c] == 0).all()
                    else:
                        o3, l3 = oracle.attn_fwd(q[b:b + 1, :, None], kc[b:b + 1, :, lo:hi],
                                                 vc[b:b + 1, :, lo:hi], False, 0.25, lib=lib)
                        _close(op[b, :, c], o3[0, :, 0], 1e-12, f"chunk {b},{c} O")
                        _close(lp[b, :, c], l3[0, :, 0], 1e-12, f"chunk {b},{c} LSE")


def _loss(q, k, v, d_o, causal, scale, lib):
    o, _ = oracle.attn_fwd(q, k, v, causal, scale, lib=lib)
    return float(np.sum(o * d_o))


def pin_bwd_finite_differences(lib):
    """Each gradient the backward oracle returns matches a central finite
    difference of L = sum(O * dO) through the forward oracle (a different
    code path: only the forward definition is shared)."""
    rng = np.random.default_rng(21)
    for (B, Hq, Hkv, Sq, Skv, d, causal) in ((1, 4, 2, 7, 9, 5, True), (1, 2, 2, 6, 6, 4, False),
                                             (2, 2, 1, 5, 3, 3, True)):
        q = _rand((B, Hq, Sq, d), rng, 1.5)
        k = _rand((B, Hkv, Skv, d), rng)
        v = _rand((B, Hkv, Skv, d), rng)
        d_o = _rand((B, Hq, Sq, d), rng)
        scale = 0.7
        grads = oracle.attn_bwd(q, k, v, d_o, causal, scale, lib=lib)
        eps = 1e-5
        for which, (x, g) in enumerate(zip((q, k, v), grads)):
            flat = x.reshape(-1)
            for idx in rng.choice(flat.size, size=min(12, flat.size), replace=False):
                keep = flat[idx]
                flat[idx] = keep + eps
                lp = _loss(q, k, v, d_o, causal, scale, lib)
                flat[idx] = keep - eps
                lm = _loss(q, k, v, d_o, causal, scale, lib)
                flat[idx] = keep
                fd = (lp - lm) / (2 * eps)
                got = g.reshape(-1)[idx]
                assert abs(fd - got) <= 1e-7 * (1 + abs(fd)), \
                    f"grad {'qkv'[which]}[{idx}] {got} vs finite difference {fd}"


def pin_bwd_torch_autograd(lib):
    """torch fp64 autograd through scaled_dot_product_attention (K/V repeated
    per group, explicit bottom-right mask) gives the same gradients."""
    rng = np.random.default_rng(22)
    for (B, Hq, Hkv, Sq, Skv, d, causal) in ((2, 4, 4, 17, 17, 8, True), (1, 8, 2, 20, 20, 8, True),
                                             (1, 4, 2, 19, 7, 8, True), (1, 2, 2, 12, 30, 16, False),
                                             (1, 4, 1, 7, 19, 8, True)):
        q = _rand((B, Hq, Sq, d), rng, 2.0)
        k = _rand((B, Hkv, Skv, d), rng)
        v = _rand((B, Hkv, Skv, d), rng)
        d_o = _rand((B, Hq, Sq, d), rng)
        scale = 1.0 / math.sqrt(d)
        dq, dk, dv = oracle.attn_bwd(q, k, v, d_o, causal, scale, lib=lib)
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        grp = Hq // Hkv
        mask = None
        if causal:
            i = torch.arange(Sq).unsqueeze(1)
            j = torch.arange(Skv).unsqueeze(0)
            mask = j <= i + (Skv - Sq)
        s = (tq @ tk.repeat_interleave(grp, 1).transpose(-1, -2)) * scale
        if mask is not None:
            s = s.masked_fill(~mask, -math.inf)
        pr = torch.softmax(s, dim=-1)
        pr = torch.nan_to_num(pr, nan=0.0)  # rows with no visible key contribute nothing
        o = pr @ tv.repeat_interleave(grp, 1)
        o.backward(torch.tensor(d_o))
        _close(dq, tq.grad.numpy(), 1e-10, "dq vs autograd")
        _close(dk, tk.grad.numpy(), 1e-10, "dk vs autograd")
        _close(dv, tv.grad.numpy(), 1e-10, "dv vs autograd")


def pin_bwd_single_key(lib):
    """One visible key: O = v_0 whatever q and k are, so dq = dk = 0 and
    dv_0 = sum over query rows of dO."""
    rng = np.random.default_rng(23)
    q = _rand((1, 3, 4, 5), rng)
    k = _rand((1, 1, 1, 5), rng)
    v = _rand((1, 1, 1, 5), rng)
    d_o = _rand((1, 3, 4, 5), rng)
    dq, dk, dv = oracle.attn_bwd(q, k, v, d_o, False, 0.9, lib=lib)
    _close(dq, np.zeros_like(dq), 1e-14, "dq single key")
    _close(dk, np.zeros_like(dk), 1e-14, "dk single key")
    _close(dv[0, 0, 0], d_o.sum(axis=(0, 1, 2)), 1e-13, "dv single key")


# --------------------------------------------------------------------------
# E4M3 inputs
E4M3_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "e4m3_codes.json")


def _torch_e4m3(codes):
    """torch's own float8_e4m3fn decoding (an independent implementation)."""
    c = torch.as_tensor(np.asarray(codes, dtype=np.uint8))
    return c.view(torch.float8_e4m3fn).double().numpy()


def pin_e4m3_golden(lib):
    """Single codes whose values were derived by hand from the E4M3 definition."""
    table = json.load(open(E4M3_GOLDEN))["codes"]
    codes = np.array([c for c, _ in table], dtype=np.uint8)
    got = oracle.e4m3_decode(codes, lib=lib)
    for (c, want), g in zip(table, got):
        if want is None:
            assert np.isnan(g), f"code {c}: {g} is not NaN"
        else:
            assert g == want and math.copysign(1.0, g) == math.copysign(1.0, want), \
                f"code {c}: {g} != {want}"


def pin_e4m3_matches_torch(lib):
    """All 256 codes agree with torch's float8_e4m3fn conversion (NaN with NaN)."""
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes, lib=lib)
    want = _torch_e4m3(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want)), "NaN codes differ"
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok]), "E4M3 values differ from torch"


def pin_e4m3_order_and_sign(lib):
    """Codes 0..126 are strictly increasing and setting bit 7 negates."""
    pos = oracle.e4m3_decode(np.arange(127, dtype=np.uint8), lib=lib)
    neg = oracle.e4m3_decode(np.arange(128, 255, dtype=np.uint8), lib=lib)
    assert np.all(np.diff(pos) > 0), "E4M3 codes not monotone"
    assert np.array_equal(neg, -pos), "sign bit does not negate"


def pin_fp8_one_key_closed_form(lib):
    """One key per head: O = dv * v_0 and LSE = scale * dq * dk * (q . k_0), with
    the factors of the query's key/value head (GQA group) in its own batch."""
    rng = np.random.default_rng(31)
    B, Hq, Hkv, Sq, d = 2, 4, 2, 3, 5

    def codes(shape):  # finite codes of either sign
        c = rng.integers(0, 127, size=shape).astype(np.uint8)
        return np.where(rng.random(shape) < 0.5, c | 0x80, c).astype(np.uint8)

    q8, k8, v8 = codes((B, Hq, Sq, d)), codes((B, Hkv, 1, d)), codes((B, Hkv, 1, d))
    dq, dk, dv = (rng.uniform(0.25, 4.0, size=(B, Hkv)) for _ in range(3))
    scale = 0.3
    o, lse = oracle.attn_fwd_fp8(q8, k8, v8, dq, dk, dv, False, scale, lib=lib)
    qv, kv, vv = _torch_e4m3(q8), _torch_e4m3(k8), _torch_e4m3(v8)
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(Sq):
                want_l = scale * dq[b, g] * dk[b, g] * float(qv[b, h, i] @ kv[b, g, 0])
                _close(lse[b, h, i], want_l, 1e-12 * max(1.0, abs(want_l)), "fp8 one-key LSE")
                _close(o[b, h, i], dv[b, g] * vv[b, g, 0], 1e-12, "fp8 one-key O")


# --------------------------------------------------------------------------
# Feed-forward network after attention (blockwise parallel transformer)

def pin_ffn_gelu_closed_forms(lib):
    """D = F = 1 with unit weights: y = gelu(x) = x * Phi(x).  Phi(1) and
    Phi(2) are the textbook values of the standard normal CDF; gelu(0) = 0;
    gelu(x) - gelu(-x) = x; gelu(x) -> x for large x."""
    xs = np.array([0.0, 1.0, -1.0, 2.0, -2.0, 10.0, 0.5, -0.5]).reshape(-1, 1)
    y = oracle.ffn(xs, np.ones((1, 1)), np.ones((1, 1)), lib=lib).ravel()
    phi1, phi2 = 0.8413447460685429, 0.9772498680518208
    _close(y[0], 0.0, 1e-15, "gelu(0)")
    _close(y[1], phi1, 1e-15, "gelu(1)")
    _close(y[2], -(1.0 - phi1), 1e-15, "gelu(-1)")
    _close(y[3], 2.0 * phi2, 1e-15, "gelu(2)")
    _close(y[4], -2.0 * (1.0 - phi2), 1e-15, "gelu(-2)")
    _close(y[5], 10.0, 1e-14, "gelu(10)")
    _close(y[6] - y[7], 0.5, 1e-15, "gelu(x) - gelu(-x) = x")


def pin_ffn_torch(lib):
    """torch's fp64 GELU (erf form) between two bias-free linear maps."""
    rng = np.random.default_rng(41)
    for n, D, F in ((7, 16, 40), (1, 3, 5), (20, 8, 32)):
        x = _rand((n, D), rng)
        w1 = _rand((F, D), rng, 0.3)
        w2 = _rand((D, F), rng, 0.3)
        y = oracle.ffn(x, w1, w2, lib=lib)
        tx, t1, t2 = (torch.tensor(a) for a in (x, w1, w2))
        want = (torch.nn.functional.gelu(tx @ t1.T) @ t2.T).numpy()
        _close(y, want, 1e-12, "ffn vs torch (n=%d D=%d F=%d)" % (n, D, F))


def pin_ffn_hidden(lib):
    """The hidden activations: torch's fp64 gelu(x W1^T), and the second map
    applied to them gives the network's output."""
    rng = np.random.default_rng(47)
    x = _rand((9, 16), rng)
    w1, w2 = _rand((24, 16), rng, 0.3), _rand((16, 24), rng, 0.3)
    h = oracle.ffn_hidden(x, w1, lib=lib)
    want = torch.nn.functional.gelu(torch.tensor(x) @ torch.tensor(w1).T).numpy()
    _close(h, want, 1e-13, "ffn hidden vs torch")
    _close(h @ w2.T, oracle.ffn(x, w1, w2, lib=lib), 1e-13, "ffn = W2 hidden")


def pin_ffn_tokens_independent(lib):
    """The property blockwise scheduling rests on ("I/O-Aware Kernels",
    section "Blockwise Parallel Transformers"): each token's output depends on
    that token alone, so blocks of any size, in any order, give the full result."""
    rng = np.random.default_rng(43)
    x = _rand((2, 23, 12), rng)
    w1, w2 = _rand((30, 12), rng, 0.4), _rand((12, 30), rng, 0.4)
    full = oracle.ffn(x, w1, w2, lib=lib)
    for blk in (1, 3, 7, 23):
        parts = [oracle.ffn(x[:, s:s + blk], w1, w2, lib=lib) for s in range(0, 23, blk)]
        _close(np.concatenate(parts, axis=1), full, 1e-15, "blockwise FFN (block %d)" % blk)
    perm = rng.permutation(23)
    _close(oracle.ffn(x[:, perm], w1, w2, lib=lib), full[:, perm], 1e-15, "token permutation")


def pin_heads_to_tokens_by_hand(lib):
    """Token t's row is (O[b,0,t,:], O[b,1,t,:], ...), written out by hand."""
    o = np.arange(1 * 2 * 3 * 2, dtype=np.float64).reshape(1, 2, 3, 2)
    want = np.array([[[0, 1, 6, 7], [2, 3, 8, 9], [4, 5, 10, 11]]], dtype=np.float64)
    got = oracle.heads_to_tokens(o)
    assert np.array_equal(got, want), got
    y, o2, _ = oracle.bpt_layer(np.ones((1, 2, 3, 2)), np.ones((1, 1, 3, 2)),
                                o[:, :1], np.eye(4), np.eye(4), False, 1.0, lib=lib)
    # equal scores: every query's O is the mean of V's rows; FFN = gelu with identity weights
    mean_v = o[0, 0].mean(axis=0)
    _close(o2[0, 1, 2], mean_v, 1e-15, "bpt attention part")
    phi = 0.5 * (1.0 + np.array([math.erf(m / math.sqrt(2.0)) for m in mean_v]))
    _close(y[0, 2], np.concatenate([mean_v * phi] * 2), 1e-14, "bpt layer with identity FFN")


ALL_PINS = [
    pin_golden_prefill,
    pin_golden_combine,
    pin_online_equals_one_shot,
    pin_invariants,
    pin_large_logits,
    pin_torch_sdpa,
    pin_rows_match_full,
    pin_gqa_equals_repeated_mha,
    pin_decode_equals_prefill,
    pin_split_combine_equals_unsplit,
    pin_paged_gather_by_hand,
    pin_paged_decode_equals_contiguous,
    pin_aligned_split,
    pin_bwd_finite_differences,
    pin_bwd_torch_autograd,
    pin_bwd_single_key,
    pin_e4m3_golden,
    pin_e4m3_matches_torch,
    pin_e4m3_order_and_sign,
    pin_fp8_one_key_closed_form,
    pin_ffn_gelu_closed_forms,
    pin_ffn_torch,
    pin_ffn_hidden,
    pin_ffn_tokens_independent,
    pin_heads_to_tokens_by_hand,
]
