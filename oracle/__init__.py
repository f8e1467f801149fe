"""fp64 CPU attention oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
shares no code with the CUDA library: the arithmetic lives in
``attn_oracle.c`` (plain C, fp64, OpenMP over rows), this module only builds
that file with gcc and marshals numpy arrays through ctypes.

What it computes (see ``attn_oracle.c`` for the per-function citations):
the one-shot, materialising softmax attention of "I/O-Aware Kernels", section
"The Memory Bottleneck", with scores scaled as in "FlashAttention & IO-aware
attention", section "Code", and LSE = max + ln(sum of exp).  A paged cache is
read through its block table by ``paged_gather`` (plain index loops, no
arithmetic) and then decoded like a contiguous one.  E4M3 inputs are decoded
from the format's definition and scaled per (batch, key/value head)
(``e4m3_decode``, ``dequant_heads``, ``attn_fwd_fp8``).  The feed-forward
network after attention of "I/O-Aware Kernels", section "Blockwise Parallel
Transformers", is ``ffn`` / ``ffn_hidden`` on the head-concatenated tokens
(``heads_to_tokens``); ``bpt_layer`` is attention followed by it.

Parity pins (tests/test_oracle_pins.py): closed-form golden cases, an
independent online-softmax recurrence, invariants, torch fp64 SDPA on small
shapes, GQA/decode/split reductions, the E4M3 decoding by hand and against
torch's float8 conversion, the per-head dequantisation in closed form, and
the feed-forward network against normal-CDF values, torch's fp64 GELU network
and token independence.
Every function here is pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_attn_oracle.so")
_lib: Optional[ctypes.CDLL] = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.POINTER(ctypes.c_int64)
_U8 = ctypes.POINTER(ctypes.c_uint8)


def build(src: str = _SRC, out: str = _LIB_PATH, force: bool = False) -> str:
    """Compile the C oracle into a shared object (gcc, -O2, no fast-math)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    ci = ctypes.c_int
    lib.oracle_attn_fwd.argtypes = [_D, _D, _D, _D, _D] + [ci] * 7 + [ctypes.c_double]
    lib.oracle_attn_fwd.restype = ci
    lib.oracle_attn_rows.argtypes = ([_D, _D, _D, _I64, ctypes.c_int64, _D, _D]
                                     + [ci] * 7 + [ctypes.c_double])
    lib.oracle_attn_rows.restype = ci
    lib.oracle_decode.argtypes = [_D, _D, _D, _I32, _D, _D] + [ci] * 5 + [ctypes.c_double]
    lib.oracle_decode.restype = ci
    lib.oracle_split_partials.argtypes = ([_D, _D, _D, _I32, _D, _D] + [ci] * 6
                                          + [ctypes.c_double])
    lib.oracle_split_partials.restype = ci
    lib.oracle_split_partials_aligned.argtypes = ([_D, _D, _D, _I32, _D, _D] + [ci] * 7
                                                  + [ctypes.c_double])
    lib.oracle_split_partials_aligned.restype = ci
    lib.oracle_attn_bwd.argtypes = [_D] * 7 + [ci] * 7 + [ctypes.c_double]
    lib.oracle_attn_bwd.restype = ci
    lib.oracle_combine.argtypes = [_D, _D, _D, _D] + [ci] * 4
    lib.oracle_combine.restype = ci
    lib.oracle_e4m3_decode.argtypes = [_U8, ctypes.c_int64, _D]
    lib.oracle_e4m3_decode.restype = ci
    lib.oracle_dequant_heads.argtypes = [_U8, _D, _D] + [ci] * 5
    lib.oracle_dequant_heads.restype = ci
    lib.oracle_ffn_hidden.argtypes = [_D, _D, _D, ctypes.c_int64, ci, ci]
    lib.oracle_ffn_hidden.restype = ci
    lib.oracle_ffn.argtypes = [_D, _D, _D, _D, ctypes.c_int64, ci, ci]
    lib.oracle_ffn.restype = ci
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ci
    return lib


def _f64(a) -> np.ndarray:
    """Exact conversion to a contiguous float64 array (bf16 and fp32 values are
    exactly representable in fp64)."""
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a: np.ndarray, t=_D):
    return a.ctypes.data_as(t)


def attn_fwd(q, k, v, causal: bool, scale: float, lib: Optional[ctypes.CDLL] = None):
    """O [B,Hq,Sq,d] and LSE [B,Hq,Sq] (float64) of softmax(scale*QK^T [+mask]) V.

    q: [B,Hq,Sq,d]; k, v: [B,Hkv,Skv,d]."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Sq, d = q.shape
    _, Hkv, Skv, _ = k.shape
    o = np.zeros((B, Hq, Sq, d))
    lse = np.zeros((B, Hq, Sq))
    rc = lib.oracle_attn_fwd(_p(q), _p(k), _p(v), _p(o), _p(lse), B, Hq, Hkv, Sq,
                             Skv, d, int(bool(causal)), float(scale))
    if rc != 0:
        raise ValueError("oracle_attn_fwd rejected its arguments")
    return o, lse


def attn_bwd(q, k, v, d_o, causal: bool, scale: float, lib: Optional[ctypes.CDLL] = None):
    """Gradients (dq, dk, dv) in float64 of the forward above for dL/dO = d_o."""
    lib = lib or load()
    q, k, v, d_o = _f64(q), _f64(k), _f64(v), _f64(d_o)
    B, Hq, Sq, d = q.shape
    _, Hkv, Skv, _ = k.shape
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    rc = lib.oracle_attn_bwd(_p(q), _p(k), _p(v), _p(d_o), _p(dq), _p(dk), _p(dv), B, Hq, Hkv,
                             Sq, Skv, d, int(bool(causal)), float(scale))
    if rc != 0:
        raise ValueError("oracle_attn_bwd rejected its arguments")
    return dq, dk, dv


def attn_rows(q_rows, k, v, rows: Sequence[Sequence[int]], Hq: int, Sq: int,
              causal: bool, scale: float, lib: Optional[ctypes.CDLL] = None):
    """Selected output rows.  q_rows[n, d] are the query rows named by
    rows[n] = (b, h, i); k, v are the full [B,Hkv,Skv,d] key/value tensors."""
    lib = lib or load()
    q_rows, k, v = _f64(q_rows), _f64(k), _f64(v)
    B, Hkv, Skv, d = k.shape
    idx = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = idx.shape[0]
    o = np.zeros((n, d))
    lse = np.zeros((n,))
    rc = lib.oracle_attn_rows(_p(q_rows), _p(k), _p(v), _p(idx, _I64), n, _p(o),
                              _p(lse), B, Hq, Hkv, Sq, Skv, d, int(bool(causal)),
                              float(scale))
    if rc != 0:
        raise ValueError("oracle_attn_rows rejected its arguments")
    return o, lse


def decode(q, k_cache, v_cache, seqlens, scale: float, lib: Optional[ctypes.CDLL] = None):
    """Single-query decode: q [B,Hq,d], caches [B,Hkv,Lmax,d], seqlens [B]."""
    lib = lib or load()
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    sl = np.ascontiguousarray(np.asarray(
        seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens, dtype=np.int32))
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = kc.shape
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    rc = lib.oracle_decode(_p(q), _p(kc), _p(vc), _p(sl, _I32), _p(o), _p(lse), B, Hq,
                           Hkv, Lmax, d, float(scale))
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return o, lse


def split_partials(q, k_cache, v_cache, seqlens, num_splits: int, scale: float,
                   lib: Optional[ctypes.CDLL] = None):
    """Per-chunk normalised outputs [B,Hq,n,d] and chunk LSEs [B,Hq,n]."""
    lib = lib or load()
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    sl = np.ascontiguousarray(np.asarray(
        seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens, dtype=np.int32))
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = kc.shape
    o = np.zeros((B, Hq, num_splits, d))
    lse = np.zeros((B, Hq, num_splits))
    rc = lib.oracle_split_partials(_p(q), _p(kc), _p(vc), _p(sl, _I32), _p(o), _p(lse),
                                   B, Hq, Hkv, Lmax, d, int(num_splits), float(scale))
    if rc != 0:
        raise ValueError("oracle_split_partials rejected its arguments")
    return o, lse


def split_partials_aligned(q, k_cache, v_cache, seqlens, num_splits: int, align: int,
                           scale: float, lib: Optional[ctypes.CDLL] = None):
    """Split partials with chunk sizes rounded up to a multiple of ``align``."""
    lib = lib or load()
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    sl = np.ascontiguousarray(np.asarray(
        seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens, dtype=np.int32))
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = kc.shape
    o = np.zeros((B, Hq, num_splits, d))
    lse = np.zeros((B, Hq, num_splits))
    rc = lib.oracle_split_partials_aligned(_p(q), _p(kc), _p(vc), _p(sl, _I32), _p(o), _p(lse),
                                           B, Hq, Hkv, Lmax, d, int(num_splits), int(align),
                                           float(scale))
    if rc != 0:
        raise ValueError("oracle_split_partials_aligned rejected its arguments")
    return o, lse


def paged_gather(k_pages, v_pages, block_table, seqlens):
    """Contiguous caches [B,Hkv,max_pages*P,d] (float64) from paged caches.

    k_pages, v_pages: [num_pages, Hkv, P, d]; block_table: [B, max_pages] int.
    Key t of sequence b is row t % P of physical page block_table[b, t // P]
    (the block-table indirection of paged KV management, which "I/O-Aware
    Kernels", section "FlashAttention", names through PagedAttention).  Rows
    at or past seqlens[b] are NaN: nothing may read them.  Data movement
    only: plain loops, no arithmetic."""
    kp, vp = _f64(k_pages), _f64(v_pages)
    bt = np.asarray(block_table.cpu().numpy() if hasattr(block_table, "cpu") else block_table)
    sl = np.asarray(seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens)
    num_pages, Hkv, P, d = kp.shape
    B, max_pages = bt.shape
    kc = np.full((B, Hkv, max_pages * P, d), np.nan)
    vc = np.full((B, Hkv, max_pages * P, d), np.nan)
    for b in range(B):
        L = int(sl[b])
        if L < 0 or L > max_pages * P:
            raise ValueError("sequence length outside the block table")
        for t in range(L):
            page = int(bt[b, t // P])
            if not 0 <= page < num_pages:
                raise ValueError("block table names a page that does not exist")
            kc[b, :, t] = kp[page, :, t % P]
            vc[b, :, t] = vp[page, :, t % P]
    return kc, vc


def decode_paged(q, k_pages, v_pages, block_table, seqlens, scale: float,
                 lib: Optional[ctypes.CDLL] = None):
    """Single-query decode over a paged cache: the decode of the gathered cache."""
    kc, vc = paged_gather(k_pages, v_pages, block_table, seqlens)
    return decode(q, kc, vc, seqlens, scale, lib=lib)


def combine(o_part, lse_part, lib: Optional[ctypes.CDLL] = None):
    """Merge split partials o_part [B,Hq,n,d], lse_part [B,Hq,n]."""
    lib = lib or load()
    op, lp = _f64(o_part), _f64(lse_part)
    B, Hq, n, d = op.shape
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    rc = lib.oracle_combine(_p(op), _p(lp), _p(o), _p(lse), B, Hq, n, d)
    if rc != 0:
        raise ValueError("oracle_combine rejected its arguments")
    return o, lse


def _codes(a) -> np.ndarray:
    """E4M3 codes as a contiguous uint8 array (torch float8 tensors are viewed
    as bytes, never converted)."""
    if hasattr(a, "detach"):
        import torch
        a = a.detach().to("cpu").contiguous()
        if a.element_size() != 1:
            raise TypeError("expected one byte per element")
        a = a.view(torch.uint8).numpy()
    a = np.asarray(a)
    if a.dtype != np.uint8:
        raise TypeError("expected uint8 codes")
    return np.ascontiguousarray(a)


def e4m3_decode(codes, lib: Optional[ctypes.CDLL] = None) -> np.ndarray:
    """float64 values of E4M3 codes (any shape)."""
    lib = lib or load()
    c = _codes(codes)
    out = np.zeros(c.shape)
    if lib.oracle_e4m3_decode(_p(c, _U8), c.size, _p(out)) != 0:
        raise ValueError("oracle_e4m3_decode rejected its arguments")
    return out


def dequant_heads(x8, descale, Hkv: int, lib: Optional[ctypes.CDLL] = None) -> np.ndarray:
    """Real values [B,H,S,d] of E4M3 codes x8 [B,H,S,d]: head h of batch b is
    scaled by descale[b, h // (H // Hkv)]; descale None means 1."""
    lib = lib or load()
    c = _codes(x8)
    B, H, S, d = c.shape
    out = np.zeros(c.shape)
    ds = None if descale is None else _f64(descale).reshape(-1)
    if ds is not None and ds.size != B * Hkv:
        raise ValueError("descale must hold B * Hkv factors")
    rc = lib.oracle_dequant_heads(_p(c, _U8), None if ds is None else _p(ds), _p(out), B, H,
                                  Hkv, S, d)
    if rc != 0:
        raise ValueError("oracle_dequant_heads rejected its arguments")
    return out


def attn_fwd_fp8(q8, k8, v8, descale_q, descale_k, descale_v, causal: bool, scale: float,
                 lib: Optional[ctypes.CDLL] = None):
    """O and LSE (float64) of the attention of the dequantised E4M3 inputs."""
    lib = lib or load()
    Hkv = int(k8.shape[1])
    q = dequant_heads(q8, descale_q, Hkv, lib)
    k = dequant_heads(k8, descale_k, Hkv, lib)
    v = dequant_heads(v8, descale_v, Hkv, lib)
    return attn_fwd(q, k, v, causal, scale, lib=lib)


def ffn(x, w1, w2, lib: Optional[ctypes.CDLL] = None) -> np.ndarray:
    """y [..., D] = W2 gelu(W1 x) per token (x [..., D], w1 [F, D], w2 [D, F])."""
    lib = lib or load()
    x, w1, w2 = _f64(x), _f64(w1), _f64(w2)
    F, D = w1.shape
    if w2.shape != (D, F) or x.shape[-1] != D:
        raise ValueError("ffn: x [..., D], w1 [F, D], w2 [D, F]")
    xs = np.ascontiguousarray(x.reshape(-1, D))
    y = np.zeros(xs.shape)
    if lib.oracle_ffn(_p(xs), _p(w1), _p(w2), _p(y), xs.shape[0], D, F) != 0:
        raise ValueError("oracle_ffn rejected its arguments")
    return y.reshape(x.shape)


def ffn_hidden(x, w1, lib: Optional[ctypes.CDLL] = None) -> np.ndarray:
    """The activations between the two maps: gelu(W1 x) [..., F] per token."""
    lib = lib or load()
    x, w1 = _f64(x), _f64(w1)
    F, D = w1.shape
    if x.shape[-1] != D:
        raise ValueError("ffn_hidden: x [..., D], w1 [F, D]")
    xs = np.ascontiguousarray(x.reshape(-1, D))
    h = np.zeros((xs.shape[0], F))
    if lib.oracle_ffn_hidden(_p(xs), _p(w1), _p(h), xs.shape[0], D, F) != 0:
        raise ValueError("oracle_ffn_hidden rejected its arguments")
    return h.reshape(x.shape[:-1] + (F,))


def heads_to_tokens(o) -> np.ndarray:
    """[B, Hq, S, d] attention output -> [B, S, Hq * d] token rows (the
    concatenation over heads; data movement only)."""
    o = _f64(o)
    B, Hq, S, d = o.shape
    return np.ascontiguousarray(o.transpose(0, 2, 1, 3).reshape(B, S, Hq * d))


def bpt_layer(q, k, v, w1, w2, causal: bool, scale: float, lib: Optional[ctypes.CDLL] = None):
    """Attention followed by the feed-forward network on every token:
    y [B, S, Hq * d] (float64), plus the attention's O and LSE."""
    o, lse = attn_fwd(q, k, v, causal, scale, lib=lib)
    return ffn(heads_to_tokens(o), w1, w2, lib=lib), o, lse


def num_threads(lib: Optional[ctypes.CDLL] = None) -> int:
    return int((lib or load()).oracle_num_threads())
