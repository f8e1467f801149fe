"""Python binding of libfa.so (include/fa.h): argument marshalling only.

Every step of the attention path runs in the library's CUDA kernels; torch is
used here to hold device memory and to name the current CUDA stream.  There is
no CPU or library fallback: if libfa.so is missing or a call fails, these
functions raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa.so")

FA_OK = 0
STATUS_NAMES = {
    0: "FA_OK",
    1: "FA_ERR_INVALID_ARG",
    2: "FA_ERR_UNSUPPORTED",
    3: "FA_ERR_ALIGNMENT",
    4: "FA_ERR_CUDA",
    5: "FA_ERR_DEVICE_TIMEOUT",
}

# Every symbol include/fa.h declares, with (restype, argtypes).
_VP, _FP, _I32P = ctypes.c_void_p, ctypes.POINTER(ctypes.c_float), ctypes.c_void_p
_I, _F = ctypes.c_int, ctypes.c_float
SIGNATURES = {
    "fa_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _F, _VP]),
    "fa_fwd_fp8": (_I, [_VP] * 8 + [_I] * 7 + [_F, _VP]),
    "fa_decode_splitkv": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _VP]),
    "fa_decode_paged_splitkv": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP] + [_I] * 8 + [_F, _VP]),
    "fa_combine": (_I, [_VP, _VP, _VP, _VP, _I, _I, _I, _I, _VP]),
    "fa_bwd": (_I, [_VP] * 10 + [_I] * 7 + [_F, _VP]),
    "fa_bwd_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "fa_bpt_ffn": (_I, [_VP] * 5 + [_I] * 6 + [_VP]),
    "fa_bpt_workspace_bytes": (ctypes.c_size_t, [_I, _I]),
    "fa_bpt_layer": (_I, [_VP] * 8 + [_I] * 7 + [_F, _I, _VP]),
    "fa_bpt_layer_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "fa_decode_default_splits": (_I, [_I, _I, _I, _I]),
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_get_device_status": (_I, []),
    "fa_debug_timeout_probe": (_I, [ctypes.c_uint, _VP]),
    "fa_decode_noalloc": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _VP]),
    "fa_debug_exp2_poly": (_I, [_VP, _VP, _I, _VP]),
    "fa_debug_bwd_tiles": (_I, [_I] * 8 + [_VP, ctypes.c_longlong, _VP, _VP]),
    "fa_shard_units": (_I, [_I, _I, _I, _I, ctypes.POINTER(ctypes.c_int),
                            ctypes.POINTER(ctypes.c_int)]),
    "fa_shard_sequences": (_I, [_VP, _I, _I, _VP]),
}

_lib: Optional[ctypes.CDLL] = None


class FAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s failed: %s" % (fn, status_string(status)))


def lib() -> ctypes.CDLL:
    """Load libfa.so (built by io_aware_exact_flashattention_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libfa.so is not built; run "
                               "`python -m io_aware_exact_flashattention_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != FA_OK:
        raise FAError(fn, status)


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else (t.data_ptr() or None)


def _need(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


# ---------------------------------------------------------------------------
# Raw C-ABI calls on device tensors (outputs preallocated by the caller)
# ---------------------------------------------------------------------------

def fa_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
           lse: torch.Tensor, causal: bool, scale: float,
           stream: Optional[torch.cuda.Stream] = None) -> None:
    """fa_fwd on q [B,Hq,Sq,d], k/v [B,Hkv,Skv,d] (bf16), o [B,Hq,Sq,d] bf16,
    lse [B,Hq,Sq] fp32, all on the same CUDA device."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _need(t, torch.bfloat16, n)
    _need(lse, torch.float32, "lse")
    B, Hq, Sq, d = q.shape
    _, Hkv, Skv, _ = k.shape
    if tuple(v.shape) != tuple(k.shape) or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k/v shapes %s/%s do not match q %s" % (tuple(k.shape), tuple(v.shape),
                                                                 tuple(q.shape)))
    if tuple(o.shape) != tuple(q.shape) or tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError("output shapes do not match q")
    _check("fa_fwd", lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Sq,
                                  Skv, d, int(bool(causal)), float(scale), _stream_ptr(stream)))


def _need_e4m3(t: torch.Tensor, name: str) -> None:
    if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise ValueError("%s must hold E4M3 codes (float8_e4m3fn or uint8), got %s"
                         % (name, t.dtype))
    _need(t, t.dtype, name)


def fa_fwd_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
               descale_q: Optional[torch.Tensor], descale_k: Optional[torch.Tensor],
               descale_v: Optional[torch.Tensor], o: torch.Tensor, lse: torch.Tensor,
               causal: bool, scale: float, stream: Optional[torch.cuda.Stream] = None) -> None:
    """fa_fwd_fp8 on E4M3 q [B,Hq,Sq,d], k/v [B,Hkv,Skv,d] with fp32
    dequantisation factors [B,Hkv] (None = 1); o [B,Hq,Sq,d] bf16, lse
    [B,Hq,Sq] fp32."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need_e4m3(t, n)
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    B, Hq, Sq, d = q.shape
    _, Hkv, Skv, _ = k.shape
    if tuple(v.shape) != tuple(k.shape) or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k/v shapes %s/%s do not match q %s" % (tuple(k.shape), tuple(v.shape),
                                                                 tuple(q.shape)))
    if tuple(o.shape) != tuple(q.shape) or tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError("output shapes do not match q")
    for t, n in ((descale_q, "descale_q"), (descale_k, "descale_k"), (descale_v, "descale_v")):
        if t is not None:
            _need(t, torch.float32, n)
            if t.numel() != B * Hkv:
                raise ValueError("%s must hold B * Hkv factors" % n)
    _check("fa_fwd_fp8", lib().fa_fwd_fp8(
        _ptr(q), _ptr(k), _ptr(v), _ptr(descale_q), _ptr(descale_k), _ptr(descale_v), _ptr(o),
        _ptr(lse), B, Hq, Hkv, Sq, Skv, d, int(bool(causal)), float(scale), _stream_ptr(stream)))


def flash_attention_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                        descale_q: Optional[torch.Tensor] = None,
                        descale_k: Optional[torch.Tensor] = None,
                        descale_v: Optional[torch.Tensor] = None, causal: bool = False,
                        scale: Optional[float] = None,
                        out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None
                        ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Exact attention of E4M3 inputs (CUDA tensors): returns (o bf16, lse fp32)
    of softmax(scale * Q K^T [+causal mask]) V on the dequantised values."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    B, Hq, Sq, d = q.shape
    if out is not None:
        o, lse = out
    else:
        o = torch.empty((B, Hq, Sq, d), device=q.device, dtype=torch.bfloat16)
        lse = torch.empty((B, Hq, Sq), device=q.device, dtype=torch.float32)
    fa_fwd_fp8(q, k, v, descale_q, descale_k, descale_v, o, lse, causal, scale)
    return o, lse


def bpt_workspace_bytes(F: int, chunk_tiles: int) -> int:
    return int(lib().fa_bpt_workspace_bytes(F, chunk_tiles))


def fa_bpt_ffn(o: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor, y: torch.Tensor,
               workspace: torch.Tensor, chunk_tiles: int,
               stream: Optional[torch.cuda.Stream] = None) -> None:
    """fa_bpt_ffn: y [B,S,D] = W2 gelu(W1 x_t) with x_t the concatenation over
    heads of o [B,Hq,S,d]; w1 [F,D], w2 [D,F]; all bf16 on one CUDA device."""
    for t, n in ((o, "o"), (w1, "w1"), (w2, "w2"), (y, "y")):
        _need(t, torch.bfloat16, n)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    B, Hq, S, d = o.shape
    D = Hq * d
    F = w1.shape[0]
    if tuple(w1.shape) != (F, D) or tuple(w2.shape) != (D, F) or tuple(y.shape) != (B, S, D):
        raise ValueError("w1 [F, D], w2 [D, F] and y [B, S, D] with D = Hq * d")
    if workspace.numel() * workspace.element_size() < bpt_workspace_bytes(F, chunk_tiles):
        raise ValueError("workspace smaller than fa_bpt_workspace_bytes")
    _check("fa_bpt_ffn", lib().fa_bpt_ffn(_ptr(o), _ptr(w1), _ptr(w2), _ptr(y), _ptr(workspace),
                                          B, Hq, S, d, F, int(chunk_tiles), _stream_ptr(stream)))


def bpt_ffn(o: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor,
            chunk_tiles: int = 16) -> torch.Tensor:
    """The feed-forward network on every token of an attention output o
    [B,Hq,S,d], run blockwise (chunk_tiles query tiles at a time): y [B,S,Hq*d]."""
    B, Hq, S, d = o.shape
    y = torch.empty((B, S, Hq * d), device=o.device, dtype=torch.bfloat16)
    ws = torch.empty(max(16, bpt_workspace_bytes(w1.shape[0], chunk_tiles)), dtype=torch.uint8,
                     device=o.device)
    fa_bpt_ffn(o, w1, w2, y, ws, chunk_tiles)
    return y


def bpt_layer_workspace_bytes(B: int, Hq: int, d: int, F: int, chunk_tiles: int) -> int:
    return int(lib().fa_bpt_layer_workspace_bytes(B, Hq, d, F, chunk_tiles))


def fa_bpt_layer(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, w1: torch.Tensor,
                 w2: torch.Tensor, y: torch.Tensor, lse: torch.Tensor, workspace: torch.Tensor,
                 causal: bool, scale: float, chunk_tiles: int,
                 stream: Optional[torch.cuda.Stream] = None) -> None:
    """fa_bpt_layer: attention then the feed-forward network, chunk by chunk
    of chunk_tiles query tiles; y [B,S,Hq*d] bf16 and lse [B,Hq,S] fp32."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (w1, "w1"), (w2, "w2"), (y, "y")):
        _need(t, torch.bfloat16, n)
    _need(lse, torch.float32, "lse")
    B, Hq, S, d = q.shape
    _, Hkv, Skv, _ = k.shape
    D = Hq * d
    F = w1.shape[0]
    if Skv != S or tuple(v.shape) != tuple(k.shape) or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("self-attention: k, v [B,Hkv,S,d] with q's B, S and d")
    if tuple(w1.shape) != (F, D) or tuple(w2.shape) != (D, F) or tuple(y.shape) != (B, S, D):
        raise ValueError("w1 [F, D], w2 [D, F] and y [B, S, D] with D = Hq * d")
    if tuple(lse.shape) != (B, Hq, S):
        raise ValueError("lse must be [B, Hq, S]")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    if workspace.numel() * workspace.element_size() < bpt_layer_workspace_bytes(B, Hq, d, F,
                                                                               chunk_tiles):
        raise ValueError("workspace smaller than fa_bpt_layer_workspace_bytes")
    _check("fa_bpt_layer", lib().fa_bpt_layer(
        _ptr(q), _ptr(k), _ptr(v), _ptr(w1), _ptr(w2), _ptr(y), _ptr(lse), _ptr(workspace), B,
        Hq, Hkv, S, d, F, int(bool(causal)), float(scale), int(chunk_tiles), _stream_ptr(stream)))


def bpt_layer(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, w1: torch.Tensor,
              w2: torch.Tensor, causal: bool = False, scale: Optional[float] = None,
              chunk_tiles: int = 16) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention followed by the feed-forward network, block by block
    (fa_bpt_layer): returns (y [B,S,Hq*d], lse).  Only one chunk's attention
    output and hidden activations exist at a time."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    B, Hq, S, d = q.shape
    F = w1.shape[0]
    y = torch.empty((B, S, Hq * d), device=q.device, dtype=torch.bfloat16)
    lse = torch.empty((B, Hq, S), device=q.device, dtype=torch.float32)
    ws = torch.empty(max(16, bpt_layer_workspace_bytes(B, Hq, d, F, chunk_tiles)),
                     dtype=torch.uint8, device=q.device)
    fa_bpt_layer(q, k, v, w1, w2, y, lse, ws, causal, scale, chunk_tiles)
    return y, lse


def bwd_workspace_bytes(B: int, Hq: int, Sq: int, d: int) -> int:
    return int(lib().fa_bwd_workspace_bytes(B, Hq, Sq, d))


def fa_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
           lse: torch.Tensor, d_o: torch.Tensor, dq: torch.Tensor, dk: torch.Tensor,
           dv: torch.Tensor, workspace: torch.Tensor, causal: bool, scale: float,
           stream: Optional[torch.cuda.Stream] = None) -> None:
    """fa_bwd: gradients dq [B,Hq,Sq,d], dk/dv [B,Hkv,Skv,d] (bf16) from q, k, v,
    the forward's o and lse, and d_o; workspace is a uint8/float tensor of at
    least bwd_workspace_bytes() bytes."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (d_o, "d_o"), (dq, "dq"), (dk, "dk"),
                 (dv, "dv")):
        _need(t, torch.bfloat16, n)
    _need(lse, torch.float32, "lse")
    B, Hq, Sq, d = q.shape
    _, Hkv, Skv, _ = k.shape
    for t, shp, n in ((o, q.shape, "o"), (d_o, q.shape, "d_o"), (dq, q.shape, "dq"),
                      (v, k.shape, "v"), (dk, k.shape, "dk"), (dv, k.shape, "dv")):
        if tuple(t.shape) != tuple(shp):
            raise ValueError("%s must have shape %s" % (n, tuple(shp)))
    if tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError("lse must be [B,Hq,Sq]")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    if workspace.numel() * workspace.element_size() < bwd_workspace_bytes(B, Hq, Sq, d):
        raise ValueError("workspace too small")
    _check("fa_bwd", lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(d_o),
                                  _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), B, Hq, Hkv, Sq,
                                  Skv, d, int(bool(causal)), float(scale), _stream_ptr(stream)))


def attention_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                       lse: torch.Tensor, d_o: torch.Tensor, causal: bool = False,
                       scale: Optional[float] = None
                       ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """(dq, dk, dv) for CUDA tensors, allocating the outputs and the workspace."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    B, Hq, Sq, d = q.shape
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    ws = torch.empty(max(16, bwd_workspace_bytes(B, Hq, Sq, d)), dtype=torch.uint8,
                     device=q.device)
    fa_bwd(q, k, v, o, lse, d_o, dq, dk, dv, ws, causal, scale)
    return dq, dk, dv


def fa_decode_splitkv(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      seqlens_k: torch.Tensor, o_partial: torch.Tensor,
                      lse_partial: torch.Tensor, scale: float,
                      stream: Optional[torch.cuda.Stream] = None) -> None:
    """fa_decode_splitkv on q [B,Hq,d], caches [B,Hkv,Lmax,d] (bf16), seqlens
    [B] int32; o_partial [B,Hq,n,d] and lse_partial [B,Hq,n] fp32."""
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _need(t, torch.bfloat16, n)
    _need(seqlens_k, torch.int32, "seqlens_k")
    _need(o_partial, torch.float32, "o_partial")
    _need(lse_partial, torch.float32, "lse_partial")
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = k_cache.shape
    n = o_partial.shape[2]
    if tuple(o_partial.shape) != (B, Hq, n, d) or tuple(lse_partial.shape) != (B, Hq, n):
        raise ValueError("partial buffers must be [B,Hq,n,d] and [B,Hq,n]")
    _check("fa_decode_splitkv", lib().fa_decode_splitkv(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens_k), _ptr(o_partial),
        _ptr(lse_partial), B, Hq, Hkv, Lmax, d, n, float(scale), _stream_ptr(stream)))


def fa_decode_paged_splitkv(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                            block_table: torch.Tensor, seqlens_k: torch.Tensor,
                            o_partial: torch.Tensor, lse_partial: torch.Tensor, scale: float,
                            stream: Optional[torch.cuda.Stream] = None) -> None:
    """fa_decode_paged_splitkv on q [B,Hq,d], page pools [num_pages,Hkv,P,d] (bf16),
    block_table [B,max_pages] and seqlens [B] int32; o_partial [B,Hq,n,d] and
    lse_partial [B,Hq,n] fp32 (chunk sizes rounded up to multiples of 128)."""
    for t, n in ((q, "q"), (k_pages, "k_pages"), (v_pages, "v_pages")):
        _need(t, torch.bfloat16, n)
    _need(block_table, torch.int32, "block_table")
    _need(seqlens_k, torch.int32, "seqlens_k")
    _need(o_partial, torch.float32, "o_partial")
    _need(lse_partial, torch.float32, "lse_partial")
    B, Hq, d = q.shape
    num_pages, Hkv, P, _ = k_pages.shape
    if tuple(v_pages.shape) != tuple(k_pages.shape):
        raise ValueError("k_pages and v_pages must have the same shape")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, max_pages]")
    max_pages = block_table.shape[1]
    n = o_partial.shape[2]
    if tuple(o_partial.shape) != (B, Hq, n, d) or tuple(lse_partial.shape) != (B, Hq, n):
        raise ValueError("partial buffers must be [B,Hq,n,d] and [B,Hq,n]")
    _check("fa_decode_paged_splitkv", lib().fa_decode_paged_splitkv(
        _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seqlens_k),
        _ptr(o_partial), _ptr(lse_partial), B, Hq, Hkv, num_pages, P, max_pages, d, n,
        float(scale), _stream_ptr(stream)))


def fa_combine(o_partial: torch.Tensor, lse_partial: torch.Tensor, o: torch.Tensor,
               lse: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """fa_combine: o_partial [B,Hq,n,d], lse_partial [B,Hq,n] fp32 -> o [B,Hq,d]
    bf16, lse [B,Hq] fp32."""
    _need(o_partial, torch.float32, "o_partial")
    _need(lse_partial, torch.float32, "lse_partial")
    _need(o, torch.bfloat16, "o")
    _need(lse, torch.float32, "lse")
    B, Hq, n, d = o_partial.shape
    if tuple(o.shape) != (B, Hq, d) or tuple(lse.shape) != (B, Hq):
        raise ValueError("outputs must be [B,Hq,d] and [B,Hq]")
    _check("fa_combine", lib().fa_combine(_ptr(o_partial), _ptr(lse_partial), _ptr(o), _ptr(lse),
                                          B, Hq, n, d, _stream_ptr(stream)))


def decode_default_splits(B: int, Hkv: int, Lmax: int, num_sms: int) -> int:
    return int(lib().fa_decode_default_splits(B, Hkv, Lmax, num_sms))


def get_device_status() -> int:
    """Read and clear the device status word (synchronises the device)."""
    return int(lib().fa_get_device_status())


def debug_exp2_poly(x: torch.Tensor) -> torch.Tensor:
    """The prefill kernel's polynomial 2^x on device (test hook)."""
    _need(x, torch.float32, "x")
    y = torch.empty_like(x)
    _check("fa_debug_exp2_poly", lib().fa_debug_exp2_poly(_ptr(x), _ptr(y), x.numel(),
                                                           _stream_ptr(None)))
    return y


def debug_timeout_probe(limit_us: int, stream: Optional[torch.cuda.Stream] = None) -> None:
    _check("fa_debug_timeout_probe", lib().fa_debug_timeout_probe(int(limit_us),
                                                                  _stream_ptr(stream)))


# ---------------------------------------------------------------------------
# User-level calls: allocate outputs; host tensors are copied in and out
# ---------------------------------------------------------------------------

def flash_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                    scale: Optional[float] = None, device: Optional[torch.device] = None,
                    out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                    chunks: Optional[int] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Exact attention O = softmax(scale*QK^T [+causal mask]) V and its LSE.

    CUDA inputs stay where they are.  CPU inputs (ideally pinned) are copied
    to `device` (default: the current CUDA device) and the results are copied
    back into `out` = (o, lse) host tensors when given, else into new pinned
    tensors; the call returns after the results landed.  With host inputs the
    work is cut into `chunks` groups of key/value heads (default: about 16 MB
    of inputs each); each group is an fa_fwd problem of its own ([n, G, S, d]
    queries against [n, 1, S, d] keys/values), so copying group c+1 in, the
    kernel on group c and copying group c-1 out run at the same time on
    three streams."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if q.is_cuda:
        B, Hq, Sq, d = q.shape
        if out is not None:
            o, lse = out
        else:
            o = torch.empty_like(q)
            lse = torch.empty((B, Hq, Sq), device=q.device, dtype=torch.float32)
        fa_fwd(q, k, v, o, lse, causal, scale)
        return o, lse

    dev = device or torch.device("cuda", torch.cuda.current_device())
    B, Hq, Sq, d = q.shape
    _, Hkv, Skv, _ = k.shape
    if Hkv < 1 or Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    rows = B * Hkv  # key/value heads; each owns G query heads
    if out is not None:
        o_h, lse_h = out
    else:
        o_h = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        lse_h = torch.empty((B, Hq, Sq), dtype=torch.float32, pin_memory=True)
    # [rows, G, S, d] / [rows, 1, S, d] views: a range of rows is a valid problem
    qf, kf, vf = q.reshape(rows, G, Sq, d), k.reshape(rows, 1, Skv, d), v.reshape(rows, 1, Skv, d)
    of, lf = o_h.view(rows, G, Sq, d), lse_h.view(rows, G, Sq)
    qd, kd, vd = (torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (qf, kf, vf))
    od = torch.empty(qf.shape, dtype=q.dtype, device=dev)
    ld = torch.empty((rows, G, Sq), dtype=torch.float32, device=dev)
    if chunks is None:
        per_row = (G * Sq + 2 * Skv) * d * q.element_size()
        chunks = max(1, min(rows, (rows * per_row) // (16 << 20)))
    bounds = [rows * c // chunks for c in range(chunks + 1)]
    compute = torch.cuda.current_stream(dev)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    s_in.wait_stream(compute)    # device buffers are free for this call's copies
    s_out.wait_stream(compute)
    for c in range(chunks):
        a, b = bounds[c], bounds[c + 1]
        if a == b:
            continue
        with torch.cuda.stream(s_in):
            for dst, src in ((qd, qf), (kd, kf), (vd, vf)):
                dst[a:b].copy_(src[a:b], non_blocking=True)
        compute.wait_stream(s_in)
        fa_fwd(qd[a:b], kd[a:b], vd[a:b], od[a:b], ld[a:b], causal, scale, stream=compute)
        s_out.wait_stream(compute)
        with torch.cuda.stream(s_out):
            of[a:b].copy_(od[a:b], non_blocking=True)
            lf[a:b].copy_(ld[a:b], non_blocking=True)
    compute.wait_stream(s_out)
    compute.synchronize()
    for t in (qd, kd, vd, od, ld):  # the caching allocator must not hand these out early
        t.record_stream(s_in)
        t.record_stream(s_out)
    return o_h, lse_h


def decode_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                     seqlens_k: torch.Tensor, scale: Optional[float] = None,
                     num_splits: Optional[int] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Single-query decode over a contiguous cache: split-KV partials, then the
    LSE-weighted merge.  All tensors on one CUDA device."""
    B, Hq, d = q.shape
    _, Hkv, Lmax, _ = k_cache.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if num_splits is None:
        sms = torch.cuda.get_device_properties(q.device).multi_processor_count
        num_splits = decode_default_splits(B, Hkv, Lmax, sms)
    o_part = torch.empty((B, Hq, num_splits, d), device=q.device, dtype=torch.float32)
    lse_part = torch.empty((B, Hq, num_splits), device=q.device, dtype=torch.float32)
    fa_decode_splitkv(q, k_cache, v_cache, seqlens_k, o_part, lse_part, scale)
    o = torch.empty((B, Hq, d), device=q.device, dtype=torch.bfloat16)
    lse = torch.empty((B, Hq), device=q.device, dtype=torch.float32)
    fa_combine(o_part, lse_part, o, lse)
    return o, lse


def decode_attention_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                           block_table: torch.Tensor, seqlens_k: torch.Tensor,
                           scale: Optional[float] = None,
                           num_splits: Optional[int] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Single-query decode over a paged cache (pages [num_pages,Hkv,P,d], block
    table [B,max_pages]): split-KV partials, then the LSE-weighted merge."""
    B, Hq, d = q.shape
    _, Hkv, P, _ = k_pages.shape
    Lmax = block_table.shape[1] * P
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if num_splits is None:
        sms = torch.cuda.get_device_properties(q.device).multi_processor_count
        num_splits = decode_default_splits(B, Hkv, Lmax, sms)
    o_part = torch.empty((B, Hq, num_splits, d), device=q.device, dtype=torch.float32)
    lse_part = torch.empty((B, Hq, num_splits), device=q.device, dtype=torch.float32)
    fa_decode_paged_splitkv(q, k_pages, v_pages, block_table, seqlens_k, o_part, lse_part, scale)
    o = torch.empty((B, Hq, d), device=q.device, dtype=torch.bfloat16)
    lse = torch.empty((B, Hq), device=q.device, dtype=torch.float32)
    fa_combine(o_part, lse_part, o, lse)
    return o, lse


# ---------------------------------------------------------------------------
# Sharding one problem over several devices (or processes): no data exchange
# ---------------------------------------------------------------------------

def shard_units(B: int, Hkv: int, n_shards: int, shard: int) -> Tuple[int, int]:
    """(first, count): the shard's range of (batch, key/value head) units in
    row-major order (fa_shard_units)."""
    first, count = ctypes.c_int(0), ctypes.c_int(0)
    _check("fa_shard_units", lib().fa_shard_units(int(B), int(Hkv), int(n_shards), int(shard),
                                                  ctypes.byref(first), ctypes.byref(count)))
    return first.value, count.value


def shard_sequences(seqlens_k, n_shards: int) -> list:
    """Bounds [n_shards + 1] of a contiguous, work-balanced split of a decode
    batch (fa_shard_sequences); seqlens_k on any device or a sequence."""
    import numpy as np
    sl = np.ascontiguousarray(np.asarray(seqlens_k.cpu().numpy() if hasattr(seqlens_k, "cpu")
                                         else seqlens_k, dtype=np.int32))
    bounds = np.zeros(int(n_shards) + 1, dtype=np.int32)
    _check("fa_shard_sequences", lib().fa_shard_sequences(sl.ctypes.data, int(sl.size),
                                                          int(n_shards), bounds.ctypes.data))
    return [int(x) for x in bounds]


def unit_views(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
    """q [B,Hq,S,d], k/v [B,Hkv,S,d] as [B*Hkv, Hq/Hkv, S, d] and
    [B*Hkv, 1, S, d] views: a range of rows of these views is one unit range,
    an fa_fwd problem of its own."""
    B, Hq, Sq, d = q.shape
    _, Hkv, Skv, _ = k.shape
    if Hkv < 1 or Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    return (q.reshape(B * Hkv, G, Sq, d), k.reshape(B * Hkv, 1, Skv, d),
            v.reshape(B * Hkv, 1, Skv, d))


def flash_attention_sharded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                            causal: bool = False, scale: Optional[float] = None,
                            devices: Optional[list] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One attention problem split over `devices` (default: every visible CUDA
    device) by (batch, key/value head) units, without any collective: shard s
    copies its units' q, k, v to device s, runs fa_fwd there on a stream of its
    own, and copies its rows of o and lse back into outputs that live where q
    lives (host or device).  Returns (o, lse) after every shard has finished.
    The result is bit-identical to one fa_fwd call on the whole problem."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if devices is None:
        devices = [torch.device("cuda", i) for i in range(torch.cuda.device_count())]
    devices = [torch.device(d) for d in devices]
    if not devices:
        raise RuntimeError("no CUDA device to shard over")
    B, Hq, Sq, d = q.shape
    _, Hkv, _, _ = k.shape
    qv, kv, vv = unit_views(q, k, v)
    pin = not q.is_cuda
    o = torch.empty(q.shape, dtype=q.dtype, device=q.device, pin_memory=pin)
    lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device, pin_memory=pin)
    ov, lv = o.view(qv.shape), lse.view(qv.shape[:3])
    pending = []
    for s, dev in enumerate(devices):
        a, n = shard_units(B, Hkv, len(devices), s)
        if n == 0:
            continue
        with torch.cuda.device(dev):
            stream = torch.cuda.Stream(dev)
            stream.wait_stream(torch.cuda.current_stream(dev))
            if q.is_cuda:
                stream.wait_stream(torch.cuda.current_stream(q.device))
            with torch.cuda.stream(stream):
                qs, ks, vs = (t[a:a + n].to(dev, non_blocking=True) for t in (qv, kv, vv))
                os_ = torch.empty(qs.shape, dtype=q.dtype, device=dev)
                ls_ = torch.empty(qs.shape[:3], dtype=torch.float32, device=dev)
                fa_fwd(qs, ks, vs, os_, ls_, causal, scale, stream=stream)
                ov[a:a + n].copy_(os_, non_blocking=True)
                lv[a:a + n].copy_(ls_, non_blocking=True)
            pending.append((stream, (qs, ks, vs, os_, ls_)))
    for stream, bufs in pending:
        stream.synchronize()
    return o, lse


def decode_attention_sharded(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                             seqlens_k: torch.Tensor, scale: Optional[float] = None,
                             devices: Optional[list] = None,
                             num_splits: Optional[int] = None
                             ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Single-query decode with the batch split over `devices` by sequences
    (fa_shard_sequences, balanced by key count), without any collective: each
    device decodes its sequences (split-KV + merge) on a stream of its own and
    its rows of o and lse are copied back to where q lives."""
    if devices is None:
        devices = [torch.device("cuda", i) for i in range(torch.cuda.device_count())]
    devices = [torch.device(d) for d in devices]
    if not devices:
        raise RuntimeError("no CUDA device to shard over")
    B, Hq, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    bounds = shard_sequences(seqlens_k, len(devices))
    pin = not q.is_cuda
    o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q.device, pin_memory=pin)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device, pin_memory=pin)
    pending = []
    for s, dev in enumerate(devices):
        a, b = bounds[s], bounds[s + 1]
        if a == b:
            continue
        with torch.cuda.device(dev):
            stream = torch.cuda.Stream(dev)
            stream.wait_stream(torch.cuda.current_stream(dev))
            if q.is_cuda:
                stream.wait_stream(torch.cuda.current_stream(q.device))
            with torch.cuda.stream(stream):
                qs, ks, vs, ss = (t[a:b].to(dev, non_blocking=True)
                                  for t in (q, k_cache, v_cache, seqlens_k))
                os_, ls_ = decode_attention(qs, ks, vs, ss, scale, num_splits)
                o[a:b].copy_(os_, non_blocking=True)
                lse[a:b].copy_(ls_, non_blocking=True)
            pending.append((stream, (qs, ks, vs, ss, os_, ls_)))
    for stream, bufs in pending:
        stream.synchronize()
    return o, lse
