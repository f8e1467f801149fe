"""Seeded synthetic inputs for the attention workloads.

This module holds no attention arithmetic: it only draws random tensors and
names the workload shapes.  It is the one module that both the CUDA-path
tests/bench and the CPU oracle's callers use.

Recipe (fixed so that every caller sees the same tensors for a seed):
  * ``torch.Generator(device).manual_seed(seed)``;
  * ``randn`` in fp32, drawn in the order Q, K, V (shape order below);
  * Q multiplied by ``q_mult`` (a power of two, so the product is exact);
  * rounded to bf16 (round-to-nearest-even, torch's ``.to(bfloat16)``).
  * FP8 prefill: the same fp32 draws, each of Q, K, V scaled per (batch,
    key/value head) so its largest magnitude is 448 and rounded to E4M3
    (quantize_e4m3); the factors are returned beside the codes;
  * feed-forward network after attention (ffn_inputs): o ~ N(0,1),
    w1 ~ N(0,1)/sqrt(D), w2 ~ N(0,1)/sqrt(F), bf16, from seed + 15485863;
  * decode: per-sequence KV lengths ``randint(lmin, lmax + 1)`` drawn after
    K and V from the same generator; cache positions at or beyond a
    sequence's length are filled with ``pad_value`` (NaN by default) so that
    any read of them shows up in the output.
The CPU and CUDA generators give different streams for the same seed; a test
draws once and hands the same tensors to both sides.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Optional

import torch


@dataclass(frozen=True)
class PrefillShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Skv: int
    d: int
    causal: bool
    q_mult: float
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    def flops(self) -> float:
        """4*B*Hq*Sq*Skv*d, halved for a causal mask (the metric's convention)."""
        f = 4.0 * self.B * self.Hq * self.Sq * self.Skv * self.d
        return f / 2.0 if self.causal else f


@dataclass(frozen=True)
class DecodeShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    Lmin: int
    Lmax: int
    d: int
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


# The five workloads of the exact-attention forward path.
CONFIGS: Dict[str, object] = {
    "mha_s512_d64": PrefillShape("mha_s512_d64", 1, 4, 4, 512, 512, 64, False, 1.0, 1),
    "causal_mha_s2048_d128_qx8": PrefillShape(
        "causal_mha_s2048_d128_qx8", 4, 16, 16, 2048, 2048, 128, True, 8.0, 2),
    "causal_gqa_s8192_d128": PrefillShape(
        "causal_gqa_s8192_d128", 2, 32, 8, 8192, 8192, 128, True, 1.0, 3),
    "causal_gqa_s32768_d128": PrefillShape(
        "causal_gqa_s32768_d128", 1, 32, 8, 32768, 32768, 128, True, 1.0, 4),
    "decode_b64_splitkv_d128": DecodeShape(
        "decode_b64_splitkv_d128", 64, 32, 8, 4096, 16384, 128, 5),
}


def prefill_inputs(B: int, Hq: int, Hkv: int, Sq: int, Skv: int, d: int, seed: int,
                   q_mult: float = 1.0, device="cpu"):
    """q [B,Hq,Sq,d], k/v [B,Hkv,Skv,d], bf16, contiguous."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    q = torch.randn((B, Hq, Sq, d), generator=g, device=device, dtype=torch.float32)
    k = torch.randn((B, Hkv, Skv, d), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((B, Hkv, Skv, d), generator=g, device=device, dtype=torch.float32)
    if q_mult != 1.0:
        q.mul_(q_mult)
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous())


def prefill_inputs_for(shape: PrefillShape, device="cpu"):
    return prefill_inputs(shape.B, shape.Hq, shape.Hkv, shape.Sq, shape.Skv, shape.d,
                          shape.seed, shape.q_mult, device)


def decode_inputs(B: int, Hq: int, Hkv: int, Lmin: int, Lmax: int, d: int, seed: int,
                  device="cpu", pad_value: Optional[float] = float("nan")):
    """q [B,Hq,d], k/v caches [B,Hkv,Lmax,d] (bf16), seqlens [B] (int32).

    The cache is drawn in fp32 one sequence at a time, so the peak host memory
    stays one sequence's worth above the bf16 caches."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    q = torch.randn((B, Hq, d), generator=g, device=device,
                    dtype=torch.float32).to(torch.bfloat16)
    kc = torch.empty((B, Hkv, Lmax, d), device=device, dtype=torch.bfloat16)
    vc = torch.empty((B, Hkv, Lmax, d), device=device, dtype=torch.bfloat16)
    for cache in (kc, vc):
        for b in range(B):
            cache[b].copy_(torch.randn((Hkv, Lmax, d), generator=g, device=device,
                                       dtype=torch.float32))
    seqlens = torch.randint(Lmin, Lmax + 1, (B,), generator=g, device=device,
                            dtype=torch.int64).to(torch.int32)
    if pad_value is not None:
        for b, L in enumerate(seqlens.tolist()):
            kc[b, :, L:, :] = pad_value
            vc[b, :, L:, :] = pad_value
    return q.contiguous(), kc.contiguous(), vc.contiguous(), seqlens.contiguous()


def decode_inputs_for(shape: DecodeShape, device="cpu", pad_value=float("nan")):
    return decode_inputs(shape.B, shape.Hq, shape.Hkv, shape.Lmin, shape.Lmax, shape.d,
                         shape.seed, device, pad_value)


def paginate(kc, vc, seqlens, page_size: int, seed: int,
             pad_value: Optional[float] = float("nan")):
    """Store contiguous caches [B,Hkv,Lmax,d] in a paged pool.

    Returns k_pages/v_pages [num_pages,Hkv,page_size,d] and block_table
    [B, ceil(Lmax/page_size)] (int32, on the caches' device).  Sequence b gets
    ceil(L_b/page_size) pages, placed in the pool in an order drawn from the
    seed (a scattered pool, as after many allocations and frees); the pool
    holds exactly the used pages.  Table entries past a sequence's last page
    are -1; rows of a last page past L_b hold pad_value."""
    B, Hkv, Lmax, d = kc.shape
    P = int(page_size)
    max_pages = (Lmax + P - 1) // P
    lens = [int(L) for L in seqlens.tolist()]
    counts = [(L + P - 1) // P for L in lens]
    num_pages = max(1, sum(counts))
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 7919)
    order = torch.randperm(num_pages, generator=g)
    fill = float("nan") if pad_value is None else pad_value
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    b_idx, j_idx = [], []
    for b in range(B):
        b_idx += [b] * counts[b]
        j_idx += list(range(counts[b]))
    phys = order[:len(b_idx)]
    table[torch.tensor(b_idx, dtype=torch.long), torch.tensor(j_idx, dtype=torch.long)] = \
        phys.to(torch.int32)
    pages = []
    for cache in (kc, vc):
        padded = torch.full((B, Hkv, max_pages * P, d), fill, device=cache.device,
                            dtype=cache.dtype)
        padded[:, :, :Lmax] = cache
        for b, L in enumerate(lens):  # rows past L_b: pad_value
            padded[b, :, L:] = fill
        blocks = padded.view(B, Hkv, max_pages, P, d).permute(0, 2, 1, 3, 4)
        pool = torch.full((num_pages, Hkv, P, d), fill, device=cache.device, dtype=cache.dtype)
        if b_idx:
            bi = torch.tensor(b_idx, dtype=torch.long, device=cache.device)
            ji = torch.tensor(j_idx, dtype=torch.long, device=cache.device)
            pool[phys.to(cache.device)] = blocks[bi, ji]
        pages.append(pool.contiguous())
        del padded, blocks
    return pages[0], pages[1], table.to(kc.device).contiguous()


def paged_decode_inputs(B: int, Hq: int, Hkv: int, Lmin: int, Lmax: int, d: int, seed: int,
                        page_size: int, device="cpu",
                        pad_value: Optional[float] = float("nan")):
    """The decode_inputs() sequences stored in a paged cache (see paginate()).

    Returns q [B,Hq,d], k_pages/v_pages [num_pages,Hkv,page_size,d] (bf16),
    block_table [B, ceil(Lmax/page_size)] and seqlens [B] (int32)."""
    q, kc, vc, seqlens = decode_inputs(B, Hq, Hkv, Lmin, Lmax, d, seed, device, pad_value)
    k_pages, v_pages, table = paginate(kc, vc, seqlens, page_size, seed, pad_value)
    return q, k_pages, v_pages, table, seqlens


E4M3_MAX = 448.0


def quantize_e4m3(x: torch.Tensor, Hkv: int):
    """E4M3 codes and per-(batch, key/value head) dequantisation factors for a
    [B,H,S,d] tensor, the way a caller would prepare FP8 inputs: the factor of
    (b, g) is max|x| over the heads of group g divided by 448 (1 for an all-zero
    group), and x8 = x / factor rounded to E4M3 by torch (nearest even).
    Returns (x8 as torch.float8_e4m3fn, factors [B, Hkv] fp32)."""
    B, H = int(x.shape[0]), int(x.shape[1])
    xf = x.float()
    flat = xf.abs().reshape(B, Hkv, -1)
    amax = (flat.amax(dim=2) if flat.shape[2] > 0
            else torch.zeros((B, Hkv), device=x.device, dtype=torch.float32))
    descale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    per_head = descale.repeat_interleave(H // Hkv, dim=1)[:, :, None, None]
    x8 = (xf / per_head).clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return x8.contiguous(), descale.contiguous()


def fp8_prefill_inputs(B: int, Hq: int, Hkv: int, Sq: int, Skv: int, d: int, seed: int,
                       q_mult: float = 1.0, device="cpu"):
    """The prefill_inputs() draws (fp32, before any rounding) quantised to E4M3
    with quantize_e4m3(): (q8, k8, v8, descale_q, descale_k, descale_v)."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    q = torch.randn((B, Hq, Sq, d), generator=g, device=device, dtype=torch.float32)
    k = torch.randn((B, Hkv, Skv, d), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((B, Hkv, Skv, d), generator=g, device=device, dtype=torch.float32)
    if q_mult != 1.0:
        q.mul_(q_mult)
    q8, dq = quantize_e4m3(q, Hkv)
    k8, dk = quantize_e4m3(k, Hkv)
    v8, dv = quantize_e4m3(v, Hkv)
    return q8, k8, v8, dq, dk, dv


def fp8_prefill_inputs_for(shape: PrefillShape, device="cpu"):
    return fp8_prefill_inputs(shape.B, shape.Hq, shape.Hkv, shape.Sq, shape.Skv, shape.d,
                              shape.seed, shape.q_mult, device)


def ffn_inputs(B: int, Hq: int, S: int, d: int, F: int, seed: int, device="cpu"):
    """Inputs of the feed-forward network after attention, random stand-ins
    for trained weights: o [B,Hq,S,d] ~ N(0,1) (an attention output's shape),
    w1 [F, D] ~ N(0,1)/sqrt(D), w2 [D, F] ~ N(0,1)/sqrt(F) with D = Hq*d, all
    rounded to bf16; drawn in that order from their own seed (seed + 15485863)."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) + 15485863)
    D = Hq * d
    o = torch.randn((B, Hq, S, d), generator=g, device=device, dtype=torch.float32)
    w1 = torch.randn((F, D), generator=g, device=device, dtype=torch.float32) / D ** 0.5
    w2 = torch.randn((D, F), generator=g, device=device, dtype=torch.float32) / F ** 0.5
    return tuple(x.to(torch.bfloat16).contiguous() for x in (o, w1, w2))


def grad_output(shape, seed: int, device="cpu"):
    """dL/dO for backward tests and benchmarks: N(0,1), bf16, its own seed."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) + 104729)
    return torch.randn(tuple(shape), generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16).contiguous()
