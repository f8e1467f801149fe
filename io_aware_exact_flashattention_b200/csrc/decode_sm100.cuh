// decode_sm100.cuh -- single-query decode: split-KV partials and their merge.
//
// Decode has one query per sequence, so its scores form a 1 x L vector and
// the step is bound by reading the key/value cache from HBM ("FlashAttention
// & IO-aware attention", sections "Direct answer" and "Interviewer
// follow-ups").  To keep every SM streaming, the key/value length is split
// into chunks that run on different SMs (the FlashDecoding idea named in the
// "Deep dive" section of the same page); each chunk writes a normalised
// partial output and its log-sum-exp, and a second kernel merges the chunks
// with the online softmax's e^(m - m_new) rule.
//
// Split kernel: one CTA per (chunk, key/value head, sequence).  All G =
// Hq/Hkv query heads of the group share every key/value byte the CTA reads,
// so each cache byte crosses HBM once.  A token row (D bf16) is read by D/8
// lanes with one 16-byte load each; T tokens per lane group are in flight per
// iteration.  Scores are kept in log2 units (q pre-multiplied by
// scale*log2(e)) and each lane group runs its own online softmax; lane groups
// are merged with shuffles, then warps through shared memory.
#pragma once

#include "sm100.cuh"

namespace fa {

constexpr int kDecodeWarps = 8;
constexpr int kDecodeThreads = kDecodeWarps * 32;
constexpr int kDecodeTokensPerIter = 4;
constexpr float kLn2 = 0.69314718055994530942f;

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  f[0] = __uint_as_float(u.x << 16);
  f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xffff0000u);
  f[4] = __uint_as_float(u.z << 16);
  f[5] = __uint_as_float(u.z & 0xffff0000u);
  f[6] = __uint_as_float(u.w << 16);
  f[7] = __uint_as_float(u.w & 0xffff0000u);
}

// Merge two online-softmax states (log2 units): (m, l, acc) <- (m, l, acc) (+) (mo, lo, acco).
__device__ __forceinline__ void merge_state(float& m, float& l, float (&acc)[8], float mo,
                                            float lo, const float (&acco)[8]) {
  const float mn = fmaxf(m, mo);
  if (mn == -INFINITY) return;  // both empty
  const float a = ex2(m - mn);   // 0 when m == -inf
  const float b = ex2(mo - mn);
  l = l * a + lo * b;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = acc[e] * a + acco[e] * b;
  m = mn;
}

template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads)
fa_decode_split_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                       const __nv_bfloat16* __restrict__ vc, const int* __restrict__ seqlens,
                       float* __restrict__ o_part, float* __restrict__ lse_part, int Hq, int Hkv,
                       int Lmax, int n_splits, float scale_log2) {
  constexpr int LPR = D / 8;          // lanes per token row
  constexpr int RPW = 32 / LPR;       // lane groups per warp
  constexpr int RG = kDecodeWarps * RPW;
  constexpr int T = kDecodeTokensPerIter;
  __shared__ float sm_m[kDecodeWarps][G];
  __shared__ float sm_l[kDecodeWarps][G];
  __shared__ float sm_acc[kDecodeWarps][G][D];

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  int L = seqlens[b];
  L = max(0, min(L, Lmax));
  const int cs = (L + n_splits - 1) / n_splits;
  const int lo = min(L, split * cs);
  const int hi = min(L, lo + cs);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPR;

  float qv[G][8];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const uint4 u = *reinterpret_cast<const uint4*>(
        q + (static_cast<size_t>(b) * Hq + g * G + hh) * D + sub * 8);
    bf16x8_to_f32(u, qv[hh]);
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[hh][e] *= scale_log2;
  }
  float m[G], l[G], acc[G][8];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[hh][e] = 0.f;
  }

  const size_t head_off = (static_cast<size_t>(b) * Hkv + g) * static_cast<size_t>(Lmax) * D;
  const __nv_bfloat16* kb = kc + head_off + sub * 8;
  const __nv_bfloat16* vb = vc + head_off + sub * 8;

  // The loop bound is warp-uniform (the shuffles below need every lane);
  // tokens at or beyond hi are masked per lane group.
  for (int base = lo + warp * RPW * T; base < hi; base += RG * T) {
    const int t0 = base + (lane / LPR) * T;
    uint4 kr[T], vr[T];
#pragma unroll
    for (int u = 0; u < T; ++u) {
      const int t = t0 + u;
      if (t < hi) {
        kr[u] = ld_stream_v4(kb + static_cast<size_t>(t) * D);
        vr[u] = ld_stream_v4(vb + static_cast<size_t>(t) * D);
      } else {
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = make_uint4(0, 0, 0, 0);
      }
    }
    float s[T][G];
#pragma unroll
    for (int u = 0; u < T; ++u) {
      float kf[8];
      bf16x8_to_f32(kr[u], kf);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaf(qv[hh][e], kf[e], a);
        s[u][hh] = a;
      }
    }
#pragma unroll
    for (int off = LPR / 2; off >= 1; off >>= 1)
#pragma unroll
      for (int u = 0; u < T; ++u)
#pragma unroll
        for (int hh = 0; hh < G; ++hh) s[u][hh] += __shfl_xor_sync(0xffffffffu, s[u][hh], off);
#pragma unroll
    for (int u = 0; u < T; ++u)
      if (t0 + u >= hi)
#pragma unroll
        for (int hh = 0; hh < G; ++hh) s[u][hh] = -INFINITY;

    float vf[T][8];
#pragma unroll
    for (int u = 0; u < T; ++u) bf16x8_to_f32(vr[u], vf[u]);
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      float mt = s[0][hh];
#pragma unroll
      for (int u = 1; u < T; ++u) mt = fmaxf(mt, s[u][hh]);
      const float mn = fmaxf(m[hh], mt);
      if (mn != -INFINITY) {  // -inf only when this lane group has seen no token
        const float a = ex2(m[hh] - mn);  // 0 when m was -inf
        float pu[T];
        float ps = 0.f;
#pragma unroll
        for (int u = 0; u < T; ++u) {
          pu[u] = ex2(s[u][hh] - mn);
          ps += pu[u];
        }
        l[hh] = l[hh] * a + ps;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float x = acc[hh][e] * a;
#pragma unroll
          for (int u = 0; u < T; ++u) x = fmaf(pu[u], vf[u][e], x);
          acc[hh][e] = x;
        }
        m[hh] = mn;
      }
    }
  }

  // merge the lane groups of this warp
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[hh], off);
      const float lo2 = __shfl_xor_sync(0xffffffffu, l[hh], off);
      float ao[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) ao[e] = __shfl_xor_sync(0xffffffffu, acc[hh][e], off);
      merge_state(m[hh], l[hh], acc[hh], mo, lo2, ao);
    }
  }
  if (lane < LPR) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      if (lane == 0) {
        sm_m[warp][hh] = m[hh];
        sm_l[warp][hh] = l[hh];
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_acc[warp][hh][sub * 8 + e] = acc[hh][e];
    }
  }
  __syncthreads();

  // merge warps: thread -> (head, element)
  for (int idx = threadIdx.x; idx < G * D; idx += kDecodeThreads) {
    const int hh = idx / D, e = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, sm_m[w][hh]);
    const size_t prow = (static_cast<size_t>(b) * Hq + g * G + hh) * n_splits + split;
    if (M == -INFINITY) {
      o_part[prow * D + e] = 0.f;
      if (e == 0) lse_part[prow] = -INFINITY;
      continue;
    }
    float Ls = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) {
      const float f = ex2(sm_m[w][hh] - M);  // 0 for an empty warp
      Ls = fmaf(sm_l[w][hh], f, Ls);
      O = fmaf(sm_acc[w][hh][e], f, O);
    }
    o_part[prow * D + e] = O / Ls;
    if (e == 0) lse_part[prow] = (M + __log2f(Ls)) * kLn2;
  }
}

// Merge kernel: one warp per (sequence, query head).
template <int D>
__global__ void __launch_bounds__(128)
fa_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                  __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int rows, int n_splits) {
  constexpr float kLog2e = 1.44269504088896340736f;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* lp = lse_part + static_cast<size_t>(row) * n_splits;
  float M = -INFINITY;
  for (int c = lane; c < n_splits; c += 32) M = fmaxf(M, lp[c]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  constexpr int EPL = D / 32;  // elements per lane
  __nv_bfloat16* orow = o + static_cast<size_t>(row) * D + lane * EPL;
  if (M == -INFINITY) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) orow[e] = __float2bfloat16_rn(0.f);
    if (lane == 0) lse[row] = -INFINITY;
    return;
  }
  float z = 0.f;
  for (int c = lane; c < n_splits; c += 32) z += ex2((lp[c] - M) * kLog2e);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  const float lse_row = M + __logf(z);
  float acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  const float* op = o_part + static_cast<size_t>(row) * n_splits * D + lane * EPL;
  for (int c = 0; c < n_splits; ++c) {
    const float wgt = ex2((lp[c] - lse_row) * kLog2e);
    if (wgt == 0.f) continue;  // empty chunk: its partial is 0 anyway
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = fmaf(wgt, op[static_cast<size_t>(c) * D + e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < EPL; e += 2)
    *reinterpret_cast<__nv_bfloat162*>(orow + e) = __floats2bfloat162_rn(acc[e], acc[e + 1]);
  if (lane == 0) lse[row] = lse_row;
}

}  // namespace fa
