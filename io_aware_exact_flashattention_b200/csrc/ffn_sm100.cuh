// ffn_sm100.cuh -- the feed-forward network after attention, run blockwise.
//
// "I/O-Aware Kernels", section "Blockwise Parallel Transformers": the
// feed-forward network acts on each token alone, so it can run on a block of
// query rows as soon as their attention output exists, and only that block's
// activations need to be materialised.  Here the attention output O
// [B, Hq, S, d] (as the forward pass writes it) feeds the network per token:
// x_t = (O[b,0,t,:], ..., O[b,Hq-1,t,:]), D = Hq * d, and
//     y_t = W2 gelu(W1 x_t),   W1 [F, D], W2 [D, F] (bf16, row-major),
// GELU in its erf form, no biases.  The host walks the query tiles in chunks;
// per chunk, one launch forms the hidden activations H = gelu(X W1^T) of the
// chunk's tokens in a chunk-sized scratch, and a second forms Y = H W2^T.
// The F-wide activations therefore exist for one chunk at a time, not for the
// whole sequence.
//
// One kernel serves both products: C[128 x 256 tile] = act(A B^T), with A
// [rows, K] and B [N, K] both K-major (row-major with K contiguous), bf16 in,
// fp32 accumulated in tensor memory (tcgen05.mma kind::f16, M = 128,
// N = 256), bf16 out.  For the first product A is read straight from O: the
// K chunk k*64 of a token is column (k*64) % d of head (k*64) / d, one TMA box
// of the [B*Hq, S, d] view, so the concatenation over heads is never formed.
//
// Roles (192 threads): warps 0-3 epilogue (thread = row = TMEM lane), warp 4
// TMA producer (4-stage ring of A and B boxes), warp 5 MMA issuer and TMEM
// owner.  Every mbarrier wait is bounded (see mbar_wait).
#pragma once

#include <cuda.h>
#include "sm100.cuh"

namespace fa {

constexpr int kFfnBM = 128;       // tokens per tile (TMEM lanes)
constexpr int kFfnBN = 256;       // output columns per tile (fp32 TMEM columns)
constexpr int kFfnBK = 64;        // K per ring stage: one 128-byte swizzle box of bf16
constexpr int kFfnStages = 4;
constexpr int kFfnThreads = 192;

struct FfnLayout {
  static constexpr int kABytes = kFfnBM * kFfnBK * 2;     // 16 KB
  static constexpr int kBBytes = kFfnBN * kFfnBK * 2;     // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;   // 48 KB
  static constexpr int kBarOff = kFfnStages * kStageBytes;
  // full[S], empty[S], acc_full, done
  static constexpr int kBarFull = 0;
  static constexpr int kBarEmpty = kFfnStages;
  static constexpr int kBarAcc = 2 * kFfnStages;
  static constexpr int kBarDone = kBarAcc + 1;
  static constexpr int kNumBars = kBarDone + 1;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemSlotOff + 4;
  static constexpr int kBytes = kAbortOff + 4 + 1024;  // + slack for 1024-byte alignment
};

struct FfnParams {
  __nv_bfloat16* c;   // output rows, N bf16 each
  int N, K;           // N % 256 == 0, K % 64 == 0
  int S;              // tokens per sequence held by A (rows past S are never stored)
  int Hq, d;          // geometry of the attention output (first product)
  int tiles_per_seq;  // ceil(S / 128)
  int mt0;            // first query tile (over all sequences) of this launch
  int a_heads;        // 1: A = attention output [B*Hq, S, d]; 0: A = chunk scratch [rows, K]
  int c_tokens;       // 1: C row = token b*S_out + tok0 + t; 0: C row = chunk-local row
  int S_out, tok0;    // tokens per sequence of C and the token of A's row 0 (c_tokens)
  int gelu;           // apply GELU (erf form) before rounding to bf16
  unsigned long long wait_limit_ns;
};

__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.f + erff(x * 0.70710678118654752f));
}

__global__ void __launch_bounds__(kFfnThreads, 1)
fa_ffn_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                   const __grid_constant__ CUtensorMap tm_b, const FfnParams p) {
  using L = FfnLayout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const uint32_t bars = sbase + L::kBarOff;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbortOff);

  // this CTA's tile: output columns [n0, n0 + 256) of query tile g
  const int n0 = static_cast<int>(blockIdx.x) * kFfnBN;
  const int local_row0 = static_cast<int>(blockIdx.y) * kFfnBM;
  const int g = p.mt0 + static_cast<int>(blockIdx.y);
  const int b = g / p.tiles_per_seq;
  const int t0 = (g % p.tiles_per_seq) * kFfnBM;
  const int nk = p.K / kFfnBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFfnStages; ++s) {
      mbar_init(bars + 8 * (L::kBarFull + s), 1);
      mbar_init(bars + 8 * (L::kBarEmpty + s), 1);
    }
    mbar_init(bars + 8 * L::kBarAcc, 1);
    mbar_init(bars + 8 * L::kBarDone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(sbase + L::kTmemSlotOff, kFfnBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlotOff);

  if (warp == 4) {
    if (lane == 0) {
      // producer: A and B boxes of each K step into the ring
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kFfnStages;
        if (!mbar_wait(bars + 8 * (L::kBarEmpty + s), ((kb / kFfnStages) & 1) ^ 1, abort_flag,
                       p.wait_limit_ns))
          break;
        const uint32_t full = bars + 8 * (L::kBarFull + s);
        const uint32_t sa = sbase + s * L::kStageBytes;
        mbar_arrive_expect_tx(full, L::kStageBytes);
        const int k0 = kb * kFfnBK;
        if (p.a_heads)
          tma_load_3d(sa, &tm_a, full, k0 % p.d, t0, b * p.Hq + k0 / p.d);
        else
          tma_load_3d(sa, &tm_a, full, k0, local_row0, 0);
        tma_load_3d(sa + L::kABytes, &tm_b, full, k0, n0, 0);
        ++issued;
      }
      // drain: no copy may still be in flight when the CTA exits
      for (int kb = (issued > kFfnStages ? issued - kFfnStages : 0); kb < issued; ++kb)
        mbar_wait(bars + 8 * (L::kBarFull + kb % kFfnStages), (kb / kFfnStages) & 1, nullptr,
                  p.wait_limit_ns);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // MMA issuer: acc[128 x 256] (+)= A_k B_k^T, four K = 16 steps per stage
      constexpr uint32_t kId = idesc_bf16_f32(kFfnBM, kFfnBN, false);
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % kFfnStages;
        ok = mbar_wait(bars + 8 * (L::kBarFull + s), (kb / kFfnStages) & 1, abort_flag,
                       p.wait_limit_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = sbase + s * L::kStageBytes;
        const uint32_t sb = sa + L::kABytes;
#pragma unroll
        for (int kk = 0; kk < kFfnBK / 16; ++kk)
          mma_ss(tmem, sw128_desc(sa + kk * 32, 16, 1024), sw128_desc(sb + kk * 32, 16, 1024), kId,
                 (kb > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bars + 8 * (L::kBarEmpty + s));
      }
      if (ok) mma_commit(bars + 8 * L::kBarAcc);
      // every MMA this thread issued completes before tensor memory is freed
      mma_commit(bars + 8 * L::kBarDone);
      mbar_wait(bars + 8 * L::kBarDone, 0u, nullptr, p.wait_limit_ns);
    }
  } else {
    // epilogue: row r of the tile, 32 columns per TMEM load
    const int r = threadIdx.x;  // warps 0-3: TMEM lanes 0-127
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const bool ok = mbar_wait(bars + 8 * L::kBarAcc, 0u, abort_flag, p.wait_limit_ns);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const bool valid = t0 + r < p.S;
      const long long row = p.c_tokens ? static_cast<long long>(b) * p.S_out + p.tok0 + t0 + r
                                       : static_cast<long long>(local_row0) + r;
      uint4* dst = reinterpret_cast<uint4*>(p.c + row * p.N + n0);
#pragma unroll 1
      for (int c = 0; c < kFfnBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + static_cast<uint32_t>(c * 32), v);
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float x0 = __uint_as_float(v[2 * e]), x1 = __uint_as_float(v[2 * e + 1]);
          if (p.gelu) {
            x0 = gelu_erf(x0);
            x1 = gelu_erf(x1);
          }
          w[e] = pack_bf16x2(x0, x1);
        }
        if (valid) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[4 * c + q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kFfnBN);
  }
}

}  // namespace fa
