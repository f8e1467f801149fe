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
// Roles (320 threads): warps 0-7 epilogue (thread = row = TMEM lane; warps w
// and w + 4 share a lane quarter and take one half of the tile's columns
// each), warp 8 TMA producer (4-stage ring of A and B boxes), warp 9 MMA
// issuer and TMEM owner.  The kernel is persistent (one CTA per SM over the launch's output
// tiles) with two accumulators in tensor memory, so a tile's epilogue
// overlaps the next tile's products.  Every mbarrier wait is bounded (see
// mbar_wait).
#pragma once

#include <cuda.h>
#include "sm100.cuh"
#include "launch_dep.cuh"

namespace fa {

constexpr int kFfnBM = 128;       // tokens per tile (TMEM lanes)
constexpr int kFfnBN = 256;       // output columns per tile (fp32 TMEM columns)
constexpr int kFfnBK = 64;        // K per ring stage: one 128-byte swizzle box of bf16
constexpr int kFfnStages = 4;
constexpr int kFfnEpiWarps = 8;   // two per TMEM lane quarter, one per column half
constexpr int kFfnThreads = 32 * kFfnEpiWarps + 64;
constexpr int kFfnProducerWarp = kFfnEpiWarps;
constexpr int kFfnMmaWarp = kFfnEpiWarps + 1;

struct FfnLayout {
  static constexpr int kABytes = kFfnBM * kFfnBK * 2;     // 16 KB
  static constexpr int kBBytes = kFfnBN * kFfnBK * 2;     // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;   // 48 KB
  static constexpr int kBarOff = kFfnStages * kStageBytes;
  // full[S], empty[S], acc_full[2], acc_empty[2], done
  static constexpr int kBarFull = 0;
  static constexpr int kBarEmpty = kFfnStages;
  static constexpr int kBarAccFull = 2 * kFfnStages;
  static constexpr int kBarAccEmpty = kBarAccFull + 2;
  static constexpr int kBarDone = kBarAccEmpty + 2;
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
  int n_row_tiles;    // query tiles of this launch
  int a_heads;        // 1: A = attention output [B*Hq, S, d]; 0: A = chunk scratch [rows, K]
  int c_tokens;       // 1: C row = token b*S_out + tok0 + t; 0: C row = chunk-local row
  int S_out, tok0;    // tokens per sequence of C and the token of A's row 0 (c_tokens)
  int gelu;           // apply GELU (erf form) before rounding to bf16
  unsigned long long wait_limit_ns;
};

__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.f + erff(x * 0.70710678118654752f));
}

// Output tile t of a launch: row tile t / (N/256) (a query tile), column
// tile t % (N/256); the column tiles of one row tile are adjacent, so CTAs
// running together share their A rows in L2.
struct FfnTile {
  int n0, local_row0, b, t0;
};
__device__ __forceinline__ FfnTile ffn_tile(const FfnParams& p, int t) {
  FfnTile f;
  const int n_col = p.N / kFfnBN;
  const int rt = t / n_col;
  f.n0 = (t % n_col) * kFfnBN;
  f.local_row0 = rt * kFfnBM;
  const int g = p.mt0 + rt;
  f.b = g / p.tiles_per_seq;
  f.t0 = (g % p.tiles_per_seq) * kFfnBM;
  return f;
}

// Persistent: one CTA per SM walks the launch's output tiles round-robin.
// Two tensor-memory accumulators (256 columns each) alternate between tiles,
// so the epilogue of one tile (TMEM read-out, GELU, stores) runs while the
// next tile's products accumulate.
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
  const int n_tiles = p.n_row_tiles * (p.N / kFfnBN);
  const int nk = p.K / kFfnBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFfnStages; ++s) {
      mbar_init(bars + 8 * (L::kBarFull + s), 1);
      mbar_init(bars + 8 * (L::kBarEmpty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bars + 8 * (L::kBarAccFull + a), 1);
      mbar_init(bars + 8 * (L::kBarAccEmpty + a), kFfnEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(bars + 8 * L::kBarDone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kFfnMmaWarp) {
    tmem_alloc(sbase + L::kTmemSlotOff, 2 * kFfnBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlotOff);

  // The next launch of the call (the other product, or the next chunk) may
  // start its setup now; it waits for this grid before its first load.
  grid_dep_launch_dependents();
  if (warp == kFfnProducerWarp) {
    if (lane == 0) {
      // producer: A and B boxes of every K step of every tile into the ring
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      // The previous kernel of the call (the attention, or the other
      // product, which reads this launch's output buffer) has completed
      // before any load; every store of this grid follows these loads.
      grid_dep_wait();
      uint32_t issued = 0;
      bool stop = false;
      for (int t = blockIdx.x; t < n_tiles && !stop; t += gridDim.x) {
        const FfnTile f = ffn_tile(p, t);
        for (int kb = 0; kb < nk; ++kb, ++issued) {
          const uint32_t s = issued % kFfnStages;
          if (!mbar_wait(bars + 8 * (L::kBarEmpty + s), ((issued / kFfnStages) & 1u) ^ 1u,
                         abort_flag, p.wait_limit_ns)) {
            stop = true;
            break;
          }
          const uint32_t full = bars + 8 * (L::kBarFull + s);
          const uint32_t sa = sbase + s * L::kStageBytes;
          mbar_arrive_expect_tx(full, L::kStageBytes);
          const int k0 = kb * kFfnBK;
          if (p.a_heads)
            tma_load_3d(sa, &tm_a, full, k0 % p.d, f.t0, f.b * p.Hq + k0 / p.d);
          else
            tma_load_3d(sa, &tm_a, full, k0, f.local_row0, 0);
          tma_load_3d(sa + L::kABytes, &tm_b, full, k0, f.n0, 0);
        }
      }
      // drain: no copy may still be in flight when the CTA exits
      const uint32_t S = kFfnStages;
      for (uint32_t k = (issued > S ? issued - S : 0u); k < issued; ++k)
        mbar_wait(bars + 8 * (L::kBarFull + k % S), (k / S) & 1u, nullptr, p.wait_limit_ns);
    }
  } else if (warp == kFfnMmaWarp) {
    if (lane == 0) {
      // MMA issuer: acc[i & 1] [128 x 256] (+)= A_k B_k^T, four K = 16 steps per stage
      constexpr uint32_t kId = idesc_bf16_f32(kFfnBM, kFfnBN, false);
      const uint64_t a_desc0 = sw128_desc(sbase, 16, 1024);
      const uint64_t b_desc0 = sw128_desc(sbase + L::kABytes, 16, 1024);
      uint32_t used = 0;  // ring stages consumed
      int i = 0;          // tiles of this CTA
      for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
        const uint32_t acc = static_cast<uint32_t>(i & 1);
        // the accumulator is free once the epilogue has read the tile two back
        if (!mbar_wait(bars + 8 * (L::kBarAccEmpty + acc), ((i >> 1) & 1) ^ 1, abort_flag,
                       p.wait_limit_ns))
          break;
        tc_fence_after();
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++used) {
          const uint32_t s = used % kFfnStages;
          ok = mbar_wait(bars + 8 * (L::kBarFull + s), (used / kFfnStages) & 1u, abort_flag,
                         p.wait_limit_ns);
          if (!ok) break;
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>((s * L::kStageBytes) >> 4);
          const uint64_t ad = a_desc0 + so, bd = b_desc0 + so;
          const uint32_t d = tmem + acc * kFfnBN;
          mma_ss_off<0, 0>(d, ad, bd, kId, kb > 0 ? 1u : 0u);
          mma_ss_off<2, 2>(d, ad, bd, kId, 1u);
          mma_ss_off<4, 4>(d, ad, bd, kId, 1u);
          mma_ss_off<6, 6>(d, ad, bd, kId, 1u);
          mma_commit(bars + 8 * (L::kBarEmpty + s));
        }
        if (!ok) break;
        mma_commit(bars + 8 * (L::kBarAccFull + acc));
      }
      // every MMA this thread issued completes before tensor memory is freed
      mma_commit(bars + 8 * L::kBarDone);
      mbar_wait(bars + 8 * L::kBarDone, 0u, nullptr, p.wait_limit_ns);
    }
  } else {
    // epilogue: row r of the tile (the warp's TMEM lane quarter), the warp's
    // half of the columns, 32 columns per TMEM load
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    constexpr int kHalfCols = kFfnBN / 2;
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const FfnTile f = ffn_tile(p, t);
      const uint32_t acc = static_cast<uint32_t>(i & 1);
      const bool ok = mbar_wait(bars + 8 * (L::kBarAccFull + acc), (i >> 1) & 1, abort_flag,
                                p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const bool valid = f.t0 + r < p.S;
      const long long row = p.c_tokens
                                ? static_cast<long long>(f.b) * p.S_out + p.tok0 + f.t0 + r
                                : static_cast<long long>(f.local_row0) + r;
      uint4* dst = reinterpret_cast<uint4*>(p.c + row * p.N + f.n0 + half * kHalfCols);
#pragma unroll 1
      for (int c = 0; c < kHalfCols / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + acc * kFfnBN + static_cast<uint32_t>(half * kHalfCols + c * 32),
                  v);
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
      // this warp's reads of the accumulator are done: hand it back
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (L::kBarAccEmpty + acc));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kFfnMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kFfnBN);
  }
}

}  // namespace fa
