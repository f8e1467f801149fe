// backward_sm100.cuh -- exact-attention backward by recomputation for sm_100a.
//
// The pages state that the backward pass recomputes the attention matrix
// instead of storing it ("Tracing Tiled QKV Data Movement in FlashAttention's
// Memory Hierarchy", closing takeaways).  With P = exp(scale*q.k - LSE) from
// the forward's LSE, D_i = dO_i . O_i and dS = P * (dO.v - D):
//   dV_j = sum_i P_ij dO_i,  dK_j = scale * sum_i dS_ij q_i,  dQ_i = scale * sum_j dS_ij k_j.
//
// Two kernels, each with its accumulators resident in tensor memory for the
// whole loop, so that every gradient is written once, in bf16, with no
// reductions in global memory (and the result does not depend on the order
// in which CTAs run):
//
// fa_bwd_dkdv_kernel -- one CTA per (batch, key/value head, 128-key tile j).
//   K_j and V_j stay in shared memory and dK_j, dV_j accumulate in TMEM while
//   the query tiles of every query head of the group stream past.  Per query
//   tile, on tcgen05 with fp32 accumulators:
//     S^T  = K_j Q_i^T      (M=128 keys, N=128 queries; SS)
//     dP^T = V_j dO_i^T     (M=128 keys, N=128 queries; SS)
//     dV  += P^T dO_i       (A = P^T in TMEM, B = dO_i MN-major; TS)
//     dK  += dS^T Q_i       (A = dS^T K-major in shared memory, B = Q_i MN-major; SS)
//   Tensor memory columns: dV [0,128), dK [128,256), S^T / P [256,384),
//   dP^T [384,512).
//
// fa_bwd_dq_kernel -- one CTA per (batch, query head, 128-query tile i).
//   Q_i and dO_i stay in shared memory, dQ_i accumulates in TMEM while the
//   key tiles the queries see stream past (K in a three-stage ring, V in a
//   two-stage one: K_j is read last by dQ_j, V_j already by dP_j):
//     S   = Q_i K_j^T       (M=128 queries, N=128 keys; SS), two buffers
//     dP  = dO_i V_j^T      (M=128 queries, N=128 keys; SS)
//     dQ += dS K_j          (A = dS packed in the S buffer; B = K_j MN-major; TS)
//   Tensor memory columns: S [0,128) and [128,256), dP [256,384), dQ [384,384+d).
//   Against a single kernel that adds partial dQ tiles into an fp32 buffer,
//   this recomputes S and dP once more (7 products per tile pair instead of
//   5) but removes 64 KB of fp32 additions per tile pair, whose memory-side
//   throughput bounded that design.
//
// Roles of both (320 threads):
//   warps 0-7  two element-wise warpgroups (P, dS; the gradients out)
//   warp  8    TMA producer
//   warp  9    MMA issuer; allocates tensor memory
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include "sm100.cuh"
#include "launch_dep.cuh"

namespace fa {

constexpr int kBwdThreads = 320;
constexpr int kBwdBM = 128;  // keys per key tile
constexpr int kBwdBN = 128;  // queries per query tile
// Of every 8 pairs of weights formed without masks in the dK/dV kernel, this
// many use the FMA-pipe polynomial instead of the MUFU: on B200, 2 of 8 took
// 2-3 % less time than none (in the dQ kernel, where the MUFU is not what
// sets the tile period, it gained nothing and stays off).
constexpr int kBwdPolyPairsPer8 = 2;

struct BwdParams {
  // per (batch, query head, 128-row query tile): 128 values of -LSE*log2(e)
  // then 128 values of D = dO . O (rows past Sq: -inf and 0), 1 KB per tile
  const float* ld;
  __nv_bfloat16* dq;   // [B, Hq, Sq, d]
  __nv_bfloat16* dk;   // [B, Hkv, Skv, d]
  __nv_bfloat16* dv;
  int B, Hq, Hkv, Sq, Skv, group, causal;
  int n_kv_tiles, n_q_tiles;
  // CTA order (see bwd_tile)
  int interleave;         // 1: per group of pairs, its dK/dV CTAs then its dQ CTAs
  int heads_per_group;    // (batch, kv-head) pairs per group (dK/dV CTAs, or both roles)
  int q_heads_per_group;  // (batch, query head) pairs per dQ group when not interleaved
  int n_kv_ctas;          // dK/dV CTAs in the grid
  float scale, scale_log2;
  unsigned long long wait_limit_ns;
};

// ---------------------------------------------------------------------------
// Per query row (rows padded to whole 128-row tiles): D = rowsum(dO * O) and
// -LSE*log2(e), packed per tile as the backward kernels read them (a tile's
// 1 KB is one bulk copy).  Rows past Sq get -LSE*log2(e) = -inf and D = 0, so
// their weights and dS are exactly 0.  The kernel only streams O and dO, so
// it is shaped for bandwidth: a lane loads 16 bytes of each, a row is D/8
// lanes, a warp covers kDsumRowsPerWarp rows with all its loads issued before
// the first use.
constexpr int kDsumRowsPerWarp = 8;
constexpr int kDsumRowsPerBlock = 8 * kDsumRowsPerWarp;  // 256 threads

template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dsum_kernel(const __nv_bfloat16* __restrict__ o,
                                                          const __nv_bfloat16* __restrict__ d_o,
                                                          const float* __restrict__ lse,
                                                          float* __restrict__ ld, int Sq,
                                                          int n_q_tiles, long long rows_padded) {
  constexpr int kLanesPerRow = D / 8;                     // 16-byte chunks per row
  constexpr int kRowsPerLoad = 32 / kLanesPerRow;         // rows one warp load covers
  constexpr int kLoads = kDsumRowsPerWarp / kRowsPerLoad;
  // the backward kernel, launched next, may start its setup and loads now;
  // it waits for this grid before reading its output
  grid_dep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow, chunk = lane % kLanesPerRow;
  const long long row0 = static_cast<long long>(blockIdx.x) * kDsumRowsPerBlock +
                         warp * kDsumRowsPerWarp;
  if (row0 >= rows_padded) return;  // (uniform per warp)
  // a warp's rows lie in one head's padded rows (128 is a multiple of them)
  const long long per_head = static_cast<long long>(n_q_tiles) * 128;
  const long long bh = row0 / per_head;
  const int q0 = static_cast<int>(row0 - bh * per_head);
  const __nv_bfloat16* o_h = o + bh * Sq * static_cast<long long>(D);
  const __nv_bfloat16* do_h = d_o + bh * Sq * static_cast<long long>(D);
  uint4 xo[kLoads], xd[kLoads];
#pragma unroll
  for (int l = 0; l < kLoads; ++l) {
    const int qq = q0 + l * kRowsPerLoad + sub;
    xo[l] = make_uint4(0u, 0u, 0u, 0u);
    xd[l] = make_uint4(0u, 0u, 0u, 0u);
    if (qq < Sq) {
      const long long src = static_cast<long long>(qq) * D + chunk * 8;
      xo[l] = __ldg(reinterpret_cast<const uint4*>(o_h + src));
      xd[l] = __ldg(reinterpret_cast<const uint4*>(do_h + src));
    }
  }
  float* dst_h = ld + bh * n_q_tiles * 256;
#pragma unroll
  for (int l = 0; l < kLoads; ++l) {
    const uint32_t* a = reinterpret_cast<const uint32_t*>(&xo[l]);
    const uint32_t* c = reinterpret_cast<const uint32_t*>(&xd[l]);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(__uint_as_float(a[e] << 16), __uint_as_float(c[e] << 16), acc);
      acc = fmaf(__uint_as_float(a[e] & 0xffff0000u), __uint_as_float(c[e] & 0xffff0000u), acc);
    }
#pragma unroll
    for (int s = kLanesPerRow / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    const int qq = q0 + l * kRowsPerLoad + sub;
    if (chunk == 0) {
      float* dst = dst_h + (qq / 128) * 256 + (qq & 127);
      if (qq >= Sq) {
        dst[0] = -INFINITY;
        dst[128] = 0.f;
      } else {
        dst[0] = lse[bh * Sq + qq] * -1.4426950408889634f;
        dst[128] = acc;
      }
    }
  }
}

// Offsets (16-byte descriptor units) of K step kk in a 128B-swizzled tile.
// K-major: rows of 64 elements, step kk at byte (kk / 4) * box + (kk % 4) * 32.
// MN-major: 64-element column blocks one box apart (LBO), step kk at byte
// kk * 16 rows * 128.
__host__ __device__ constexpr uint32_t bwd_km_off(int kk) {
  return static_cast<uint32_t>(((kk / 4) * (128 * 128) + (kk % 4) * 32) >> 4);
}
__host__ __device__ constexpr uint32_t bwd_mn_off(int kk) { return static_cast<uint32_t>(kk * 128); }

// TMEM column of the packed bf16 pairs for elements 16*kk .. 16*kk+15 of a
// 128-wide row whose two 64-wide halves are packed by two warpgroups, each at
// the start of its own 64 columns.
__host__ __device__ constexpr uint32_t bwd_packed_col(int kk) {
  return static_cast<uint32_t>(kk * 8 + (kk >= 4 ? 32 : 0));
}

// d_tmem = A B^T over K = D, A and B K-major 128-row tiles (descriptor bases).
template <int D>
__device__ __forceinline__ void bwd_gemm_kmajor(uint32_t d_tmem, uint64_t a, uint64_t b) {
  constexpr uint32_t kId = idesc_bf16_f32(128, 128, false);
  static_for<D / 16>([&](auto kk_c) {
    constexpr int kk = decltype(kk_c)::value;
    mma_ss_off<bwd_km_off(kk), bwd_km_off(kk)>(d_tmem, a, b, kId, kk > 0 ? 1u : 0u);
  });
}

// ===========================================================================
// dK, dV: key-stationary kernel
// ===========================================================================
template <int D>
struct BwdKvLayout {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxBytes = 128 * 128;  // 128 rows x 64 bf16, 128B swizzled
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kQOff = 2 * kTileBytes;  // stage s: Q at kQOff + 2*s*tile, dO after it
  static constexpr int kDsOff = 6 * kTileBytes;  // dS^T: 128 keys x 128 queries bf16 (2 boxes)
  // stage s: the query tile's 128 values of -LSE*log2(e), then 128 of D
  static constexpr int kLdOff = kDsOff + 128 * 128 * 2;
  static constexpr int kLdBytes = 2 * 128 * 4;
  static constexpr int kBarOff = kLdOff + 2 * kLdBytes;
  static constexpr int kBKv = 0;
  static constexpr int kBQFull = 1;    // [2]
  static constexpr int kBQEmpty = 3;   // [2]
  static constexpr int kBSFull = 5;
  static constexpr int kBDpFull = 6;
  static constexpr int kBPFull = 7;    // 8 arrivals (one per element-wise warp)
  static constexpr int kBDsFull = 8;   // 8 arrivals
  static constexpr int kBDone = 9;
  static constexpr int kBStaged = 10;  // 8 arrivals: dK, dV staged for the stores
  static constexpr int kNumBars = 11;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemSlotOff + 4;
  static constexpr int kContent = kAbortOff + 4;
  // slack for aligning the base to 1024 bytes, as far as the 227 KB allow
  // (the kernel checks that the pad it needs fits)
  static constexpr int kBytes = kContent + 1024 <= 232448 ? kContent + 1024 : 232448;
};
static_assert(BwdKvLayout<128>::kContent <= 232448, "dK/dV shared memory over the limit");

// First query tile that sees any key of key tile j (causal: key k is visible
// to query q iff k <= q + Skv - Sq).
__device__ __forceinline__ int bwd_first_q_tile(const BwdParams& p, int j) {
  if (!p.causal) return 0;
  const long long need = static_cast<long long>(j) * kBwdBM - (p.Skv - p.Sq);  // q >= need
  if (need <= 0) return 0;
  return static_cast<int>(need / kBwdBN);
}

// The CTA's role and tile.  CTAs go out in groups of heads, heavy tiles first
// within a group and role (under a causal mask key tile 0 sees every query
// tile, and the last query tiles see the most keys), so that the data a group
// streams stays in L2 while the launch order stays longest-first.  Two orders:
//  - interleaved: per group of p.heads_per_group (batch, kv-head) pairs, its
//    dK/dV CTAs, key tile by key tile, then the dQ CTAs of its query heads,
//    query tile by query tile: a group's Q, dO, K and V are read from DRAM once
//    for both roles.  Chosen when a group that hides its own longest CTA also
//    leaves room in L2 for the next one.
//  - by role: all dK/dV CTAs (groups of p.heads_per_group pairs), then all dQ
//    CTAs (groups of p.q_heads_per_group query heads).  Chosen when the dK/dV
//    CTAs are long (several query heads per kv head and long sequences): they
//    then all start first, and only short dQ CTAs form the tail; the dQ CTAs
//    read their inputs from DRAM a second time.
struct BwdTile {
  bool kv;    // dK/dV CTA (else dQ CTA)
  int b, hg;  // batch; kv head (dK/dV) or query head (dQ)
  int t;      // key tile (dK/dV) or query tile (dQ)
};
__host__ __device__ inline int bwd_imin(int a, int b) { return a < b ? a : b; }

// The tile of CTA blk (host and device: the host checks the mapping).
__host__ __device__ inline BwdTile bwd_tile_of(const BwdParams& p, int blk) {
  BwdTile tile;
  if (p.interleave) {
    const int units = p.B * p.Hkv;
    const int full = p.heads_per_group * (p.n_kv_tiles + p.group * p.n_q_tiles);
    const int grp = blk / full;
    const int r = blk - grp * full;
    const int in_group = bwd_imin(p.heads_per_group, units - grp * p.heads_per_group);
    const int kv_ctas = in_group * p.n_kv_tiles;
    if (r < kv_ctas) {
      tile.kv = true;
      tile.t = r / in_group;
      const int bg = grp * p.heads_per_group + r % in_group;
      tile.b = bg / p.Hkv;
      tile.hg = bg % p.Hkv;
    } else {
      // the group's query heads are consecutive: (b, g)'s are b*Hq + g*group + [0, group)
      const int q_heads = in_group * p.group;
      const int r2 = r - kv_ctas;
      tile.kv = false;
      tile.t = p.n_q_tiles - 1 - r2 / q_heads;
      const int bh = grp * p.heads_per_group * p.group + r2 % q_heads;
      tile.b = bh / p.Hq;
      tile.hg = bh % p.Hq;
    }
  } else if (blk < p.n_kv_ctas) {
    const int per_group = p.heads_per_group * p.n_kv_tiles;
    const int grp = blk / per_group;
    const int r = blk % per_group;
    const int in_group = bwd_imin(p.heads_per_group, p.B * p.Hkv - grp * p.heads_per_group);
    tile.kv = true;
    tile.t = r / in_group;
    const int bg = grp * p.heads_per_group + r % in_group;
    tile.b = bg / p.Hkv;
    tile.hg = bg % p.Hkv;
  } else {
    const int cta = blk - p.n_kv_ctas;
    const int per_group = p.q_heads_per_group * p.n_q_tiles;
    const int grp = cta / per_group;
    const int r = cta % per_group;
    const int in_group = bwd_imin(p.q_heads_per_group, p.B * p.Hq - grp * p.q_heads_per_group);
    tile.kv = false;
    tile.t = p.n_q_tiles - 1 - r / in_group;
    const int bh = grp * p.q_heads_per_group + r % in_group;
    tile.b = bh / p.Hq;
    tile.hg = bh % p.Hq;
  }
  return tile;
}
__device__ __forceinline__ BwdTile bwd_tile(const BwdParams& p) {
  return bwd_tile_of(p, static_cast<int>(blockIdx.x));
}

__device__ __forceinline__ void bwd_kv_cta(const BwdParams& p, int& b, int& g, int& j) {
  const BwdTile tile = bwd_tile(p);
  b = tile.b;
  g = tile.hg;
  j = tile.t;
}

template <int D>
__device__ __forceinline__ void bwd_kv_producer(const CUtensorMap* tq, const CUtensorMap* tk,
                                                const CUtensorMap* tv, const CUtensorMap* tdo,
                                                const BwdParams& p, uint32_t sbase,
                                                volatile int* abort_flag) {
  using L = BwdKvLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  int b, g, j;
  bwd_kv_cta(p, b, g, j);
  tma_prefetch_desc(tq);
  tma_prefetch_desc(tk);
  tma_prefetch_desc(tv);
  tma_prefetch_desc(tdo);
  const uint32_t bkv = bars + 8 * L::kBKv;
  mbar_arrive_expect_tx(bkv, 2 * L::kTileBytes);
#pragma unroll
  for (int kb = 0; kb < D / 64; ++kb) {
    tma_load_3d(sbase + L::kKOff + kb * L::kBoxBytes, tk, bkv, kb * 64, j * kBwdBM, b * p.Hkv + g);
    tma_load_3d(sbase + L::kVOff + kb * L::kBoxBytes, tv, bkv, kb * 64, j * kBwdBM, b * p.Hkv + g);
  }
  const int i0 = bwd_first_q_tile(p, j);
  uint32_t n = 0;  // query tiles loaded
  for (int hh = 0; hh < p.group; ++hh) {
    const int plane = b * p.Hq + g * p.group + hh;
    for (int i = i0; i < p.n_q_tiles; ++i, ++n) {
      const uint32_t s = n & 1u;
      if (!mbar_wait(bars + 8 * (L::kBQEmpty + s), ((n >> 1) & 1u) ^ 1u, abort_flag,
                     p.wait_limit_ns))
        goto drain;
      const uint32_t full = bars + 8 * (L::kBQFull + s);
      const uint32_t qa = sbase + L::kQOff + 2 * s * L::kTileBytes;
      mbar_arrive_expect_tx(full, 2 * L::kTileBytes + L::kLdBytes);
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb) {
        tma_load_3d(qa + kb * L::kBoxBytes, tq, full, kb * 64, i * kBwdBN, plane);
        tma_load_3d(qa + L::kTileBytes + kb * L::kBoxBytes, tdo, full, kb * 64, i * kBwdBN, plane);
      }
      grid_dep_wait();  // the D kernel's per-tile values are complete (free after the first)
      bulk_load(sbase + L::kLdOff + s * L::kLdBytes,
                p.ld + (static_cast<size_t>(plane) * p.n_q_tiles + i) * 256, L::kLdBytes, full);
    }
  }
drain:
  mbar_wait(bkv, 0u, nullptr, p.wait_limit_ns);
  for (uint32_t k = (n > 2 ? n - 2 : 0u); k < n; ++k)
    mbar_wait(bars + 8 * (L::kBQFull + (k & 1u)), (k >> 1) & 1u, nullptr, p.wait_limit_ns);
}

// Per query tile n the MMA thread issues dV_n once P_n is announced, the next
// tile's S^T (its columns hold P_n, which dV_n reads first), then dK_n once
// dS_n is in shared memory, and the next tile's dP^T (the element-wise warps
// have read dP_n before announcing dS_n).  dK_n precedes dP^T_{n+1}, so the
// commit that announces dP^T_{n+1} also covers dK_n's reads of dS_n, which
// the next dS overwrites.
template <int D>
__device__ __forceinline__ void bwd_kv_mma(const BwdParams& p, uint32_t sbase, uint32_t tmem,
                                           volatile int* abort_flag) {
  using L = BwdKvLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  constexpr uint32_t kIdAcc = idesc_bf16_f32(kBwdBM, D, true);  // A K-major, B MN-major
  const uint32_t t_dv = tmem, t_dk = tmem + 128, t_s = tmem + 256, t_dp = tmem + 384;
  int b, g, j;
  bwd_kv_cta(p, b, g, j);
  const int i0 = bwd_first_q_tile(p, j);
  const int per_head = p.n_q_tiles - i0;
  const uint32_t total = per_head > 0 ? static_cast<uint32_t>(per_head * p.group) : 0u;
  auto wait = [&](int bar, uint32_t parity) -> bool {
    if (!mbar_wait(bars + 8 * bar, parity, abort_flag, p.wait_limit_ns)) return false;
    tc_fence_after();
    return true;
  };
  // Descriptors are built once; a K step adds a compile-time offset inside
  // the MMA's own asm, a Q/dO stage a multiple of the stage size.
  const uint64_t k_km = sw128_desc(sbase + L::kKOff, 16, 1024);
  const uint64_t v_km = sw128_desc(sbase + L::kVOff, 16, 1024);
  const uint64_t ds_km = sw128_desc(sbase + L::kDsOff, 16, 1024);
  const uint64_t q_km0 = sw128_desc(sbase + L::kQOff, 16, 1024);
  const uint64_t q_mn0 = sw128_desc(sbase + L::kQOff, L::kBoxBytes, 1024);
  constexpr uint64_t kStageStep = (2 * L::kTileBytes) >> 4;
  constexpr uint64_t kDoStep = L::kTileBytes >> 4;  // dO after Q
  if (total > 0) {
    if (!wait(L::kBKv, 0u) || !wait(L::kBQFull + 0, 0u)) goto done;
    bwd_gemm_kmajor<D>(t_s, k_km, q_km0);             // S^T = K Q^T
    mma_commit(bars + 8 * L::kBSFull);
    bwd_gemm_kmajor<D>(t_dp, v_km, q_km0 + kDoStep);  // dP^T = V dO^T
    mma_commit(bars + 8 * L::kBDpFull);
  }
  for (uint32_t n = 0; n < total; ++n) {
    const uint32_t s = n & 1u, ph = n & 1u;
    const uint64_t q_mn = q_mn0 + s * kStageStep, do_mn = q_mn + kDoStep;
    const bool more = n + 1 < total;
    const uint32_t s1 = (n + 1) & 1u;
    const uint64_t q_km1 = q_km0 + s1 * kStageStep;
    if (!wait(L::kBPFull, ph)) goto done;
    static_for<kBwdBN / 16>([&](auto kk_c) {      // dV += P^T dO
      constexpr int kk = decltype(kk_c)::value;
      mma_ts_off<bwd_mn_off(kk)>(t_dv, t_s + bwd_packed_col(kk), do_mn, kIdAcc,
                                 (n > 0 || kk > 0) ? 1u : 0u);
    });
    if (more) {                                   // next tile's scores
      if (!wait(L::kBQFull + s1, ((n + 1) >> 1) & 1u)) goto done;
      bwd_gemm_kmajor<D>(t_s, k_km, q_km1);
      mma_commit(bars + 8 * L::kBSFull);
    }
    if (!wait(L::kBDsFull, ph)) goto done;
    static_for<kBwdBN / 16>([&](auto kk_c) {      // dK += dS^T Q (K-dim = queries)
      constexpr int kk = decltype(kk_c)::value;
      mma_ss_off<bwd_km_off(kk), bwd_mn_off(kk)>(t_dk, ds_km, q_mn, kIdAcc,
                                                 (n > 0 || kk > 0) ? 1u : 0u);
    });
    mma_commit(bars + 8 * (L::kBQEmpty + s));     // Q_n, dO_n read by everything issued so far
    if (more) {                                   // next tile's dP^T
      bwd_gemm_kmajor<D>(t_dp, v_km, q_km1 + kDoStep);
      mma_commit(bars + 8 * L::kBDpFull);
    }
  }
done:
  mma_commit(bars + 8 * L::kBDone);
  mbar_wait(bars + 8 * L::kBDone, 0u, nullptr, p.wait_limit_ns);
}

// Element-wise warpgroups (warps 0-7).  Warpgroup hf takes queries
// [64*hf, 64*hf + 64) of each tile for P and dS (thread t = key row t, the
// TMEM lane) and d-columns [hf*D/2, (hf+1)*D/2) of dK, dV at the end.
template <int D>
__device__ __forceinline__ void bwd_kv_elementwise(const BwdParams& p, uint32_t sbase,
                                                   uint8_t* smem, uint32_t tmem,
                                                   const CUtensorMap* tm_dk,
                                                   const CUtensorMap* tm_dv,
                                                   volatile int* abort_flag) {
  using L = BwdKvLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  const int t = threadIdx.x & 127;
  const int hf = threadIdx.x >> 7;  // warpgroup: query half / column half
  const int warp = (threadIdx.x >> 5) & 3;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t t_dv = tmem + lane_off, t_dk = tmem + lane_off + 128;
  const uint32_t t_s = tmem + lane_off + 256, t_dp = tmem + lane_off + 384;
  constexpr int kQH = kBwdBN / 2;   // queries per warpgroup
  constexpr int kDH = D / 2;        // d-columns per warpgroup
  uint8_t* ds_smem = smem + L::kDsOff;
  int b, g, j;
  bwd_kv_cta(p, b, g, j);
  const int key = j * kBwdBM + t;
  const int off = p.Skv - p.Sq;
  const int i0 = bwd_first_q_tile(p, j);
  uint32_t n = 0;
  bool ok = true;
  for (int hh = 0; hh < p.group && ok; ++hh) {
    for (int i = i0; i < p.n_q_tiles; ++i, ++n) {
      const uint32_t ph = n & 1u;
      const int q0 = i * kBwdBN;
      // the tile's -LSE (log2 units) and D arrived with its Q and dO (the
      // stage is reloaded only after dK_n, which follows this tile's dS)
      const float* lse_s = reinterpret_cast<const float*>(smem + L::kLdOff + (n & 1u) * L::kLdBytes);
      const float* d_s = lse_s + 128;
      ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (L::kBQFull + (n & 1u)), (n >> 1) & 1u,
                                             abort_flag, p.wait_limit_ns));
      if (!ok) break;
      // P^T for this key and the warpgroup's queries: p = 2^(s*scale*log2e - LSE*log2e)
      // (a key that every query of the half sees takes the branch without masks)
      ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * L::kBSFull, ph, abort_flag, p.wait_limit_ns));
      if (!ok) break;
      tc_fence_after();
      uint32_t pk[kQH / 2];
      {
        const int lim = key - off;  // first query that sees this key
        const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
        const bool all_vis = (key < p.Skv) && (!p.causal || q0 + hf * kQH >= lim);
        const bool fast = __all_sync(0xffffffffu, all_vis);
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {  // 32 queries per pass
          uint32_t ra[32];
          tmem_ld32(t_s + hf * kQH + hq * 32, ra);
          if (fast) {
#pragma unroll
            for (int c2 = 0; c2 < 16; ++c2) {
              const float2 nl = *reinterpret_cast<const float2*>(lse_s + hf * kQH + hq * 32 + 2 * c2);
              const float2 x = ffma2(make_float2(__uint_as_float(ra[2 * c2]),
                                                 __uint_as_float(ra[2 * c2 + 1])), sl2, nl);
              if ((c2 & 7) >= 8 - kBwdPolyPairsPer8) {  // the FMA-pipe polynomial
                const float2 e = exp2_poly2(x);
                pk[hq * 16 + c2] = pack_bf16x2(e.x, e.y);
              } else {
                pk[hq * 16 + c2] = pack_bf16x2(ex2(x.x), ex2(x.y));
              }
            }
          } else {
#pragma unroll
            for (int c2 = 0; c2 < 16; ++c2) {
              float pr[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int c = hf * kQH + hq * 32 + 2 * c2 + e;
                const bool vis = (key < p.Skv) && (!p.causal || q0 + c >= lim);
                const float x = fmaf(__uint_as_float(ra[2 * c2 + e]), p.scale_log2, lse_s[c]);
                pr[e] = vis ? ex2(x) : 0.f;
              }
              pk[hq * 16 + c2] = pack_bf16x2(pr[0], pr[1]);
            }
          }
        }
      }
      // packed pairs of queries, inside this warpgroup's own (already read)
      // score columns: the other warpgroup's scores are never overwritten
      tmem_st32(t_s + hf * kQH, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bars + 8 * L::kBPFull);

      // dS = P * (dP - D) to shared memory: rows = keys, 64-query boxes, 128B
      // swizzle (the K-major A operand of dK += dS^T Q)
      ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * L::kBDpFull, ph, abort_flag, p.wait_limit_ns));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {  // 32 queries per pass
        uint32_t dp[32];
        tmem_ld32(t_dp + hf * kQH + hq * 32, dp);
        uint32_t dsk[16];
        const float2 m1 = make_float2(-1.f, -1.f);
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          const int cl = hq * 32 + 2 * e2;  // local query index in the half
          // the pair of bf16 weights as fp32, and dP - D rounded once, as pairs
          const uint32_t pw = pk[cl >> 1];
          const float2 pf = make_float2(__uint_as_float(pw << 16), __uint_as_float(pw & 0xffff0000u));
          const float2 dd = *reinterpret_cast<const float2*>(d_s + hf * kQH + cl);
          const float2 t2 = ffma2(dd, m1, make_float2(__uint_as_float(dp[2 * e2]),
                                                      __uint_as_float(dp[2 * e2 + 1])));
          const float2 ds2 = fmul2(pf, t2);
          dsk[e2] = pack_bf16x2(ds2.x, ds2.y);
        }
        // queries hf*64 + hq*32 .. +31: box hf, 16-byte chunks hq*4 .. +3 of row t
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int chunk = hq * 4 + k4;
          uint4* dst = reinterpret_cast<uint4*>(ds_smem + hf * L::kBoxBytes + t * 128 +
                                                ((chunk ^ (t & 7)) * 16));
          *dst = make_uint4(dsk[4 * k4], dsk[4 * k4 + 1], dsk[4 * k4 + 2], dsk[4 * k4 + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();  // the dP^T loads are complete before the next dP^T overwrites them
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bars + 8 * L::kBDsFull);
    }
  }
  if (!ok) return;

  // dK = scale * (dS^T Q summed), dV = P^T dO summed: thread t = key row,
  // this warpgroup's d-columns, staged as 128B-swizzled boxes in the (now
  // idle) Q/dO ring and written by tiled bulk stores, which skip rows past Skv.
  if (!__all_sync(0xffffffffu, mbar_wait(bars + 8 * L::kBDone, 0u, abort_flag, p.wait_limit_ns)))
    return;
  tc_fence_after();
  const bool any = (i0 < p.n_q_tiles);
  constexpr int kBoxes = D / 64;  // 64-column boxes per gradient tile
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    const float mul = (which == 0) ? 1.f : p.scale;
    uint8_t* stage = smem + L::kQOff + which * kBoxes * L::kBoxBytes;
#pragma unroll
    for (int c4 = 0; c4 < kDH / 32; ++c4) {
      uint32_t r[32];
      tmem_ld32((which == 0 ? t_dv : t_dk) + hf * kDH + c4 * 32, r);
      const int col0 = hf * kDH + c4 * 32;  // first d-column of these 32
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        const float* f = reinterpret_cast<const float*>(r) + v4 * 8;
        const int col = col0 + v4 * 8;
        const int chunk = (col & 63) >> 3;
        uint4* dst = reinterpret_cast<uint4*>(stage + (col >> 6) * L::kBoxBytes + t * 128 +
                                              ((chunk ^ (t & 7)) * 16));
        *dst = make_uint4(pack_bf16x2(any ? f[0] * mul : 0.f, any ? f[1] * mul : 0.f),
                          pack_bf16x2(any ? f[2] * mul : 0.f, any ? f[3] * mul : 0.f),
                          pack_bf16x2(any ? f[4] * mul : 0.f, any ? f[5] * mul : 0.f),
                          pack_bf16x2(any ? f[6] * mul : 0.f, any ? f[7] * mul : 0.f));
      }
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bars + 8 * L::kBStaged);
  // one thread stores once every warp has staged its rows (a bounded wait:
  // a warp that gave up earlier never arrives, and then nothing is stored)
  if (threadIdx.x == 0 && mbar_wait(bars + 8 * L::kBStaged, 0u, abort_flag, p.wait_limit_ns)) {
#pragma unroll
    for (int which = 0; which < 2; ++which)
#pragma unroll
      for (int kb = 0; kb < kBoxes; ++kb)
        tma_store_3d(which == 0 ? tm_dv : tm_dk,
                     sbase + L::kQOff + (which * kBoxes + kb) * L::kBoxBytes, kb * 64,
                     j * kBwdBM, b * p.Hkv + g);
    bulk_commit_group();
    bulk_wait_group0();
  }
}

template <int D>
struct BwdQLayout;

// Shared memory of a backward CTA: the larger of the two roles' layouts.
template <int D>
__host__ __device__ constexpr int bwd_smem_bytes() {
  return BwdKvLayout<D>::kBytes > BwdQLayout<D>::kBytes ? BwdKvLayout<D>::kBytes
                                                         : BwdQLayout<D>::kBytes;
}

// One dK/dV CTA (the whole block).
template <int D>
__device__ __forceinline__ void bwd_dkdv_block(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                               const CUtensorMap* tm_v, const CUtensorMap* tm_do,
                                               const CUtensorMap* tm_dk, const CUtensorMap* tm_dv,
                                               const BwdParams& p, uint8_t* smem_raw) {
  using L = BwdKvLayout<D>;
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  if (pad + L::kContent > static_cast<uint32_t>(bwd_smem_bytes<D>())) {  // uniform: every thread leaves
    if (threadIdx.x == 0) atomicExch(&g_device_status, kStatusTimeout);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbortOff);
  const uint32_t bars = sbase + L::kBarOff;
  if (threadIdx.x == 0) {
    mbar_init(bars + 8 * L::kBKv, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bars + 8 * (L::kBQFull + s), 1);
      mbar_init(bars + 8 * (L::kBQEmpty + s), 1);
    }
    mbar_init(bars + 8 * L::kBSFull, 1);
    mbar_init(bars + 8 * L::kBDpFull, 1);
    mbar_init(bars + 8 * L::kBPFull, 8);   // one arrival per element-wise warp
    mbar_init(bars + 8 * L::kBDsFull, 8);
    mbar_init(bars + 8 * L::kBDone, 1);
    mbar_init(bars + 8 * L::kBStaged, 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(sbase + L::kTmemSlotOff, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlotOff);

  if (warp < 8) {
    bwd_kv_elementwise<D>(p, sbase, smem, tmem, tm_dk, tm_dv, abort_flag);
  } else if (warp == 8) {
    if (lane == 0) bwd_kv_producer<D>(tm_q, tm_k, tm_v, tm_do, p, sbase, abort_flag);
  } else {
    if (lane == 0) bwd_kv_mma<D>(p, sbase, tmem, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// dQ: query-stationary kernel
// ===========================================================================
template <int D>
struct BwdQLayout {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kQOff = 0;
  static constexpr int kDoOff = kTileBytes;
  static constexpr int kKOff = 2 * kTileBytes;                    // K stage s at kKOff + s*tile
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;     // V stage s at kVOff + s*tile
  static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
  static constexpr int kBQ = 0;                          // Q_i and dO_i loaded
  static constexpr int kBKFull = 1;                      // [kKStages]
  static constexpr int kBKEmpty = kBKFull + kKStages;    // [kKStages]
  static constexpr int kBVFull = kBKEmpty + kKStages;    // [kVStages]
  static constexpr int kBVEmpty = kBVFull + kVStages;    // [kVStages]
  static constexpr int kBSFull = kBVEmpty + kVStages;    // [2] one per S buffer
  static constexpr int kBDpFull = kBSFull + 2;
  static constexpr int kBDsFull = kBDpFull + 1;          // 8 arrivals (one per element-wise warp)
  static constexpr int kBDone = kBDsFull + 1;
  static constexpr int kBStaged = kBDone + 1;            // 8 arrivals: dQ staged for the stores
  static constexpr int kNumBars = kBStaged + 1;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemSlotOff + 4;
  static constexpr int kContent = kAbortOff + 4;
  static constexpr int kBytes = kContent + 1024 <= 232448 ? kContent + 1024 : 232448;
};
static_assert(BwdQLayout<128>::kBytes <= 232448, "dQ shared memory over the limit");

__device__ __forceinline__ void bwd_q_cta(const BwdParams& p, int& b, int& h, int& i) {
  const BwdTile tile = bwd_tile(p);
  b = tile.b;
  h = tile.hg;
  i = tile.t;
}

// Key tiles that query tile i sees: [0, n).
__device__ __forceinline__ int bwd_q_kv_tiles(const BwdParams& p, int i) {
  if (!p.causal) return p.n_kv_tiles;
  const long long q_last = min(static_cast<long long>(i) * kBwdBN + kBwdBN - 1,
                               static_cast<long long>(p.Sq) - 1);
  const long long k_last = q_last + (p.Skv - p.Sq);  // last key the last row sees
  if (k_last < 0) return 0;
  return static_cast<int>(min(static_cast<long long>(p.n_kv_tiles), k_last / kBwdBM + 1));
}

template <int D>
__device__ __forceinline__ void bwd_q_producer(const CUtensorMap* tq, const CUtensorMap* tk,
                                               const CUtensorMap* tv, const CUtensorMap* tdo,
                                               const BwdParams& p, uint32_t sbase,
                                               volatile int* abort_flag) {
  using L = BwdQLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  int b, h, i;
  bwd_q_cta(p, b, h, i);
  const int nk = bwd_q_kv_tiles(p, i);
  if (nk == 0) return;
  tma_prefetch_desc(tq);
  tma_prefetch_desc(tk);
  tma_prefetch_desc(tv);
  tma_prefetch_desc(tdo);
  const int g = h / p.group;
  const uint32_t bq = bars + 8 * L::kBQ;
  mbar_arrive_expect_tx(bq, 2 * L::kTileBytes);
#pragma unroll
  for (int kb = 0; kb < D / 64; ++kb) {
    tma_load_3d(sbase + L::kQOff + kb * L::kBoxBytes, tq, bq, kb * 64, i * kBwdBN, b * p.Hq + h);
    tma_load_3d(sbase + L::kDoOff + kb * L::kBoxBytes, tdo, bq, kb * 64, i * kBwdBN, b * p.Hq + h);
  }
  int jn = 0;  // key tiles whose K and V were both issued
  for (; jn < nk; ++jn) {
    const int ks = jn % L::kKStages, vs = jn % L::kVStages;
    if (!mbar_wait(bars + 8 * (L::kBKEmpty + ks),
                   (static_cast<uint32_t>(jn / L::kKStages) & 1u) ^ 1u, abort_flag, p.wait_limit_ns))
      break;
    const uint32_t kfull = bars + 8 * (L::kBKFull + ks);
    mbar_arrive_expect_tx(kfull, L::kTileBytes);
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb)
      tma_load_3d(sbase + L::kKOff + ks * L::kTileBytes + kb * L::kBoxBytes, tk, kfull, kb * 64,
                  jn * kBwdBM, b * p.Hkv + g);
    if (!mbar_wait(bars + 8 * (L::kBVEmpty + vs),
                   (static_cast<uint32_t>(jn / L::kVStages) & 1u) ^ 1u, abort_flag, p.wait_limit_ns)) {
      mbar_wait(kfull, static_cast<uint32_t>(jn / L::kKStages) & 1u, nullptr, p.wait_limit_ns);
      break;
    }
    const uint32_t vfull = bars + 8 * (L::kBVFull + vs);
    mbar_arrive_expect_tx(vfull, L::kTileBytes);
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb)
      tma_load_3d(sbase + L::kVOff + vs * L::kTileBytes + kb * L::kBoxBytes, tv, vfull, kb * 64,
                  jn * kBwdBM, b * p.Hkv + g);
  }
  // drain: the CTA does not exit with copies in flight
  mbar_wait(bq, 0u, nullptr, p.wait_limit_ns);
  for (int k = (jn > L::kKStages ? jn - L::kKStages : 0); k < jn; ++k)
    mbar_wait(bars + 8 * (L::kBKFull + k % L::kKStages),
              static_cast<uint32_t>(k / L::kKStages) & 1u, nullptr, p.wait_limit_ns);
  for (int k = (jn > L::kVStages ? jn - L::kVStages : 0); k < jn; ++k)
    mbar_wait(bars + 8 * (L::kBVFull + k % L::kVStages),
              static_cast<uint32_t>(k / L::kVStages) & 1u, nullptr, p.wait_limit_ns);
}

// Per key tile j: dQ_j once dS_j is announced (it reads dS_j from S buffer
// j%2 and K_j), which frees K_j's stage; then dP_{j+1} (the element-wise
// warps have read dP_j before announcing dS_j), which frees V_{j+1}'s stage
// once done, and S_{j+2} into buffer j%2 (after dQ_j, which reads it, in
// issue order).
template <int D>
__device__ __forceinline__ void bwd_q_mma(const BwdParams& p, uint32_t sbase, uint32_t tmem,
                                          volatile int* abort_flag) {
  using L = BwdQLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  constexpr uint32_t kIdDq = idesc_bf16_f32(kBwdBN, D, true);  // A TMEM, B MN-major
  const uint32_t t_s0 = tmem, t_dp = tmem + 256, t_dq = tmem + 384;
  int b, h, i;
  bwd_q_cta(p, b, h, i);
  const int nk = bwd_q_kv_tiles(p, i);
  auto wait = [&](int bar, uint32_t parity) -> bool {
    if (!mbar_wait(bars + 8 * bar, parity, abort_flag, p.wait_limit_ns)) return false;
    tc_fence_after();
    return true;
  };
  auto k_wait = [&](int jj) -> bool {
    return wait(L::kBKFull + jj % L::kKStages, static_cast<uint32_t>(jj / L::kKStages) & 1u);
  };
  auto v_wait = [&](int jj) -> bool {
    return wait(L::kBVFull + jj % L::kVStages, static_cast<uint32_t>(jj / L::kVStages) & 1u);
  };
  const uint64_t q_km = sw128_desc(sbase + L::kQOff, 16, 1024);
  const uint64_t do_km = sw128_desc(sbase + L::kDoOff, 16, 1024);
  const uint64_t k_km0 = sw128_desc(sbase + L::kKOff, 16, 1024);
  const uint64_t k_mn0 = sw128_desc(sbase + L::kKOff, L::kBoxBytes, 1024);
  const uint64_t v_km0 = sw128_desc(sbase + L::kVOff, 16, 1024);
  constexpr uint64_t kTileStep = L::kTileBytes >> 4;  // one stage, descriptor units
  // dP_j = dO V_j^T, then V_j's stage is free once it completes
  auto issue_dp = [&](int jj) {
    const int vs = jj % L::kVStages;
    bwd_gemm_kmajor<D>(t_dp, do_km, v_km0 + vs * kTileStep);
    mma_commit(bars + 8 * L::kBDpFull);
    mma_commit(bars + 8 * (L::kBVEmpty + vs));
  };
  if (nk > 0) {
    if (!wait(L::kBQ, 0u) || !k_wait(0)) goto done;
    bwd_gemm_kmajor<D>(t_s0, q_km, k_km0);               // S_0 = Q K_0^T
    mma_commit(bars + 8 * (L::kBSFull + 0));
    if (!v_wait(0)) goto done;
    issue_dp(0);
    if (nk > 1) {
      if (!k_wait(1)) goto done;
      bwd_gemm_kmajor<D>(t_s0 + 128, q_km, k_km0 + kTileStep);
      mma_commit(bars + 8 * (L::kBSFull + 1));
    }
  }
  for (int jj = 0; jj < nk; ++jj) {
    const int buf = jj & 1;
    const int ks = jj % L::kKStages;
    if (!wait(L::kBDsFull, static_cast<uint32_t>(jj) & 1u)) goto done;
    const uint64_t k_mn = k_mn0 + ks * kTileStep;
    const uint32_t t_ds = t_s0 + 128 * buf;
    static_for<kBwdBM / 16>([&](auto kk_c) {             // dQ += dS K (K-dim = keys)
      constexpr int kk = decltype(kk_c)::value;
      mma_ts_off<bwd_mn_off(kk)>(t_dq, t_ds + bwd_packed_col(kk), k_mn, kIdDq,
                                 (jj > 0 || kk > 0) ? 1u : 0u);
    });
    mma_commit(bars + 8 * (L::kBKEmpty + ks));           // K_j consumed
    if (jj + 1 < nk) {
      if (!v_wait(jj + 1)) goto done;
      issue_dp(jj + 1);
    }
    if (jj + 2 < nk) {                                    // S_{j+2} into buffer j%2
      if (!k_wait(jj + 2)) goto done;
      const int ks2 = (jj + 2) % L::kKStages;
      bwd_gemm_kmajor<D>(t_ds, q_km, k_km0 + ks2 * kTileStep);
      mma_commit(bars + 8 * (L::kBSFull + buf));
    }
  }
done:
  mma_commit(bars + 8 * L::kBDone);
  mbar_wait(bars + 8 * L::kBDone, 0u, nullptr, p.wait_limit_ns);
}

// Element-wise warpgroups: thread = query row (its TMEM lane); warpgroup hf
// takes keys [64*hf, 64*hf + 64) of each key tile, and d-columns
// [hf*D/2, (hf+1)*D/2) of dQ at the end.
template <int D>
__device__ __forceinline__ void bwd_q_elementwise(const BwdParams& p, uint32_t sbase,
                                                  uint8_t* smem, uint32_t tmem,
                                                  const CUtensorMap* tm_dq,
                                                  volatile int* abort_flag) {
  using L = BwdQLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  const int hf = threadIdx.x >> 7;
  const int warp = (threadIdx.x >> 5) & 3;
  const int row = warp * 32 + (threadIdx.x & 31);
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t t_s0 = tmem + lane_off, t_dp = tmem + lane_off + 256, t_dq = tmem + lane_off + 384;
  constexpr int kKH = kBwdBM / 2;  // keys per warpgroup
  constexpr int kDH = D / 2;
  int b, h, i;
  bwd_q_cta(p, b, h, i);
  const int nk = bwd_q_kv_tiles(p, i);
  const int q = i * kBwdBN + row;
  // -LSE in log2 units (rows past Sq: -inf, weights exactly 0) and D
  grid_dep_wait();  // the D kernel's per-tile values are complete
  const float* ldt = p.ld + (static_cast<size_t>(b * p.Hq + h) * p.n_q_tiles + i) * 256;
  const float nlse = ldt[row];
  const float dval = ldt[128 + row];
  const int off = p.Skv - p.Sq;
  const float2 sl2 = make_float2(p.scale_log2, p.scale_log2);
  const float2 nl2 = make_float2(nlse, nlse);
  bool ok = true;
  for (int jj = 0; jj < nk; ++jj) {
    const int buf = jj & 1;
    const uint32_t t_s = t_s0 + 128 * buf;
    ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * (L::kBSFull + buf),
                                           static_cast<uint32_t>(jj >> 1) & 1u, abort_flag,
                                           p.wait_limit_ns));
    if (!ok) break;
    tc_fence_after();
    // P = 2^(s*scale*log2e - LSE*log2e) for this row and the warpgroup's keys
    const int k0 = jj * kBwdBM + hf * kKH;  // first key of this half
    float pr[kKH];
    {
      uint32_t ra[64];
      tmem_ld64_nowait(t_s + hf * kKH, ra);
      tmem_ld_wait_hold(ra);
      const bool all_vis = (k0 + kKH <= p.Skv) && (!p.causal || k0 + kKH - 1 <= q + off);
      if (__all_sync(0xffffffffu, all_vis)) {
#pragma unroll
        for (int c2 = 0; c2 < kKH / 2; ++c2) {
          const float2 x = ffma2(make_float2(__uint_as_float(ra[2 * c2]),
                                             __uint_as_float(ra[2 * c2 + 1])), sl2, nl2);
          pr[2 * c2] = ex2(x.x);
          pr[2 * c2 + 1] = ex2(x.y);
        }
      } else {
        // keys [k0, k0 + lim) of the half are visible to this row
        const int lim = (p.causal ? min(p.Skv, q + off + 1) : p.Skv) - k0;
#pragma unroll
        for (int c = 0; c < kKH; ++c) {
          const float x = fmaf(__uint_as_float(ra[c]), p.scale_log2, nlse);
          pr[c] = (c < lim) ? ex2(x) : 0.f;
        }
      }
    }
    // dS = P * (dP - D), packed bf16 pairs into this warpgroup's own
    // (already read) score columns: the A operand of dQ += dS K
    ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * L::kBDpFull, static_cast<uint32_t>(jj) & 1u,
                                           abort_flag, p.wait_limit_ns));
    if (!ok) break;
    tc_fence_after();
#pragma unroll
    for (int hk = 0; hk < 2; ++hk) {  // 32 keys per pass
      uint32_t dp[32];
      tmem_ld32(t_dp + hf * kKH + hk * 32, dp);
      uint32_t dsk[16];
      const float2 nd2 = make_float2(-dval, -dval);
#pragma unroll
      for (int e2 = 0; e2 < 16; ++e2) {
        const int c = hk * 32 + 2 * e2;
        const float2 ds2 = fmul2(make_float2(pr[c], pr[c + 1]),
                                 fadd2(make_float2(__uint_as_float(dp[2 * e2]),
                                                   __uint_as_float(dp[2 * e2 + 1])), nd2));
        dsk[e2] = pack_bf16x2(ds2.x, ds2.y);
      }
      tmem_st16(t_s + hf * kKH + hk * 16, dsk);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bars + 8 * L::kBDsFull);
  }
  if (!ok) return;
  // dQ = scale * (dS K summed): this row, the warpgroup's d-columns (zero for
  // a tile that sees no key)
  if (nk > 0) {
    if (!__all_sync(0xffffffffu, mbar_wait(bars + 8 * L::kBDone, 0u, abort_flag, p.wait_limit_ns)))
      return;
    tc_fence_after();
  }
  // staged as 128B-swizzled boxes in the (now idle) Q/dO buffers and written
  // by tiled bulk stores, which skip rows past Sq
  uint8_t* stage = smem + L::kQOff;
#pragma unroll
  for (int c4 = 0; c4 < kDH / 32; ++c4) {
    uint32_t r[32];
    if (nk > 0) {
      tmem_ld32(t_dq + hf * kDH + c4 * 32, r);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) r[e] = 0u;
    }
    const int col0 = hf * kDH + c4 * 32;
#pragma unroll
    for (int v4 = 0; v4 < 4; ++v4) {
      const float* f = reinterpret_cast<const float*>(r) + v4 * 8;
      const int col = col0 + v4 * 8;
      const int chunk = (col & 63) >> 3;
      uint4* dst = reinterpret_cast<uint4*>(stage + (col >> 6) * L::kBoxBytes + row * 128 +
                                            ((chunk ^ (row & 7)) * 16));
      *dst = make_uint4(pack_bf16x2(f[0] * p.scale, f[1] * p.scale),
                        pack_bf16x2(f[2] * p.scale, f[3] * p.scale),
                        pack_bf16x2(f[4] * p.scale, f[5] * p.scale),
                        pack_bf16x2(f[6] * p.scale, f[7] * p.scale));
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bars + 8 * L::kBStaged);
  if (threadIdx.x == 0 && mbar_wait(bars + 8 * L::kBStaged, 0u, abort_flag, p.wait_limit_ns)) {
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb)
      tma_store_3d(tm_dq, sbase + L::kQOff + kb * L::kBoxBytes, kb * 64, i * kBwdBN,
                   b * p.Hq + h);
    bulk_commit_group();
    bulk_wait_group0();
  }
}

// One dQ CTA (the whole block).
template <int D>
__device__ __forceinline__ void bwd_dq_block(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                             const CUtensorMap* tm_v, const CUtensorMap* tm_do,
                                             const CUtensorMap* tm_dq, const BwdParams& p,
                                             uint8_t* smem_raw) {
  using L = BwdQLayout<D>;
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  if (pad + L::kContent > static_cast<uint32_t>(bwd_smem_bytes<D>())) {  // uniform: every thread leaves
    if (threadIdx.x == 0) atomicExch(&g_device_status, kStatusTimeout);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbortOff);
  const uint32_t bars = sbase + L::kBarOff;
  if (threadIdx.x == 0) {
    mbar_init(bars + 8 * L::kBQ, 1);
    for (int s = 0; s < L::kKStages; ++s) {
      mbar_init(bars + 8 * (L::kBKFull + s), 1);
      mbar_init(bars + 8 * (L::kBKEmpty + s), 1);
    }
    for (int s = 0; s < L::kVStages; ++s) {
      mbar_init(bars + 8 * (L::kBVFull + s), 1);
      mbar_init(bars + 8 * (L::kBVEmpty + s), 1);
    }
    mbar_init(bars + 8 * (L::kBSFull + 0), 1);
    mbar_init(bars + 8 * (L::kBSFull + 1), 1);
    mbar_init(bars + 8 * L::kBDpFull, 1);
    mbar_init(bars + 8 * L::kBDsFull, 8);  // one arrival per element-wise warp
    mbar_init(bars + 8 * L::kBDone, 1);
    mbar_init(bars + 8 * L::kBStaged, 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(sbase + L::kTmemSlotOff, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlotOff);

  if (warp < 8) {
    bwd_q_elementwise<D>(p, sbase, smem, tmem, tm_dq, abort_flag);
  } else if (warp == 8) {
    if (lane == 0) bwd_q_producer<D>(tm_q, tm_k, tm_v, tm_do, p, sbase, abort_flag);
  } else {
    if (lane == 0) bwd_q_mma<D>(p, sbase, tmem, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The backward in one launch: each CTA takes a dK/dV key tile or a dQ query
// tile, in the order bwd_tile gives.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
              const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  if (bwd_tile(p).kv)
    bwd_dkdv_block<D>(&tm_q, &tm_k, &tm_v, &tm_do, &tm_dk, &tm_dv, p, smem_raw);
  else
    bwd_dq_block<D>(&tm_q, &tm_k, &tm_v, &tm_do, &tm_dq, p, smem_raw);
}

}  // namespace fa
