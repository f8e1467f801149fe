// backward_sm100.cuh -- exact-attention backward by recomputation for sm_100a.
//
// The pages state that the backward pass recomputes the attention matrix
// instead of storing it ("Tracing Tiled QKV Data Movement in FlashAttention's
// Memory Hierarchy", closing takeaways).  With P = exp(scale*q.k - LSE) from
// the forward's LSE, D_i = dO_i . O_i and dS = P * (dO.v - D):
//   dV_j = sum_i P_ij dO_i,  dK_j = scale * sum_i dS_ij q_i,  dQ_i = scale * sum_j dS_ij k_j.
//
// One CTA per (batch, key/value head, 128-key tile j): K_j and V_j stay in
// shared memory and dK_j, dV_j accumulate in tensor memory while the query
// tiles of every query head of the group stream past (key-stationary loop, so
// dK and dV are written once; dQ rows collect contributions from every key
// tile and are added into an fp32 workspace by bulk tensor reductions).  Per
// query tile, all on tcgen05 with fp32 accumulators in TMEM:
//   S^T  = K_j Q_i^T      (M=128 keys, N=128 queries; SS)
//   dP^T = V_j dO_i^T     (M=128 keys, N=128 queries; SS)
//   dV  += P^T dO_i       (A = P^T in TMEM, B = dO_i MN-major; TS)
//   dK  += dS^T Q_i       (A = dS^T in TMEM, B = Q_i MN-major; TS)
//   dQ_i = dS K_j         (A = dS from shared memory MN-major, B = K_j MN-major; SS)
// Roles (320 threads):
//   warps 0-7  two warpgroups, each half of every tile's queries: thread =
//              key row for P and dS (from S^T, dP^T, LSE and D); thread =
//              query row for the dQ partial (half the d-columns each) into
//              the workspace; dK, dV out
//   warp  8    TMA producer: K_j, V_j once, then Q_i and dO_i (two stages)
//   warp  9    MMA issuer; allocates tensor memory
// Tensor memory columns: dV [0,128), dK [128,256), S^T / P [256,384),
// dP^T / dS / dQ partial [384,512).  The next tile's S^T is issued as soon as
// dQ_i is, so it runs while dQ_i is read out; its dP^T waits for the read-out.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include "sm100.cuh"

namespace fa {

constexpr int kBwdThreads = 320;
constexpr int kBwdBM = 128;  // keys per CTA (TMEM lanes)
constexpr int kBwdBN = 128;  // queries per tile

template <int D>
struct BwdLayout {
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kBoxBytes = 128 * 128;  // 128 rows x 64 bf16, 128B swizzled
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kQOff = 2 * kTileBytes;  // stage s: Q at kQOff + 2*s*tile, dO after it
  static constexpr int kDsOff = 6 * kTileBytes;  // dS^T: 128 keys x 128 queries bf16 (2 boxes)
  static constexpr int kLseOff = kDsOff + 128 * 128 * 2;  // [128] LSE*log2(e), [128] D
  static constexpr int kBarOff = kLseOff + 2 * 128 * 4;
  static constexpr int kBKv = 0;
  static constexpr int kBQFull = 1;    // [2]
  static constexpr int kBQEmpty = 3;   // [2]
  static constexpr int kBSFull = 5;
  static constexpr int kBDpFull = 6;
  static constexpr int kBPFull = 7;    // 8 arrivals (one per element-wise warp)
  static constexpr int kBDsFull = 8;   // 8 arrivals
  static constexpr int kBDqFull = 9;
  static constexpr int kBSFree = 10;   // 8 arrivals: dQ partial read out of the dP columns
  static constexpr int kBDone = 11;
  static constexpr int kNumBars = 12;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemSlotOff + 4;
  static constexpr int kBytes = kAbortOff + 4 + 1024;  // + slack for 1024-byte alignment
};
static_assert(BwdLayout<128>::kBytes <= 232448, "backward shared memory over the limit");

struct BwdParams {
  float* dq_acc;       // [B, Hq, Sq, d] fp32, zeroed; receives scale * dS K
  const float* lse;    // [B, Hq, Sq] natural log
  const float* dsum;   // [B, Hq, Sq]: D = dO . O
  __nv_bfloat16* dk;   // [B, Hkv, Skv, d]
  __nv_bfloat16* dv;
  int B, Hq, Hkv, Sq, Skv, group, causal;
  int n_kv_tiles, n_q_tiles;
  int heads_per_group;  // CTA order: groups of this many (b, kv-head) pairs (see bwd_cta)
  float scale, scale_log2;
  unsigned long long wait_limit_ns;
};

// First query tile that sees any key of key tile j (causal: key k is visible
// to query q iff k <= q + Skv - Sq).
__device__ __forceinline__ int bwd_first_q_tile(const BwdParams& p, int j) {
  if (!p.causal) return 0;
  const long long need = static_cast<long long>(j) * kBwdBM - (p.Skv - p.Sq);  // q >= need
  if (need <= 0) return 0;
  return static_cast<int>(need / kBwdBN);
}

__device__ __forceinline__ void bwd_cta(const BwdParams& p, int& b, int& g, int& j) {
  // CTAs go out in groups of p.heads_per_group (batch, key/value head)
  // pairs; within a group key tile by key tile, heavy tiles first (under a
  // causal mask key tile 0 sees every query tile), so the launch order stays
  // longest-first and the tail is short.  The CTAs resident at a time then
  // cover about two groups, whose Q, dO and fp32 dQ rows stay in L2 while all
  // their key tiles stream them; ordered key tile by key tile over all heads,
  // the resident CTAs touch every head's Q, dO and dQ at once, more than L2
  // holds.
  const int per_group = p.heads_per_group * p.n_kv_tiles;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int r = static_cast<int>(blockIdx.x) % per_group;
  const int units = p.B * p.Hkv;
  const int in_group = min(p.heads_per_group, units - grp * p.heads_per_group);
  j = r / in_group;
  const int bg = grp * p.heads_per_group + r % in_group;
  b = bg / p.Hkv;
  g = bg % p.Hkv;
}

// Element-wise add of a shared-memory box into global memory (bulk reduction
// in L2), tracked by the issuing thread's bulk-async group.
__device__ __forceinline__ void tma_reduce_add_3d(const void* tmap, uint32_t src, int c0, int c1,
                                                  int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(tmap)), "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every committed bulk operation of this thread has completed.
__device__ __forceinline__ void bulk_wait_group0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Wait until every committed bulk operation of this thread has finished
// reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// D = rowsum(dO * O) for every query row (one warp per row); the row's fp32
// dq accumulator is zeroed on the way.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dsum_kernel(const __nv_bfloat16* __restrict__ o,
                                                          const __nv_bfloat16* __restrict__ d_o,
                                                          float* __restrict__ dsum,
                                                          float* __restrict__ dq_acc,
                                                          long long rows) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
#pragma unroll
  for (int c = lane * 4; c < D; c += 128)
    *reinterpret_cast<float4*>(dq_acc + row * D + c) = make_float4(0.f, 0.f, 0.f, 0.f);
  float acc = 0.f;
#pragma unroll
  for (int c = lane * 2; c < D; c += 64) {
    const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(o + row * D + c);
    const __nv_bfloat162 y = *reinterpret_cast<const __nv_bfloat162*>(d_o + row * D + c);
    acc = fmaf(__bfloat162float(x.x), __bfloat162float(y.x), acc);
    acc = fmaf(__bfloat162float(x.y), __bfloat162float(y.y), acc);
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) dsum[row] = acc;
}

// dq (bf16) from the fp32 workspace.
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float* __restrict__ acc,
                                                        __nv_bfloat16* __restrict__ dq,
                                                        long long n) {
  const long long i = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) * 4;
  if (i >= n) return;
  const float4 v = *reinterpret_cast<const float4*>(acc + i);
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 c = __floats2bfloat162_rn(v.z, v.w);
  uint2 w;
  w.x = *reinterpret_cast<uint32_t*>(&a);
  w.y = *reinterpret_cast<uint32_t*>(&c);
  *reinterpret_cast<uint2*>(dq + i) = w;
}

// ---------------------------------------------------------------------------
// Producer (one thread)
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void bwd_producer(const CUtensorMap* tq, const CUtensorMap* tk,
                                             const CUtensorMap* tv, const CUtensorMap* tdo,
                                             const BwdParams& p, uint32_t sbase,
                                             volatile int* abort_flag) {
  using L = BwdLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  int b, g, j;
  bwd_cta(p, b, g, j);
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
      mbar_arrive_expect_tx(full, 2 * L::kTileBytes);
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb) {
        tma_load_3d(qa + kb * L::kBoxBytes, tq, full, kb * 64, i * kBwdBN, plane);
        tma_load_3d(qa + L::kTileBytes + kb * L::kBoxBytes, tdo, full, kb * 64, i * kBwdBN, plane);
      }
    }
  }
drain:
  mbar_wait(bkv, 0u, nullptr, p.wait_limit_ns);
  for (uint32_t k = (n > 2 ? n - 2 : 0u); k < n; ++k)
    mbar_wait(bars + 8 * (L::kBQFull + (k & 1u)), (k >> 1) & 1u, nullptr, p.wait_limit_ns);
}

// ---------------------------------------------------------------------------
// MMA issuer (one thread)
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void bwd_mma(const BwdParams& p, uint32_t sbase, uint32_t tmem,
                                        volatile int* abort_flag) {
  using L = BwdLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  constexpr uint32_t kIdS = idesc_bf16_f32(kBwdBM, kBwdBN, false);         // K-major A and B
  constexpr uint32_t kIdAcc = idesc_bf16_f32(kBwdBM, D, true);             // A TMEM, B MN-major
  constexpr uint32_t kIdDq = idesc_bf16_f32(kBwdBN, D, true, true);        // A, B MN-major
  const uint32_t t_dv = tmem, t_dk = tmem + 128, t_s = tmem + 256, t_dp = tmem + 384;
  const uint32_t ka = sbase + L::kKOff, va = sbase + L::kVOff, dsa = sbase + L::kDsOff;
  int b, g, j;
  bwd_cta(p, b, g, j);
  const int i0 = bwd_first_q_tile(p, j);
  const int per_head = p.n_q_tiles - i0;
  const uint32_t total = per_head > 0 ? static_cast<uint32_t>(per_head * p.group) : 0u;
  // TMEM column of the packed bf16 pairs for queries 16*kk .. 16*kk+15: each
  // warpgroup packs its 64 queries at the start of its own 64 columns
  auto packed_col = [](int kk) -> uint32_t {
    constexpr int kSteps = kBwdBN / 16;
    return static_cast<uint32_t>(kk * 8 + (kk >= kSteps / 2 ? 32 : 0));
  };
  auto wait = [&](int bar, uint32_t parity) -> bool {
    if (!mbar_wait(bars + 8 * bar, parity, abort_flag, p.wait_limit_ns)) return false;
    tc_fence_after();
    return true;
  };
  // A, B both K-major (rows of 64 elements, 128B swizzle), K = D in steps of 16
  auto gemm_kmajor = [&](uint32_t d_tmem, uint32_t a, uint32_t bb) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t o = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
      mma_ss(d_tmem, sw128_desc(a + o, 16, 1024), sw128_desc(bb + o, 16, 1024), kIdS,
             kk > 0 ? 1u : 0u);
    }
  };
  if (total > 0) {
    if (!wait(L::kBKv, 0u) || !wait(L::kBQFull + 0, 0u)) goto done;
    gemm_kmajor(t_s, ka, sbase + L::kQOff);                        // S^T = K Q^T
    mma_commit(bars + 8 * L::kBSFull);
    gemm_kmajor(t_dp, va, sbase + L::kQOff + L::kTileBytes);       // dP^T = V dO^T
    mma_commit(bars + 8 * L::kBDpFull);
  }
  for (uint32_t n = 0; n < total; ++n) {
    const uint32_t s = n & 1u, ph = n & 1u;
    const uint32_t qa = sbase + L::kQOff + 2 * s * L::kTileBytes;
    const uint32_t doa = qa + L::kTileBytes;
    if (!wait(L::kBPFull, ph)) goto done;
#pragma unroll
    for (int kk = 0; kk < kBwdBN / 16; ++kk)       // dV += P^T dO
      mma_ts(t_dv, t_s + packed_col(kk), sw128_desc(doa + kk * 16 * 128, L::kBoxBytes, 1024),
             kIdAcc, (n > 0 || kk > 0) ? 1u : 0u);
    if (!wait(L::kBDsFull, ph)) goto done;
#pragma unroll
    for (int kk = 0; kk < kBwdBN / 16; ++kk)       // dK += dS^T Q
      mma_ts(t_dk, t_dp + packed_col(kk), sw128_desc(qa + kk * 16 * 128, L::kBoxBytes, 1024),
             kIdAcc, (n > 0 || kk > 0) ? 1u : 0u);
    mma_commit(bars + 8 * (L::kBQEmpty + s));     // Q_i, dO_i read by everything issued so far
    // dQ_i = dS K (K = keys) into the dP^T / dS columns (dS already read by dK)
#pragma unroll
    for (int kk = 0; kk < kBwdBM / 16; ++kk)
      mma_ss(t_dp, sw128_desc(dsa + kk * 16 * 128, L::kBoxBytes, 1024),
             sw128_desc(ka + kk * 16 * 128, L::kBoxBytes, 1024), kIdDq, kk > 0 ? 1u : 0u);
    mma_commit(bars + 8 * L::kBDqFull);
    if (n + 1 < total) {
      // next tile's scores while dQ_i is read out (P_i was read by dV already)
      const uint32_t s1 = (n + 1) & 1u;
      const uint32_t qa1 = sbase + L::kQOff + 2 * s1 * L::kTileBytes;
      if (!wait(L::kBQFull + s1, ((n + 1) >> 1) & 1u)) goto done;
      gemm_kmajor(t_s, ka, qa1);
      mma_commit(bars + 8 * L::kBSFull);
      // dP^T of the next tile once dQ_i has left the dP^T columns
      if (!wait(L::kBSFree, ph)) goto done;
      gemm_kmajor(t_dp, va, qa1 + L::kTileBytes);
      mma_commit(bars + 8 * L::kBDpFull);
    }
  }
done:
  mma_commit(bars + 8 * L::kBDone);
  mbar_wait(bars + 8 * L::kBDone, 0u, nullptr, p.wait_limit_ns);
}

// ---------------------------------------------------------------------------
// Element-wise warpgroups (warps 0-7).  Warpgroup hf takes queries
// [64*hf, 64*hf + 64) of each tile for P and dS (thread t = key row t, the
// TMEM lane) and d-columns [hf*D/2, (hf+1)*D/2) for the dQ partial (thread t
// = query row t) and for dK, dV; the two halves run side by side.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void bwd_elementwise(const BwdParams& p, const CUtensorMap* tm_dq,
                                                uint32_t sbase, uint8_t* smem, uint32_t tmem,
                                                volatile int* abort_flag) {
  using L = BwdLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  const int t = threadIdx.x & 127;
  const int hf = threadIdx.x >> 7;  // warpgroup: query half / column half
  const int warp = (threadIdx.x >> 5) & 3;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t t_dv = tmem + lane_off, t_dk = tmem + lane_off + 128;
  const uint32_t t_s = tmem + lane_off + 256, t_dp = tmem + lane_off + 384;
  constexpr int kQH = kBwdBN / 2;   // queries per warpgroup
  constexpr int kDH = D / 2;        // d-columns per warpgroup
  float* lse_s = reinterpret_cast<float*>(smem + L::kLseOff);
  float* d_s = lse_s + 128;
  uint8_t* ds_smem = smem + L::kDsOff;
  int b, g, j;
  bwd_cta(p, b, g, j);
  const int key = j * kBwdBM + t;
  const int off = p.Skv - p.Sq;
  const int i0 = bwd_first_q_tile(p, j);
  uint32_t n = 0;
  // LSE (in log2 units) and D of this thread's query for a tile: loaded one
  // tile ahead, so the load latency hides behind the previous tile's work.
  auto load_ld = [&](int hh_, int i_, float& lse_v, float& d_v) {
    const int c = hf * kQH + t;
    const int q = i_ * kBwdBN + c;
    const size_t rb = (static_cast<size_t>(b) * p.Hq + g * p.group + hh_) * p.Sq;
    lse_v = (t < kQH && q < p.Sq) ? p.lse[rb + q] * 1.4426950408889634f : INFINITY;
    d_v = (t < kQH && q < p.Sq) ? p.dsum[rb + q] : 0.f;
  };
  float lse_next = INFINITY, d_next = 0.f;
  if (i0 < p.n_q_tiles) load_ld(0, i0, lse_next, d_next);
  // After a failed wait a warp skips the remaining work but still takes every
  // named barrier, so the other warps of its warpgroup can never block there.
  bool ok = true;
  for (int hh = 0; hh < p.group; ++hh) {
    const int h = g * p.group + hh;
    for (int i = i0; i < p.n_q_tiles; ++i, ++n) {
      const uint32_t ph = n & 1u;
      const int q0 = i * kBwdBN;
      // this warpgroup's 64 queries: LSE and D into shared memory
      named_barrier(1 + hf, 128);
      if (t < kQH) {
        lse_s[hf * kQH + t] = lse_next;
        d_s[hf * kQH + t] = d_next;
      }
      named_barrier(1 + hf, 128);
      {  // next tile's values (same head, or the next head's first tile)
        const bool more_i = (i + 1 < p.n_q_tiles);
        if (more_i) load_ld(hh, i + 1, lse_next, d_next);
        else if (hh + 1 < p.group) load_ld(hh + 1, i0, lse_next, d_next);
      }

      if (!ok) continue;
      // P^T for this key and the warpgroup's queries: p = 2^(s*scale*log2e - LSE*log2e)
      ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * L::kBSFull, ph, abort_flag, p.wait_limit_ns));
      if (!ok) continue;
      tc_fence_after();
      uint32_t pk[kQH / 2];
      {
        uint32_t ra[64];
        tmem_ld64_nowait(t_s + hf * kQH, ra);
        tmem_ld_wait_hold(ra);
        const int lim = key - off;  // first query that sees this key
#pragma unroll
        for (int c2 = 0; c2 < kQH / 2; ++c2) {
          float pr[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = hf * kQH + 2 * c2 + e;
            const bool vis = (key < p.Skv) && (!p.causal || q0 + c >= lim);
            const float x = fmaf(__uint_as_float(ra[2 * c2 + e]), p.scale_log2, -lse_s[c]);
            pr[e] = vis ? ex2(x) : 0.f;
          }
          pk[c2] = pack_bf16x2(pr[0], pr[1]);
        }
      }
      // packed pairs of queries, inside this warpgroup's own (already read)
      // score columns: the other warpgroup's scores are never overwritten
      tmem_st32(t_s + hf * kQH, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bars + 8 * L::kBPFull);

      // dS = P * (dP - D): to TMEM (A of dK += dS^T Q) and to shared memory
      // (A of dQ = dS K, MN-major: rows = keys, 64-query boxes, 128B swizzle)
      ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * L::kBDpFull, ph, abort_flag, p.wait_limit_ns));
      if (!ok) continue;
      tc_fence_after();
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {  // 32 queries per pass
        uint32_t dp[32];
        tmem_ld32(t_dp + hf * kQH + hq * 32, dp);
        uint32_t dsk[16];
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          const int cl = hq * 32 + 2 * e2;  // local query index in the half
          const __nv_bfloat162 pb = *reinterpret_cast<const __nv_bfloat162*>(&pk[cl >> 1]);
          const int c = hf * kQH + cl;
          const float d0 = __bfloat162float(pb.x) * (__uint_as_float(dp[2 * e2]) - d_s[c]);
          const float d1 = __bfloat162float(pb.y) * (__uint_as_float(dp[2 * e2 + 1]) - d_s[c + 1]);
          dsk[e2] = pack_bf16x2(d0, d1);
        }
        tmem_st16(t_dp + hf * kQH + hq * 16, dsk);  // own columns, already read
        // queries hf*64 + hq*32 .. +31: box hf, 16-byte chunks hq*4 .. +3 of row t
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int chunk = hq * 4 + k4;
          uint4* dst = reinterpret_cast<uint4*>(ds_smem + hf * L::kBoxBytes + t * 128 +
                                                ((chunk ^ (t & 7)) * 16));
          *dst = make_uint4(dsk[4 * k4], dsk[4 * k4 + 1], dsk[4 * k4 + 2], dsk[4 * k4 + 3]);
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bars + 8 * L::kBDsFull);

      // dQ partial (thread = query row q0 + t, this warpgroup's d-columns),
      // scaled, staged 32 columns at a time in this warpgroup's half of the
      // dS buffer (free: the dQ MMA that read dS is complete) and added into
      // the fp32 workspace by one bulk tensor reduction per 128 x 32 box.
      ok = __all_sync(0xffffffffu, mbar_wait(bars + 8 * L::kBDqFull, ph, abort_flag, p.wait_limit_ns));
      if (!ok) continue;
      tc_fence_after();
      {
        uint8_t* stage = ds_smem + hf * L::kBoxBytes;  // 128 rows x 128 B, 128B swizzle
        const uint32_t stage_s = sbase + L::kDsOff + hf * L::kBoxBytes;
#pragma unroll
        for (int c4 = 0; c4 < kDH / 32; ++c4) {
          uint32_t r[32];
          tmem_ld32(t_dp + hf * kDH + c4 * 32, r);
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            float4 v4 = make_float4(__uint_as_float(r[4 * k4]) * p.scale,
                                    __uint_as_float(r[4 * k4 + 1]) * p.scale,
                                    __uint_as_float(r[4 * k4 + 2]) * p.scale,
                                    __uint_as_float(r[4 * k4 + 3]) * p.scale);
            *reinterpret_cast<float4*>(stage + t * 128 + ((k4 ^ (t & 7)) * 16)) = v4;
          }
          fence_proxy_async_smem();
          named_barrier(1 + hf, 128);
          if (t == 0) {
            tma_reduce_add_3d(tm_dq, stage_s, hf * kDH + c4 * 32, q0, static_cast<int>(
                static_cast<size_t>(b) * p.Hq + h));
            bulk_commit_group();
            bulk_wait_group_read0();  // the box has been read: the buffer is free again
          }
          named_barrier(1 + hf, 128);
        }
      }
      tc_fence_before();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bars + 8 * L::kBSFree);
    }
  }
  if (t == 0) bulk_wait_group0();  // this thread's reductions have landed
  if (!ok) return;

  // dK = scale * (dS^T Q summed), dV = P^T dO summed: thread t = key row,
  // this warpgroup's d-columns
  if (!__all_sync(0xffffffffu, mbar_wait(bars + 8 * L::kBDone, 0u, abort_flag, p.wait_limit_ns)))
    return;
  tc_fence_after();
  const bool any = (i0 < p.n_q_tiles);
  // tcgen05.ld is warp-collective: every thread loads, only rows of real keys
  // are stored.
  const bool real = key < p.Skv;
  const size_t krow = (static_cast<size_t>(b) * p.Hkv + g) * p.Skv + (real ? key : 0);
#pragma unroll
  for (int which = 0; which < 2; ++which) {
    __nv_bfloat16* out = (which == 0 ? p.dv : p.dk) + krow * D + hf * kDH;
    const float mul = (which == 0) ? 1.f : p.scale;
#pragma unroll
    for (int c4 = 0; c4 < kDH / 32; ++c4) {
      uint32_t r[32];
      tmem_ld32((which == 0 ? t_dv : t_dk) + hf * kDH + c4 * 32, r);
      if (real) {
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          uint4 w;
          const float* f = reinterpret_cast<const float*>(r) + v4 * 8;
          w.x = pack_bf16x2(any ? f[0] * mul : 0.f, any ? f[1] * mul : 0.f);
          w.y = pack_bf16x2(any ? f[2] * mul : 0.f, any ? f[3] * mul : 0.f);
          w.z = pack_bf16x2(any ? f[4] * mul : 0.f, any ? f[5] * mul : 0.f);
          w.w = pack_bf16x2(any ? f[6] * mul : 0.f, any ? f[7] * mul : 0.f);
          reinterpret_cast<uint4*>(out + c4 * 32)[v4] = w;
        }
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
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
    mbar_init(bars + 8 * L::kBDqFull, 1);
    mbar_init(bars + 8 * L::kBSFree, 8);
    mbar_init(bars + 8 * L::kBDone, 1);
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
    bwd_elementwise<D>(p, &tm_dq, sbase, smem, tmem, abort_flag);
  } else if (warp == 8) {
    if (lane == 0) bwd_producer<D>(&tm_q, &tm_k, &tm_v, &tm_do, p, sbase, abort_flag);
  } else {
    if (lane == 0) bwd_mma<D>(p, sbase, tmem, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
