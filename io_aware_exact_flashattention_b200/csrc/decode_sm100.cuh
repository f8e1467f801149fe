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
// Split kernel (persistent, one CTA per SM, items = (sequence, key/value
// head, chunk) taken round-robin).  The G = Hq/Hkv query heads of a group
// share every key/value byte, so the cache crosses HBM once.  Their scores
// and outputs are two small dense contractions per 128-key tile, run on
// tcgen05 with the roles swapped so the tile's keys fill the 128 MMA rows:
//   S^T[key, head] = K_tile[key, :] . q[head, :]     (M=128 keys, N=16 heads)
//   O^T[d, head]  += V_tile^T[d, key] . P[head, key]  (M=128 d, N=16 heads)
// with S^T and O^T in tensor memory and the G real heads padded to 16.
// Roles (192 threads):
//   warps 0-3  softmax + epilogue: thread = key row of S^T, then d row of O^T
//   warp  4    TMA producer: q of each item, then K and V tiles into a ring
//              (full tiles in one 128-row box, the last tile of a chunk in
//              32-row boxes so at most 31 rows past the chunk are fetched)
// A paged cache ([num_pages, Hkv, page_size, d] with a block table per
// sequence; paged KV management is named in "I/O-Aware Kernels", section
// "FlashAttention") changes the producer: chunks start on multiples of 128
// keys, so a tile covers whole pages (page_size <= 128) or lies inside one,
// and it is loaded as boxes of min(page_size, 128) rows (min(page_size, 32)
// for a chunk's last tile), each from the physical page the block table
// names.  At d = 128 a row is two 128-byte swizzle spans, and a tile laid out
// span by span ([half][128 rows]) would take two boxes per page; small pages
// make the per-box cost the limit.  So a paged tile at d = 128 is laid out
// [8-row group][half][8 rows] ("interleaved"): a page of P rows is then one
// contiguous 256*P-byte box of a 5-D view of the pool (64 columns, 8 rows,
// 2 halves, P/8 groups, planes), and the MMA descriptors step 1024 bytes
// between halves and 2048 between 8-row groups instead of 16 KB and 1024.
//   warp  5    MMA issuer
// The online softmax keeps a per-head reference max m that only moves when
// the max grows by more than 2^8; exp2 on scores times scale*log2(e).
#pragma once

#include <cuda.h>
#include "sm100.cuh"
#include "launch_dep.cuh"

namespace fa {

constexpr int kDecBN = 128;       // keys per tile (= TMEM lanes of S^T)
constexpr int kDecNPad = 16;      // head columns of S^T / O^T (G real, rest zero)
constexpr int kDecSubRows = 32;   // rows per box of a chunk's last tile
constexpr int kDecThreads = 192;
constexpr int kDecMaxPagesPerTile = kDecBN / 16;  // pages of the smallest size in a tile
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kDecRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct DecodeLayout {
  static constexpr int kStages = (D == 128) ? 6 : 8;  // ring of K or V tiles
  static constexpr int kTileBytes = kDecBN * D * 2;
  static constexpr int kBoxBytes = kDecBN * 128;       // one 64-wide column block of a tile
  static constexpr int kRingOff = 0;
  // D=64: a zero block that stands in for the upper 64 rows of V^T (M=128)
  static constexpr int kZeroOff = kRingOff + kStages * kTileBytes;
  static constexpr int kZeroBytes = (D == 64) ? kBoxBytes : 0;
  static constexpr int kQBytes = kDecNPad * D * 2;     // 16 query rows
  static constexpr int kQBoxBytes = kDecNPad * 128;
  static constexpr int kQOff = kZeroOff + kZeroBytes;  // 2 slots
  static constexpr int kPBytes = kDecNPad * kDecBN * 2;
  static constexpr int kPOff = kQOff + 2 * kQBytes;    // 2 buffers, K-major, 128B swizzle
  static constexpr int kRedMaxOff = kPOff + 2 * kPBytes;              // [2][4 warps][16] f32
  static constexpr int kRedSumOff = kRedMaxOff + 2 * 4 * kDecNPad * 4;
  static constexpr int kMetaOff = kRedSumOff + 2 * 4 * kDecNPad * 4;  // [2] x {lo, hi}
  static constexpr int kBarOff = kMetaOff + 2 * 16;
  static constexpr int kBKvFull = 0;
  static constexpr int kBKvEmpty = kStages;
  static constexpr int kBQFull = 2 * kStages;
  static constexpr int kBQEmpty = kBQFull + 2;
  static constexpr int kBSFull = kBQEmpty + 2;
  static constexpr int kBPFull = kBSFull + 2;
  static constexpr int kBODone = kBPFull + 2;
  static constexpr int kBOFree = kBODone + 1;
  static constexpr int kBRedMax = kBOFree + 2;
  static constexpr int kBRedSum = kBRedMax + 2;
  static constexpr int kBDone = kBRedSum + 2;
  static constexpr int kNumBars = kBDone + 1;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemSlotOff + 4;
  static constexpr int kBytes = kAbortOff + 4 + 1024;  // + slack for 1024-byte alignment
};

struct DecodeParams {
  float* o_part;
  float* lse_part;
  const int* seqlens;
  int B, Hq, Hkv, Lmax, n_splits, n_items;
  float scale, scale_log2;
  unsigned long long wait_limit_ns;
  // paged cache (block_table == nullptr: contiguous [B, Hkv, Lmax, d] cache)
  const int* block_table;  // [B, max_pages]
  int max_pages;
  int page_shift;          // log2(page_size)
  int rows_main;           // rows per box of a full tile: min(page_size, 128)
  int rows_tail;           // rows per box of a chunk's last tile: min(page_size, 32)
  int interleaved;         // tile layout [8-row group][half][8 rows] (paged, d = 128)
  int chunk_align;         // chunk sizes are rounded up to a multiple of this
};

// Chunk [lo, hi) of the keys of sequence b for split c (see fa.h).
__device__ __forceinline__ void decode_chunk(const DecodeParams& p, int b, int c, int& lo,
                                             int& hi) {
  int L = p.seqlens[b];
  L = max(0, min(L, p.Lmax));
  const int cs0 = (L + p.n_splits - 1) / p.n_splits;
  const int cs = (cs0 + p.chunk_align - 1) / p.chunk_align * p.chunk_align;
  lo = min(L, c * cs);
  hi = min(L, lo + cs);
}

__device__ __forceinline__ void decode_item(const DecodeParams& p, int item, int& b, int& g,
                                            int& c) {
  c = item % p.n_splits;
  const int bg = item / p.n_splits;
  g = bg % p.Hkv;
  b = bg / p.Hkv;
}

// ---------------------------------------------------------------------------
// TMA producer (one warp).  Lane 0 waits for buffers, accounts the bytes and
// issues the query loads and the contiguous-cache tile loads; for a paged
// cache a tile is many small boxes (two per page of 16 rows at d=128), and
// each lane issues one of them so their issue costs overlap.
// ---------------------------------------------------------------------------
template <int D, int G>
__device__ __forceinline__ void decode_producer(const CUtensorMap* tk, const CUtensorMap* tv,
                                                const CUtensorMap* tk32, const CUtensorMap* tv32,
                                                const CUtensorMap* tq, const DecodeParams& p,
                                                uint32_t sbase, volatile int* abort_flag,
                                                int lane) {
  using L = DecodeLayout<D>;
  const bool leader = (lane == 0);
  const bool paged = (p.block_table != nullptr);
  if (!paged && !leader) return;  // a contiguous cache needs lane 0 only
  const unsigned mask = paged ? 0xffffffffu : 1u;
  const uint32_t bars = sbase + L::kBarOff;
  if (leader) {
    tma_prefetch_desc(tk);
    tma_prefetch_desc(tv);
    tma_prefetch_desc(tk32);
    tma_prefetch_desc(tv32);
    tma_prefetch_desc(tq);
  }
  // lane 0 waits; every lane follows its verdict
  auto leader_wait = [&](uint32_t bar, uint32_t parity) -> bool {
    bool ok = true;
    if (leader) ok = mbar_wait(bar, parity, abort_flag, p.wait_limit_ns);
    return __shfl_sync(mask, ok ? 1 : 0, 0) != 0;
  };
  uint32_t ld = 0;  // K/V tile loads issued
  int it = 0;
  bool stop = false;
  for (int item = blockIdx.x; item < p.n_items && !stop; item += gridDim.x, ++it) {
    int b, g, c, lo, hi;
    decode_item(p, item, b, g, c);
    decode_chunk(p, b, c, lo, hi);
    const int slot = it & 1;
    if (!leader_wait(bars + 8 * (L::kBQEmpty + slot), (static_cast<uint32_t>(it >> 1) & 1u) ^ 1u))
      break;
    if (leader) {
      volatile int* meta = reinterpret_cast<volatile int*>(
          __cvta_shared_to_generic(sbase + L::kMetaOff + slot * 16));
      meta[0] = lo;
      meta[1] = hi;
      const uint32_t qbar = bars + 8 * (L::kBQFull + slot);
      mbar_arrive_expect_tx(qbar, L::kQBytes);
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_2d(sbase + L::kQOff + slot * L::kQBytes + kb * L::kQBoxBytes, tq, qbar, kb * 64,
                    b * p.Hq + g * G);
    }
    const int plane = b * p.Hkv + g;
    for (int t0 = lo; t0 < hi && !stop; t0 += kDecBN) {
      const int ntok = min(kDecBN, hi - t0);
      // Paged cache: the physical page of each page-sized (at most 128-row)
      // slice of the tile, read before the ring-slot waits so the loads'
      // latency overlaps them.
      int pg[kDecMaxPagesPerTile];
      if (paged) {
        const int* bt = p.block_table + static_cast<size_t>(b) * p.max_pages;
        const int slice = min(1 << p.page_shift, kDecBN);
#pragma unroll
        for (int j = 0; j < kDecMaxPagesPerTile; ++j)
          pg[j] = (j * slice < ntok) ? __ldg(bt + ((t0 + j * slice) >> p.page_shift)) : 0;
      }
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const int stage = static_cast<int>(ld % L::kStages);
        if (!leader_wait(bars + 8 * (L::kBKvEmpty + stage), ((ld / L::kStages) & 1u) ^ 1u)) {
          stop = true;
          break;
        }
        const uint32_t full = bars + 8 * (L::kBKvFull + stage);
        const uint32_t dst = sbase + L::kRingOff + stage * L::kTileBytes;
        if (paged) {
          // Boxes never straddle a page: t0 is a multiple of 128 and the box
          // height divides both 128 and the page size.
          const bool whole = (ntok == kDecBN);
          const int rows = whole ? p.rows_main : p.rows_tail;
          const int nsub = (ntok + rows - 1) / rows;
          const CUtensorMap* tm = whole ? (kv ? tv : tk) : (kv ? tv32 : tk32);
          if (leader) mbar_arrive_expect_tx(full, nsub * rows * 128 * (D / 64));
          __syncwarp(mask);
          if (p.interleaved) {
            // one box per slice, both column halves ([group][half][8 rows])
            if (lane < nsub) {
              const int slice = min(1 << p.page_shift, kDecBN);
              int page = pg[0];
#pragma unroll
              for (int j = 1; j < kDecMaxPagesPerTile; ++j)
                if (lane * rows >= j * slice) page = pg[j];
              const int prow = (t0 + lane * rows) & ((1 << p.page_shift) - 1);
              tma_load_5d(dst + lane * rows * 256, tm, full, 0, 0, 0, prow >> 3,
                          page * p.Hkv + g);
            }
          } else if (lane < nsub * (D / 64)) {  // at most 16 boxes per tile (page size 16)
            const int sub = lane / (D / 64), kb = lane % (D / 64);
            const int slice = min(1 << p.page_shift, kDecBN);
            int page = pg[0];
#pragma unroll
            for (int j = 1; j < kDecMaxPagesPerTile; ++j)
              if (sub * rows >= j * slice) page = pg[j];
            const int prow = (t0 + sub * rows) & ((1 << p.page_shift) - 1);
            tma_load_3d(dst + kb * L::kBoxBytes + sub * rows * 128, tm, full, kb * 64, prow,
                        page * p.Hkv + g);
          }
        } else if (leader) {
          if (ntok == kDecBN) {
            mbar_arrive_expect_tx(full, L::kTileBytes);
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_3d(dst + kb * L::kBoxBytes, kv ? tv : tk, full, kb * 64, t0, plane);
          } else {
            const int nsub = (ntok + kDecSubRows - 1) / kDecSubRows;
            mbar_arrive_expect_tx(full, nsub * kDecSubRows * 128 * (D / 64));
            for (int sub = 0; sub < nsub; ++sub)
#pragma unroll
              for (int kb = 0; kb < D / 64; ++kb)
                tma_load_3d(dst + kb * L::kBoxBytes + sub * kDecSubRows * 128, kv ? tv32 : tk32,
                            full, kb * 64, t0 + sub * kDecSubRows, plane);
          }
        }
        ++ld;
      }
    }
    if (stop) ++it;  // this item's q load was issued
  }
  // Drain: no copy may still be in flight when the CTA exits.
  if (leader) {
    const uint32_t S = static_cast<uint32_t>(L::kStages);
    for (uint32_t k = (ld > S ? ld - S : 0u); k < ld; ++k)
      mbar_wait(bars + 8 * (L::kBKvFull + k % S), (k / S) & 1u, nullptr, p.wait_limit_ns);
    for (int k = (it > 2 ? it - 2 : 0); k < it; ++k)
      mbar_wait(bars + 8 * (L::kBQFull + (k & 1)), static_cast<uint32_t>(k >> 1) & 1u, nullptr,
                p.wait_limit_ns);
  }
}

// ---------------------------------------------------------------------------
// MMA issuer (one thread)
// ---------------------------------------------------------------------------
template <int D, int G>
__device__ __forceinline__ void decode_mma(const DecodeParams& p, uint32_t sbase, uint32_t tmem,
                                           volatile int* abort_flag) {
  using L = DecodeLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  constexpr uint32_t kIdS = idesc_bf16_f32(kDecBN, kDecNPad, false, false);
  constexpr uint32_t kIdO = idesc_bf16_f32(128, kDecNPad, false, true);
  const uint32_t S = static_cast<uint32_t>(L::kStages);
  uint32_t jg = 0;  // tiles issued so far (global over items)
  int it = 0;

  // S^T for global tile t of the item whose q sits in slot `slot`
  auto issue_s = [&](uint32_t t, int slot) -> bool {
    const uint32_t idx = 2 * t;  // K of tile t is ring load 2t, V is 2t+1
    const uint32_t stage = idx % S;
    if (!mbar_wait(bars + 8 * (L::kBKvFull + stage), (idx / S) & 1u, abort_flag, p.wait_limit_ns))
      return false;
    tc_fence_after();
    const uint32_t ka = sbase + L::kRingOff + stage * L::kTileBytes;
    const uint32_t qa = sbase + L::kQOff + slot * L::kQBytes;
    // K tile: halves 16 KB apart and 8-row groups 1 KB apart, or (interleaved)
    // halves 1 KB apart and groups 2 KB apart
    const uint32_t k_half = p.interleaved ? 1024u : static_cast<uint32_t>(L::kBoxBytes);
    const uint32_t k_sbo = p.interleaved ? 2048u : 1024u;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t ko = (kk >> 2) * k_half + (kk & 3) * 32;
      const uint32_t qo = (kk >> 2) * L::kQBoxBytes + (kk & 3) * 32;
      mma_ss(tmem + (t & 1) * kDecNPad, sw128_desc(ka + ko, 16, k_sbo), sw128_desc(qa + qo, 16, 1024),
             kIdS, kk > 0 ? 1u : 0u);
    }
    mma_commit(bars + 8 * (L::kBSFull + (t & 1)));
    mma_commit(bars + 8 * (L::kBKvEmpty + stage));
    return true;
  };

  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++it) {
    const int slot = it & 1;
    if (!mbar_wait(bars + 8 * (L::kBQFull + slot), static_cast<uint32_t>(it >> 1) & 1u, abort_flag,
                   p.wait_limit_ns))
      goto done;
    {
      const volatile int* meta = reinterpret_cast<const volatile int*>(
          __cvta_shared_to_generic(sbase + L::kMetaOff + slot * 16));
      const int lo = meta[0], hi = meta[1];
      const uint32_t n_tiles = static_cast<uint32_t>((hi - lo + kDecBN - 1) / kDecBN);
      // the O^T buffer of this item is free once the epilogue two items back has read it
      if (!mbar_wait(bars + 8 * (L::kBOFree + (it & 1)), (static_cast<uint32_t>(it >> 1) & 1u) ^ 1u,
                     abort_flag, p.wait_limit_ns))
        goto done;
      if (n_tiles == 0) {
        mbar_arrive(bars + 8 * (L::kBQEmpty + slot));
        continue;
      }
      if (!issue_s(jg, slot)) goto done;
      const uint32_t to = tmem + 32 + (it & 1) * kDecNPad;
      for (uint32_t jt = 0; jt < n_tiles; ++jt) {
        const uint32_t t = jg + jt;
        if (jt + 1 < n_tiles) {
          if (!issue_s(t + 1, slot)) goto done;
        } else {
          mma_commit(bars + 8 * (L::kBQEmpty + slot));  // q no longer read once the last S is done
        }
        const uint32_t vidx = 2 * t + 1;
        const uint32_t vstage = vidx % S;
        if (!mbar_wait(bars + 8 * (L::kBKvFull + vstage), (vidx / S) & 1u, abort_flag,
                       p.wait_limit_ns))
          goto done;
        if (!mbar_wait(bars + 8 * (L::kBPFull + (t & 1)), (t >> 1) & 1u, abort_flag,
                       p.wait_limit_ns))
          goto done;
        tc_fence_after();
        const uint32_t va = sbase + L::kRingOff + vstage * L::kTileBytes;
        // second 64-row block of V^T: the tile's upper column block, or zeros
        // for D=64; 16 keys are 2 KB (4 KB interleaved) and 8-key groups 1 KB
        // (2 KB interleaved) apart
        const uint32_t lbo = (D == 128) ? (p.interleaved ? 1024u : static_cast<uint32_t>(L::kBoxBytes))
                                        : (sbase + L::kZeroOff) - va;
        const uint32_t v_sbo = p.interleaved ? 2048u : 1024u;
        const uint32_t pa = sbase + L::kPOff + (t & 1) * L::kPBytes;
#pragma unroll
        for (int kk = 0; kk < kDecBN / 16; ++kk) {
          mma_ss(to, sw128_desc(va + kk * 16 * (v_sbo / 8), lbo, v_sbo),
                 sw128_desc(pa + (kk >> 2) * (kDecNPad * 128) + (kk & 3) * 32, 16, 1024), kIdO,
                 (jt > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bars + 8 * L::kBODone);
        mma_commit(bars + 8 * (L::kBKvEmpty + vstage));
      }
      jg += n_tiles;
    }
  }
done:
  mma_commit(bars + 8 * L::kBDone);
  mbar_wait(bars + 8 * L::kBDone, 0u, nullptr, p.wait_limit_ns);
}

// ---------------------------------------------------------------------------
// Softmax + epilogue warpgroup (warps 0-3)
// ---------------------------------------------------------------------------
template <int D, int G>
__device__ __forceinline__ void decode_softmax(const DecodeParams& p, uint32_t sbase,
                                               uint32_t tmem, volatile int* abort_flag) {
  using L = DecodeLayout<D>;
  const uint32_t bars = sbase + L::kBarOff;
  const uint32_t S = static_cast<uint32_t>(L::kStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = threadIdx.x;  // key row of S^T / d row of O^T
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const float c = p.scale_log2;
  float* red_max = reinterpret_cast<float*>(__cvta_shared_to_generic(sbase + L::kRedMaxOff));
  float* red_sum = reinterpret_cast<float*>(__cvta_shared_to_generic(sbase + L::kRedSumOff));
  // element (head h, key t) of P in the K-major 128B-swizzled layout
  const uint32_t p_row_base = (t >> 6) * (kDecNPad * 128) + (t & 7) * 2;
  const uint32_t p_chunk = (t & 63) >> 3;

  bool dead = false;
  uint32_t jg = 0;
  int it = 0;
  for (int item = blockIdx.x; item < p.n_items && !dead; item += gridDim.x, ++it) {
    int b, g, ci;
    decode_item(p, item, b, g, ci);
    const int slot = it & 1;
    bool ok = mbar_wait(bars + 8 * (L::kBQFull + slot), static_cast<uint32_t>(it >> 1) & 1u,
                        abort_flag, p.wait_limit_ns);
    if (!__all_sync(0xffffffffu, ok)) {
      dead = true;
      break;
    }
    const volatile int* meta = reinterpret_cast<const volatile int*>(
        __cvta_shared_to_generic(sbase + L::kMetaOff + slot * 16));
    const int lo = meta[0], hi = meta[1];
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + 8 * (L::kBQEmpty + slot));
    const uint32_t n_tiles = static_cast<uint32_t>((hi - lo + kDecBN - 1) / kDecBN);
    const uint32_t to = tmem + lane_off + 32 + (it & 1) * kDecNPad;

    float m[G], l[G];  // m: reference max (raw score units), CTA-uniform; l: this row's share
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
    }

    for (uint32_t jt = 0; jt < n_tiles; ++jt) {
      const uint32_t tg = jg + jt;
      const int ntok = min(kDecBN, hi - (lo + static_cast<int>(jt) * kDecBN));
      const bool valid = t < ntok;
      ok = mbar_wait(bars + 8 * (L::kBSFull + (tg & 1)), (tg >> 1) & 1u, abort_flag,
                     p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        dead = true;
        break;
      }
      tc_fence_after();
      float s[G];
      {
        uint32_t r[16];
        tmem_ld16(tmem + lane_off + (tg & 1) * kDecNPad, r);
#pragma unroll
        for (int h = 0; h < G; ++h) s[h] = valid ? __uint_as_float(r[h]) : -INFINITY;
      }
      // tile max per head: warp, then across the four warps
      float* rm = red_max + (tg & 1) * (4 * kDecNPad);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = s[h];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
        if (lane == 0) rm[warp * kDecNPad + h] = v;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (L::kBRedMax + (tg & 1)));
      ok = mbar_wait(bars + 8 * (L::kBRedMax + (tg & 1)), (tg >> 1) & 1u, abort_flag,
                     p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        dead = true;
        break;
      }
      float alpha[G];
      bool rescale = false;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mt = fmaxf(fmaxf(rm[h], rm[kDecNPad + h]),
                               fmaxf(rm[2 * kDecNPad + h], rm[3 * kDecNPad + h]));
        alpha[h] = 1.f;
        if ((mt - m[h]) * c > kDecRescaleThreshold) {  // false while both are -inf (NaN)
          alpha[h] = ex2((m[h] - mt) * c);              // 0 when m was -inf
          l[h] *= alpha[h];
          m[h] = mt;
          rescale |= (jt > 0);
        }
      }
      // probabilities -> P (bf16, head rows, key columns)
      const uint32_t pa = sbase + L::kPOff + (tg & 1) * L::kPBytes + p_row_base;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mc = (m[h] == -INFINITY) ? 0.f : m[h] * c;
        const float pr = ex2(fmaf(s[h], c, -mc));  // <= 2^8; 0 for a masked key
        l[h] += pr;
        const __nv_bfloat16 pb = __float2bfloat16_rn(pr);
        const uint32_t addr = pa + h * 128 + ((p_chunk ^ static_cast<uint32_t>(h & 7)) << 4);
        asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr),
                     "h"(*reinterpret_cast<const unsigned short*>(&pb))
                     : "memory");
      }
      // last tile of a chunk: rows past the chunk must hold zeros for P.V
      if (ntok < kDecBN) {
        const uint32_t vidx = 2 * tg + 1;
        const uint32_t vstage = vidx % S;
        ok = mbar_wait(bars + 8 * (L::kBKvFull + vstage), (vidx / S) & 1u, abort_flag,
                       p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, ok)) {
          dead = true;
          break;
        }
        if (!valid) {
          const uint32_t tile = sbase + L::kRingOff + vstage * L::kTileBytes;
          const uint32_t row = p.interleaved ? tile + (t >> 3) * 2048 + (t & 7) * 128
                                             : tile + t * 128;
          const uint32_t half = p.interleaved ? 1024u : static_cast<uint32_t>(L::kBoxBytes);
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb)
#pragma unroll
            for (int q16 = 0; q16 < 8; ++q16)
              asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};"
                           ::"r"(row + kb * half + q16 * 16), "r"(0u)
                           : "memory");
        }
      }
      fence_proxy_async_smem();
      // the previous tile's P.V has finished: O^T is stable and may be rescaled
      if (tg > 0) {
        ok = mbar_wait(bars + 8 * L::kBODone, (tg - 1) & 1u, abort_flag, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, ok)) {
          dead = true;
          break;
        }
      }
      if (rescale) {
        tc_fence_after();
        uint32_t r[16];
        tmem_ld16(to, r);
#pragma unroll
        for (int h = 0; h < G; ++h) r[h] = __float_as_uint(__uint_as_float(r[h]) * alpha[h]);
        tmem_st16(to, r);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(bars + 8 * (L::kBPFull + (tg & 1)));
    }
    if (dead) break;

    // epilogue: sum l over the 128 rows, then O^T / l and the chunk LSE
    float* rs = red_sum + (it & 1) * (4 * kDecNPad);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float v = l[h];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) rs[warp * kDecNPad + h] = v;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + 8 * (L::kBRedSum + (it & 1)));
    ok = mbar_wait(bars + 8 * (L::kBRedSum + (it & 1)), static_cast<uint32_t>(it >> 1) & 1u,
                   abort_flag, p.wait_limit_ns);
    if (!__all_sync(0xffffffffu, ok)) {
      dead = true;
      break;
    }
    const size_t row0 =
        (static_cast<size_t>(b) * p.Hq + static_cast<size_t>(g) * G) * p.n_splits + ci;
    if (n_tiles == 0) {
      for (int idx = t; idx < G * D; idx += 128)
        p.o_part[(row0 + static_cast<size_t>(idx / D) * p.n_splits) * D + idx % D] = 0.f;
      if (t < G) p.lse_part[row0 + static_cast<size_t>(t) * p.n_splits] = -INFINITY;
    } else {
      ok = mbar_wait(bars + 8 * L::kBODone, (jg + n_tiles - 1) & 1u, abort_flag, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        dead = true;
        break;
      }
      tc_fence_after();
      uint32_t r[16];
      tmem_ld16(to, r);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float Lh = rs[h] + rs[kDecNPad + h] + rs[2 * kDecNPad + h] + rs[3 * kDecNPad + h];
        if (t < D)
          p.o_part[(row0 + static_cast<size_t>(h) * p.n_splits) * D + t] =
              __uint_as_float(r[h]) / Lh;
        if (t == h)
          p.lse_part[row0 + static_cast<size_t>(h) * p.n_splits] = m[h] * p.scale + logf(Lh);
      }
    }
    tc_fence_before();
    mbar_arrive(bars + 8 * (L::kBOFree + (it & 1)));
    jg += n_tiles;
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, 1)
fa_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_k32,
                       const __grid_constant__ CUtensorMap tm_v32,
                       const __grid_constant__ CUtensorMap tm_q, const DecodeParams p) {
  using L = DecodeLayout<D>;
  // the combine, launched next as a dependent, may be scheduled now; it
  // waits for this grid before reading the partials
  grid_dep_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbortOff);
  const uint32_t bars = sbase + L::kBarOff;
  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bars + 8 * (L::kBKvFull + s), 1);
      mbar_init(bars + 8 * (L::kBKvEmpty + s), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bars + 8 * (L::kBQFull + k), 1);
      mbar_init(bars + 8 * (L::kBQEmpty + k), 5);  // MMA + four softmax warps
      mbar_init(bars + 8 * (L::kBSFull + k), 1);
      mbar_init(bars + 8 * (L::kBPFull + k), 128);
      mbar_init(bars + 8 * (L::kBOFree + k), 128);
      mbar_init(bars + 8 * (L::kBRedMax + k), 4);
      mbar_init(bars + 8 * (L::kBRedSum + k), 4);
    }
    mbar_init(bars + 8 * L::kBODone, 1);
    mbar_init(bars + 8 * L::kBDone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp < 4) {
    // P rows of the padding heads, and the D=64 zero block, must read as zero
    uint4* z = reinterpret_cast<uint4*>(smem + L::kPOff);
    for (int i = threadIdx.x; i < 2 * L::kPBytes / 16; i += 128) z[i] = make_uint4(0, 0, 0, 0);
    uint4* z2 = reinterpret_cast<uint4*>(smem + L::kZeroOff);
    for (int i = threadIdx.x; i < L::kZeroBytes / 16; i += 128) z2[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 5) {
    tmem_alloc(sbase + L::kTmemSlotOff, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlotOff);

  if (warp < 4) {
    decode_softmax<D, G>(p, sbase, tmem, abort_flag);
  } else if (warp == 4) {
    decode_producer<D, G>(&tm_k, &tm_v, &tm_k32, &tm_v32, &tm_q, p, sbase, abort_flag, lane);
  } else {
    if (lane == 0) decode_mma<D, G>(p, sbase, tmem, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// Merge kernel: one warp per (sequence, query head); each lane owns D/32
// consecutive elements and walks the splits four at a time with independent
// loads.
template <int D>
__global__ void __launch_bounds__(128)
fa_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                  __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int rows, int n_splits) {
  constexpr float kLog2e = 1.44269504088896340736f;
  constexpr int EPL = D / 32;  // elements per lane: 4 (D=128) or 2 (D=64)
  // launched as a programmatic dependent: the kernel before it on the stream
  // (normally the split kernel writing the partials) has completed after this
  grid_dep_wait();
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* lp = lse_part + static_cast<size_t>(row) * n_splits;
  float M = -INFINITY;
  for (int c = lane; c < n_splits; c += 32) M = fmaxf(M, lp[c]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  __nv_bfloat16* orow = o + static_cast<size_t>(row) * D + lane * EPL;
  if (M == -INFINITY) {
#pragma unroll
    for (int e = 0; e < EPL; e += 2)
      *reinterpret_cast<__nv_bfloat162*>(orow + e) = __floats2bfloat162_rn(0.f, 0.f);
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
  int c = 0;
  for (; c + 4 <= n_splits; c += 4) {
    float w[4];
    float x[4][EPL];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      w[k] = ex2((lp[c + k] - lse_row) * kLog2e);  // 0 for an empty chunk (its partial is 0)
#pragma unroll
      for (int e = 0; e < EPL; ++e) x[k][e] = op[static_cast<size_t>(c + k) * D + e];
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w[k], x[k][e], acc[e]);
  }
  for (; c < n_splits; ++c) {
    const float w = ex2((lp[c] - lse_row) * kLog2e);
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, op[static_cast<size_t>(c) * D + e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < EPL; e += 2)
    *reinterpret_cast<__nv_bfloat162*>(orow + e) = __floats2bfloat162_rn(acc[e], acc[e + 1]);
  if (lane == 0) lse[row] = lse_row;
}

}  // namespace fa
