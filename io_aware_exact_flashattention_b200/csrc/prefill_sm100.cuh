// prefill_sm100.cuh -- fused exact-attention forward for sm_100a.
//
// A work item is two 128-row query tiles of one (batch, query head); the
// key/value tiles of that head's key/value head stream past them, so the
// score matrix never leaves the SM ("I/O-Aware Kernels", section "FlashAttention":
// query blocks stay resident while K and V blocks stream through; "Tracing
// Tiled QKV Data Movement in FlashAttention's Memory Hierarchy", section 2,
// tiling plus online softmax).  The loop order is query-stationary: the
// output tile is accumulated on chip and written to HBM once.  The kernel is
// persistent: one CTA per SM walks the items longest first (under a causal
// mask the last query tiles have the most keys), in a snake order over the
// CTAs, so the next item's query load and first score MMAs overlap the
// current item's last tiles and epilogue.
//
// Roles (384 threads, three warpgroups):
//   warps 0-3  softmax warpgroup for query tile 0 (thread = row = TMEM lane)
//   warps 4-7  softmax warpgroup for query tile 1
//   warp  8    TMA producer: Q tiles once, then K_j, V_j into a smem ring
//   warp  9    MMA issuer: S_w = Q_w K_j^T and O_w += P_w V_j on tcgen05
//   warps 10-11 idle
// Registers are moved from the third warpgroup to the softmax warpgroups
// (setmaxnreg): 216 + 216 + 72 per SM sub-partition = 3 x 168 at launch.
// Both shares are the smallest that compile without spills (the MMA issuer
// adds descriptor offsets inside its instruction sequences to fit in 72).
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [0,128)   S_0 (fp32 scores); P_0 (bf16) overwrites its first 64 columns
//   [128,256) S_1 / P_1
//   [256, 256+D) O_0 accumulator, then O_1
// Online softmax ("FlashAttention & IO-aware attention", section "Direct
// answer"): each row keeps a running max m and sum l; when the max grows the
// accumulated l and O are multiplied by e^(m - m_new).  Two sums are kept:
// l of the fp32 weights for the LSE, and lq of the bf16-rounded weights that
// P.V multiplies, by which O is divided.  Here the reference max
// only moves when it grows by more than 2^24 in the exponent, so the rescale
// of O (a round trip of O through registers) is rare even for logits spread
// over tens of binades; the result is unchanged because the final O / l and
// LSE use the same reference max.  p <= 2^24 loses nothing: bf16 P and the
// fp32 l and O round relative to magnitude and have ~2^100 of headroom.
// Exponentials are 2^x on scores pre-multiplied by scale*log2(e).
//
// 8-bit inputs (kF8; FlashAttention-3's FP8 variant, which "FlashAttention &
// IO-aware attention", section "Deep dive", names): Q, K and V are E4M3 codes
// with one fp32 dequantisation factor per (batch, key/value head) each.  Both
// products run as tcgen05 kind::f8f6f4 MMAs (K = 32 per instruction): S from
// Q and K in shared memory, O from P in tensor memory (E4M3, four per 32-bit
// column, 32 columns per tile) and V in shared memory (MN-major).  A d = 128
// tile of E4M3 is 128-byte rows, the shared-memory geometry of a bf16 d = 64
// tile, so it takes that layout (16 KB tiles, 8 ring stages).  The factors of
// Q and K fold into the exponent constant and that of V into the epilogue's
// 1/l.  P is quantised as p * 2^6 with the reference max allowed to lag the
// row max by at most 2^2, so every quantised value lies in (0, 256], inside
// E4M3's range (448), and the row's largest one is >= 64, which keeps the
// absolute rounding of E4M3 subnormals (<= 2^-10) below 2^-16 of l.  The
// power of two cancels in O / l; LSE subtracts it.
#pragma once

#include <climits>
#include <type_traits>
#include <cuda.h>
#include "sm100.cuh"

namespace fa {

constexpr int kBM = 128;       // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;       // keys per key/value tile
constexpr int kPrefillThreads = 384;
constexpr int kPrefillLaunchRegs = 168;   // 65536 / 384, rounded down to a multiple of 8
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
static_assert(2 * kSoftmaxRegs + kControlRegs <= 3 * kPrefillLaunchRegs,
              "register split exceeds the launch budget");
constexpr int kSwzBytes = 128 * 128;  // one 128-row x 64-element bf16 box, 128B swizzled
constexpr float kRescaleThreshold = 24.0f;  // log2 units
constexpr float kRescaleThresholdF8 = 2.0f;  // log2 units, 8-bit P
constexpr float kPOffsetF8 = 6.0f;           // 8-bit P is stored as p * 2^6

// Of every 8 pairs of scores, this many use the polynomial.  Off: on B200,
// with the other choices in this kernel, every share tried (1 to 4 of 8)
// took more cycles than the MUFU alone (2-7 %); the polynomial stays as a
// tested option (fa_debug_exp2_poly checks it against the MUFU).
constexpr int kPolyPairsPer8 = 0;
// The same share for 8-bit P.  There the E4M3 products take half the tensor
// time, so the softmax's exponentials rather than the MMA set the key tile
// period: on B200, 2 of 8 pairs on the polynomial took 2.6 % (S = 2048) and
// 4.4 % (S = 8192) less time than none, 3 of 8 about the same, 4 of 8 more.
constexpr int kPolyPairsPer8F8 = 2;

// D[tmem] (+)= A[smem] * B[smem], kind::f8f6f4 (A and B both E4M3 here).
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// mma_ss_f8 / mma_ts_f8 with descriptors as a base plus an offset in 16-byte
// units added inside the instruction sequence (see mma_ss_off).
template <uint32_t kAOff, uint32_t kBOff>
__device__ __forceinline__ void mma_ss_f8_off(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 a, b;\n\t"
      "add.s64 a, %1, %5;\n\t"
      "add.s64 b, %2, %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a, b, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "n"(kAOff),
        "n"(kBOff)
      : "memory");
}
template <uint32_t kBOff>
__device__ __forceinline__ void mma_ts_f8_off(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 b;\n\t"
      "add.s64 b, %2, %5;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], b, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "n"(kBOff)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], kind::f8f6f4; A is read from tensor memory.
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f8f6f4: D fp32 (bits 4-5 = 1), A and B E4M3
// (format 0 in bits 7-9 and 10-12), B major at bit 16 (1 = MN-major), N >> 3
// at bits 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Four fp32 values -> four E4M3 codes (nearest even, saturating), a in the
// lowest byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r) : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

struct PrefillParams {
  __nv_bfloat16* o;
  float* lse;
  int B, Hq, Hkv, Sq, Skv, group;
  int causal;
  // The launch computes query tiles [q_tile0, q_tile_end) of every (b, h)
  // (all tiles for a whole forward; a range for blockwise use).  Output row
  // `row` of head (b, h) is o[((b*Hq + h) * o_rows + row - o_row0) * D] and
  // lse[(b*Hq + h) * lse_rows + row - lse_row0].
  int q_tile0, q_tile_end;
  int o_rows, o_row0, lse_rows, lse_row0;
  int n_qpairs;    // ceil((q_tile_end - q_tile0) / 2)
  int n_items;     // n_qpairs * B * Hq
  int n_kv_tiles;  // ceil(Skv / 128)
  float scale;     // natural units
  float scale_log2;
  unsigned long long wait_limit_ns;
  int o_align32;   // o is 32-byte aligned: 32-byte stores in the epilogue
  // 8-bit inputs only: dequantisation factors [B, Hkv] of Q, K, V (null = 1)
  const float* descale_q;
  const float* descale_k;
  const float* descale_v;
};

template <int D, bool kF8 = false>
struct PrefillLayout {
  static constexpr int kRowBytes = D * (kF8 ? 1 : 2);
  static constexpr int kBoxes = kRowBytes / 128;  // 128-byte swizzle boxes per row
  static constexpr int kBoxElems = 128 / (kF8 ? 1 : 2);
  static constexpr int kTileBytes = kBM * kRowBytes;
  static constexpr int kStages = (kTileBytes == 32768) ? 4 : 8;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
  // q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2][2 halves], o_full[2], mma_done,
  // q_empty
  static constexpr int kBarQ = 0;
  static constexpr int kBarKvFull = 1;
  static constexpr int kBarKvEmpty = 1 + kStages;
  static constexpr int kBarSFull = 1 + 2 * kStages;
  static constexpr int kBarPFull = kBarSFull + 2;
  static constexpr int kBarOFull = kBarPFull + 4;
  static constexpr int kBarDone = kBarOFull + 2;
  static constexpr int kBarQEmpty = kBarDone + 1;
  static constexpr int kNumBars = kBarQEmpty + 1;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemSlotOff + 4;
  static constexpr int kBytes = kAbortOff + 4 + 1024;  // + slack for 1024-byte alignment
};

// Number of key/value tiles query tile starting at row r0 must visit (0 for
// a tile outside the launch's range).
__device__ __forceinline__ int prefill_tiles_for(const PrefillParams& p, int r0) {
  if (r0 >= p.Sq || r0 >= p.q_tile_end * kBM || p.Skv <= 0) return 0;
  if (!p.causal) return p.n_kv_tiles;
  const int last_row = min(r0 + kBM - 1, p.Sq - 1);
  const long long last_key = static_cast<long long>(last_row) + (p.Skv - p.Sq);
  if (last_key < 0) return 0;
  return min(p.n_kv_tiles, static_cast<int>(last_key / kBN) + 1);
}

struct PrefillItem {
  int tile0, b, h, g, n0, n1;  // query tiles tile0 and tile0 + 1 of head (b, h)
};

// Item k in longest-first order: pairs of query tiles in descending order
// under a causal mask, heads of one key/value group adjacent.
__device__ __forceinline__ PrefillItem prefill_item(const PrefillParams& p, int k) {
  PrefillItem it;
  const int bh_count = p.B * p.Hq;
  int pair = k / bh_count;
  if (p.causal) pair = p.n_qpairs - 1 - pair;
  it.tile0 = p.q_tile0 + 2 * pair;
  const int bh = k % bh_count;
  it.b = bh / p.Hq;
  it.h = bh % p.Hq;
  it.g = it.h / p.group;
  it.n0 = prefill_tiles_for(p, it.tile0 * kBM);
  it.n1 = prefill_tiles_for(p, (it.tile0 + 1) * kBM);
  return it;
}

// The item this CTA takes in round r (snake order over the CTAs), or -1.
__device__ __forceinline__ int prefill_item_index(const PrefillParams& p, int r) {
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const long long k = static_cast<long long>(r) * G + ((r & 1) ? (G - 1 - c) : c);
  return k < p.n_items ? static_cast<int>(k) : -1;
}

// ---------------------------------------------------------------------------
// Softmax warpgroup: one thread per query row.
// ---------------------------------------------------------------------------
template <int D, bool kF8>
__device__ __forceinline__ void prefill_softmax(const PrefillParams& p, uint32_t tmem,
                                                uint32_t bar_s, uint32_t bar_p, uint32_t bar_o,
                                                int w, volatile int* abort_flag) {
  const int warp_in_wg = (threadIdx.x >> 5) & 3;
  const int row_in_tile = warp_in_wg * 32 + (threadIdx.x & 31);
  const uint32_t lane_off = static_cast<uint32_t>(warp_in_wg * 32) << 16;
  const uint32_t tS = tmem + lane_off + static_cast<uint32_t>(w * 128);
  const uint32_t tO = tmem + lane_off + static_cast<uint32_t>(256 + w * D);
  constexpr float kThreshold = kF8 ? kRescaleThresholdF8 : kRescaleThreshold;
  const int off = p.Skv - p.Sq;
  uint32_t tcount = 0;  // tiles this warpgroup has processed (phase of s_full / p_full)
  uint32_t ocount = 0;  // items this warpgroup has finished with tiles (phase of o_full)

  for (int r = 0;; ++r) {
  const int k_item = prefill_item_index(p, r);
  if (k_item < 0) break;
  const PrefillItem item = prefill_item(p, k_item);
  const int n_tiles = w ? item.n1 : item.n0;
  // score-to-exponent constant, natural-unit score scale, output factor
  float c = p.scale_log2, lse_scale = p.scale, o_factor = 1.f;
  if constexpr (kF8) {
    const int bg = item.b * p.Hkv + item.g;
    const float f = (p.descale_q ? p.descale_q[bg] : 1.f) * (p.descale_k ? p.descale_k[bg] : 1.f);
    c *= f;
    lse_scale *= f;
    o_factor = p.descale_v ? p.descale_v[bg] : 1.f;
  }
  const int q_row0 = (item.tile0 + w) * kBM;
  const int row = q_row0 + row_in_tile;
  // rows of this launch: inside the sequence and inside the launch's tile range
  const bool row_out = row < p.Sq && item.tile0 + w < p.q_tile_end;
  // keys with index > last_key are masked for this row
  const long long last_key_ll = p.causal ? static_cast<long long>(row) + off
                                         : static_cast<long long>(p.Skv) - 1;
  const int last_key = static_cast<int>(min(last_key_ll, static_cast<long long>(p.Skv) - 1));

  float m = -INFINITY;
  float l = 0.f;   // sum of the fp32 weights: the LSE's
  float lq = 0.f;  // sum of the weights as P.V sees them (bf16): O's normaliser
  const size_t bh = static_cast<size_t>(item.b) * p.Hq + item.h;
  const size_t o_index = bh * p.o_rows + (row - p.o_row0);
  const size_t lse_index = bh * p.lse_rows + (row - p.lse_row0);

  if (n_tiles == 0) {
    if (row_out) {
      uint4* dst = reinterpret_cast<uint4*>(p.o + o_index * D);
#pragma unroll
      for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
      p.lse[lse_index] = -INFINITY;
    }
    continue;
  }

  for (int j = 0; j < n_tiles; ++j, ++tcount) {
    bool ok = mbar_wait(bar_s, tcount & 1u, abort_flag, p.wait_limit_ns);
    if (!__all_sync(0xffffffffu, ok)) return;
    tc_fence_after();

    // scores: the second half streams in while the first half's max runs
    float s[kBN];
    {
      uint32_t ra[64], rb[64];
      tmem_ld64_nowait(tS, ra);
      tmem_ld_wait_hold(ra);
      tmem_ld64_nowait(tS + 64, rb);
#pragma unroll
      for (int e = 0; e < 64; ++e) s[e] = __uint_as_float(ra[e]);
      tmem_ld_wait_hold(rb);
#pragma unroll
      for (int e = 0; e < 64; ++e) s[64 + e] = __uint_as_float(rb[e]);
    }

    const int key0 = j * kBN;
    const bool tile_masked = (key0 + kBN > p.Skv) ||
                             (p.causal && static_cast<long long>(key0) + kBN - 1 >
                                              static_cast<long long>(q_row0) + off);
    if (tile_masked) {
      const int lim = last_key - key0;  // columns > lim are invisible
#pragma unroll
      for (int e = 0; e < kBN; ++e)
        if (e > lim) s[e] = -INFINITY;
    }

    // row max (exact in any order): three-input max over eight partial maxima
    float mx[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) mx[k] = fmaxf(s[2 * k], s[2 * k + 1]);
#pragma unroll
    for (int i = 16; i < kBN; i += 16)
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], s[i + 2 * k], s[i + 2 * k + 1]);
    const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                           fmaxf(mx[6], mx[7]));
    const float m_new = fmaxf(m, mt);
    float alpha = 1.f;
    if ((m_new - m) * c > kThreshold) {  // false while both are -inf (NaN)
      alpha = ex2((m - m_new) * c);              // 0 when m was -inf
      l *= alpha;
      lq *= alpha;
      m = m_new;
    }
    const bool rescale_o = (j > 0) && __any_sync(0xffffffffu, alpha != 1.f);
    const float mc = (m == -INFINITY) ? 0.f : m * c;

    if (rescale_o) {
      // PV for tile j-1 has completed (its commit precedes this tile's S
      // commit) and PV for tile j waits for the arrives below.
#pragma unroll
      for (int q4 = 0; q4 < D / 32; ++q4) {
        uint32_t r[32];
        tmem_ld32(tO + q4 * 32, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
        tmem_st32(tO + q4 * 32, r);
      }
    }

    // p = 2^(s*c - m*c) on pairs; l sums the fp32 p, P keeps them as bf16.
    // Each half of the row (64 keys) is stored to tensor memory and
    // announced on its own barrier, so P.V on the first 64 keys runs while
    // the second half is computed.
    const float2 c2 = make_float2(c, c);
    const float nmc = kF8 ? kPOffsetF8 - mc : -mc;
    const float2 nmc2 = make_float2(nmc, nmc);
    float2 rs[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                    make_float2(0.f, 0.f)};
    float2 rq[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    // Masked tiles take every exponential on the MUFU (2^-inf is exactly 0);
    // the others move kPolyPairsPer8 of every 8 pairs to the FMA pipe.
    auto exps_half = [&](auto poly_tag, int half) {
      constexpr bool kPoly = decltype(poly_tag)::value;
      if constexpr (kF8) {
        // four keys per 32-bit column; pairs (2i, 2i+1) of the row
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = half * 64 + 4 * i;
          const float2 x0 = ffma2(make_float2(s[e], s[e + 1]), c2, nmc2);
          const float2 x1 = ffma2(make_float2(s[e + 2], s[e + 3]), c2, nmc2);
          const float2 p0 = (kPoly && ((2 * i) & 7) >= 8 - kPolyPairsPer8F8)
                                ? exp2_poly2(x0) : make_float2(ex2(x0.x), ex2(x0.y));
          const float2 p1 = (kPoly && ((2 * i + 1) & 7) >= 8 - kPolyPairsPer8F8)
                                ? exp2_poly2(x1) : make_float2(ex2(x1.x), ex2(x1.y));
          rs[(2 * i) & 3] = fadd2(rs[(2 * i) & 3], p0);
          rs[(2 * i + 1) & 3] = fadd2(rs[(2 * i + 1) & 3], p1);
          pk[i] = pack_e4m3x4(p0.x, p0.y, p1.x, p1.y);
        }
        tmem_st16(tS + half * 16, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(bar_p + 8 * half);
        return;
      }
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int e = half * 64 + 2 * i;
        const float2 x = ffma2(make_float2(s[e], s[e + 1]), c2, nmc2);
        const float2 pp = (kPoly && (i & 7) >= 8 - kPolyPairsPer8)
                              ? exp2_poly2(x)
                              : make_float2(ex2(x.x), ex2(x.y));
        rs[i & 3] = fadd2(rs[i & 3], pp);
        pk[i] = pack_bf16x2(pp.x, pp.y);
        // the pair as the tensor core reads it, added straight from bf16
        add_bf16x2_to(rq[i & 1], pk[i]);
      }
      tmem_st32(tS + half * 32, pk);
      tmem_st_wait();
      tc_fence_before();
      // one arrival per warp once all its lanes' stores are done
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bar_p + 8 * half);
    };
    // (with no polynomial share the two variants would be the same code twice)
    if (tile_masked || (kF8 ? kPolyPairsPer8F8 : kPolyPairsPer8) == 0) {
      exps_half(std::false_type{}, 0);
      exps_half(std::false_type{}, 1);
    } else {
      exps_half(std::true_type{}, 0);
      exps_half(std::true_type{}, 1);
    }
    {
      const float2 t2 = fadd2(fadd2(rs[0], rs[1]), fadd2(rs[2], rs[3]));
      l += t2.x + t2.y;
      const float2 q2 = fadd2(rq[0], rq[1]);
      lq += q2.x + q2.y;
    }
  }

  // epilogue: O / l -> bf16, LSE = m*scale + ln l
  bool ok = mbar_wait(bar_o, ocount & 1u, abort_flag, p.wait_limit_ns);
  ++ocount;
  if (!__all_sync(0xffffffffu, ok)) return;
  tc_fence_after();
  // O is divided by the sum of the very weights P.V used (the bf16-rounded
  // ones), so a weight's rounding moves numerator and denominator alike: a
  // row dominated by one key gets that key's value almost exactly, which an
  // fp32 normaliser misses by up to half a bf16 ulp of the dominant weight.
  // 8-bit P keeps the fp32 normaliser (its rounding is covered by the E4M3
  // error bound).  The LSE always uses the fp32 sum.
  const float l_o = kF8 ? l : lq;
  const float inv_l = (l_o > 0.f) ? o_factor / l_o : 0.f;
  {
    uint32_t r[D];
    tmem_ld_row<D>(tO, r);
    if (row_out) {
      uint8_t* dst = reinterpret_cast<uint8_t*>(p.o + o_index * D);
      const float2 il = make_float2(inv_l, inv_l);
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t w8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 x = fmul2(make_float2(__uint_as_float(r[16 * c + 2 * e]),
                                             __uint_as_float(r[16 * c + 2 * e + 1])), il);
          w8[e] = pack_bf16x2(x.x, x.y);
        }
        if (p.o_align32) {
          st_global_v8(dst + 32 * c, w8);
        } else {
          reinterpret_cast<uint4*>(dst + 32 * c)[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
          reinterpret_cast<uint4*>(dst + 32 * c)[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
        }
      }
    }
  }
  if (row_out) {
    float lse = m * lse_scale + logf(l);
    if constexpr (kF8) lse -= kPOffsetF8 * 0.69314718055994531f;  // the 2^6 of P
    p.lse[lse_index] = (l > 0.f) ? lse : -INFINITY;
  }
  }
}

// ---------------------------------------------------------------------------
// TMA producer (one thread).
// ---------------------------------------------------------------------------
template <int D, bool kF8>
__device__ __forceinline__ void prefill_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                                 const CUtensorMap* tm_v, const PrefillParams& p,
                                                 uint32_t sbase, volatile int* abort_flag) {
  using L = PrefillLayout<D, kF8>;
  const uint32_t bars = sbase + L::kBarOff;
  tma_prefetch_desc(tm_q);
  tma_prefetch_desc(tm_k);
  tma_prefetch_desc(tm_v);
  const uint32_t bar_q = bars + 8 * L::kBarQ;
  uint32_t nq = 0;  // query loads issued (one per item)
  uint32_t ld = 0;  // key/value tile loads issued
  bool stop = false;
  for (int r = 0; !stop; ++r) {
    const int k_item = prefill_item_index(p, r);
    if (k_item < 0) break;
    const PrefillItem item = prefill_item(p, k_item);
    // The query buffer is free once the previous item's last score MMA is done.
    if (nq > 0 && !mbar_wait(bars + 8 * L::kBarQEmpty, (nq - 1) & 1u, abort_flag,
                             p.wait_limit_ns))
      break;
    mbar_arrive_expect_tx(bar_q, 2 * L::kTileBytes);
#pragma unroll
    for (int w = 0; w < 2; ++w)
#pragma unroll
      for (int kb = 0; kb < L::kBoxes; ++kb)
        tma_load_3d(sbase + L::kQOff + w * L::kTileBytes + kb * kSwzBytes, tm_q, bar_q,
                    kb * L::kBoxElems, (item.tile0 + w) * kBM, item.b * p.Hq + item.h);
    ++nq;
    const int n_max = max(item.n0, item.n1);
    for (int idx = 0; idx < 2 * n_max; ++idx) {
      const uint32_t stage = ld % L::kStages;
      if (!mbar_wait(bars + 8 * (L::kBarKvEmpty + stage), ((ld / L::kStages) & 1u) ^ 1u,
                     abort_flag, p.wait_limit_ns)) {
        stop = true;
        break;
      }
      const uint32_t bar_full = bars + 8 * (L::kBarKvFull + stage);
      mbar_arrive_expect_tx(bar_full, L::kTileBytes);
      const CUtensorMap* tm = (idx & 1) ? tm_v : tm_k;
#pragma unroll
      for (int kb = 0; kb < L::kBoxes; ++kb)
        tma_load_3d(sbase + L::kRingOff + stage * L::kTileBytes + kb * kSwzBytes, tm, bar_full,
                    kb * L::kBoxElems, (idx >> 1) * kBN, item.b * p.Hkv + item.g);
      ++ld;
    }
  }

  // Drain: no copy may still be in flight when the CTA exits.
  if (nq > 0) mbar_wait(bar_q, (nq - 1) & 1u, nullptr, p.wait_limit_ns);
  const uint32_t S = static_cast<uint32_t>(L::kStages);
  for (uint32_t k = (ld > S ? ld - S : 0u); k < ld; ++k)
    mbar_wait(bars + 8 * (L::kBarKvFull + k % S), (k / S) & 1u, nullptr, p.wait_limit_ns);
}

// ---------------------------------------------------------------------------
// MMA issuer (one thread).
// ---------------------------------------------------------------------------
template <int D, bool kF8>
__device__ __forceinline__ void prefill_mma(const PrefillParams& p, uint32_t sbase, uint32_t tmem,
                                            volatile int* abort_flag) {
  using L = PrefillLayout<D, kF8>;
  const uint32_t bars = sbase + L::kBarOff;
  constexpr uint32_t kIdS = kF8 ? idesc_e4m3_f32(kBM, kBN, false) : idesc_bf16_f32(kBM, kBN, false);
  constexpr uint32_t kIdPV = kF8 ? idesc_e4m3_f32(kBM, D, true) : idesc_bf16_f32(kBM, D, true);
  constexpr int kKeysPerMma = kF8 ? 32 : 16;  // K of one MMA: 32 bytes of a row

  auto kv_stage = [](uint32_t idx) { return static_cast<int>(idx % L::kStages); };
  auto kv_wait = [&](uint32_t idx) -> bool {
    return mbar_wait(bars + 8 * (L::kBarKvFull + kv_stage(idx)),
                     static_cast<uint32_t>(idx / L::kStages) & 1u, abort_flag, p.wait_limit_ns);
  };
  // Shared-memory descriptors are formed once; a descriptor of the same
  // layout at a byte offset o is the base plus o / 16 (the start address
  // field holds address / 16 and never carries: shared addresses are below
  // 2^18).  Keeping one 64-bit base per operand keeps this thread's register
  // count inside the control warpgroup's share.
  const uint64_t q_desc0 = sw128_desc(sbase + L::kQOff, 16, 1024);
  const uint64_t k_desc0 = sw128_desc(sbase + L::kRingOff, 16, 1024);
  const uint64_t v_desc0 = sw128_desc(sbase + L::kRingOff, kSwzBytes, 1024);
  // S_w = Q_w K^T: M=128 rows, N=128 keys, K=D in steps of 32 bytes (16 bf16
  // or 32 E4M3 elements).
  auto issue_s = [&](int w, int stage) {
    const uint64_t qd = q_desc0 + static_cast<uint64_t>((w * L::kTileBytes) >> 4);
    const uint64_t kd = k_desc0 + static_cast<uint64_t>((stage * L::kTileBytes) >> 4);
    auto step = [&](auto kk_c) {
      constexpr int kk = decltype(kk_c)::value;
      constexpr uint32_t o = static_cast<uint32_t>(((kk >> 2) * kSwzBytes + (kk & 3) * 32) >> 4);
      if constexpr (kF8)
        mma_ss_f8_off<o, o>(tmem + w * 128, qd, kd, kIdS, kk > 0 ? 1u : 0u);
      else
        mma_ss_off<o, o>(tmem + w * 128, qd, kd, kIdS, kk > 0 ? 1u : 0u);
    };
    static_for<L::kRowBytes / 32>(step);
  };
  // O_w += P_w V: A = P_w in TMEM (8 columns per MMA: 16 bf16 or 32 E4M3
  // keys), B = V tile (keys x D, D contiguous: MN-major; bf16 d = 128 has two
  // 64-element column blocks 16 KB apart).  Issued per half of the keys, each
  // after its half of P is announced.
  auto issue_pv_half = [&](int w, int stage, int half, bool accumulate) {
    const uint64_t vd0 = v_desc0 + static_cast<uint64_t>((stage * L::kTileBytes) >> 4);
    constexpr int kSteps = (kBN / 2) / kKeysPerMma;
    const uint64_t vdh = vd0 + static_cast<uint64_t>((half * kSteps * kKeysPerMma * 128) >> 4);
    auto step = [&](auto k4_c) {
      constexpr int k4 = decltype(k4_c)::value;
      constexpr uint32_t o = static_cast<uint32_t>((k4 * kKeysPerMma * 128) >> 4);
      const int kk = half * kSteps + k4;
      if constexpr (kF8)
        mma_ts_f8_off<o>(tmem + 256 + w * D, tmem + w * 128 + kk * 8, vdh, kIdPV,
                         (accumulate || kk > 0) ? 1u : 0u);
      else
        mma_ts_off<o>(tmem + 256 + w * D, tmem + w * 128 + kk * 8, vdh, kIdPV,
                      (accumulate || kk > 0) ? 1u : 0u);
    };
    static_for<kSteps>(step);
  };
  auto wait_p = [&](int w, int half, uint32_t cnt) -> bool {
    if (!mbar_wait(bars + 8 * (L::kBarPFull + 2 * w + half), cnt & 1u,
                   abort_flag, p.wait_limit_ns))
      return false;
    tc_fence_after();
    return true;
  };

  {
    uint32_t nq = 0;                 // items started (phase of q_full / q_empty)
    uint32_t base = 0;               // ring index of the current item's first K tile
    uint32_t pc[2] = {0u, 0u};       // tiles of each query tile consumed (phase of p_full)
    for (int r = 0;; ++r) {
      const int k_item = prefill_item_index(p, r);
      if (k_item < 0) break;
      const PrefillItem item = prefill_item(p, k_item);
      if (!mbar_wait(bars + 8 * L::kBarQ, nq & 1u, abort_flag, p.wait_limit_ns)) goto done;
      ++nq;
      const int n0 = item.n0, n1 = item.n1;
      const int n_max = max(n0, n1);
      if (n_max == 0) {
        mma_commit(bars + 8 * L::kBarQEmpty);
        continue;
      }
      if (!kv_wait(base)) goto done;
      tc_fence_after();
      if (n0 > 0) { issue_s(0, kv_stage(base)); mma_commit(bars + 8 * (L::kBarSFull + 0)); }
      if (n1 > 0) { issue_s(1, kv_stage(base)); mma_commit(bars + 8 * (L::kBarSFull + 1)); }
      mma_commit(bars + 8 * (L::kBarKvEmpty + kv_stage(base)));
      if (n_max == 1) mma_commit(bars + 8 * L::kBarQEmpty);  // last score MMA of the item

      for (int j = 0; j < n_max; ++j) {
        const uint32_t iv = base + 2 * j + 1, ik = base + 2 * j + 2;
        if (!kv_wait(iv)) goto done;
        tc_fence_after();
        if (j < n0) {
          if (!wait_p(0, 0, pc[0])) goto done;
          issue_pv_half(0, kv_stage(iv), 0, j > 0);
          if (!wait_p(0, 1, pc[0])) goto done;
          issue_pv_half(0, kv_stage(iv), 1, j > 0);
          ++pc[0];
          if (j == n0 - 1) mma_commit(bars + 8 * (L::kBarOFull + 0));
        }
        const bool next = (j + 1 < n_max);
        if (next) {
          if (!kv_wait(ik)) goto done;
          tc_fence_after();
          if (j + 1 < n0) { issue_s(0, kv_stage(ik)); mma_commit(bars + 8 * (L::kBarSFull + 0)); }
        }
        if (j < n1) {
          if (!wait_p(1, 0, pc[1])) goto done;
          issue_pv_half(1, kv_stage(iv), 0, j > 0);
          if (!wait_p(1, 1, pc[1])) goto done;
          issue_pv_half(1, kv_stage(iv), 1, j > 0);
          ++pc[1];
          if (j == n1 - 1) mma_commit(bars + 8 * (L::kBarOFull + 1));
        }
        mma_commit(bars + 8 * (L::kBarKvEmpty + kv_stage(iv)));
        if (next) {
          if (j + 1 < n1) { issue_s(1, kv_stage(ik)); mma_commit(bars + 8 * (L::kBarSFull + 1)); }
          mma_commit(bars + 8 * (L::kBarKvEmpty + kv_stage(ik)));
          if (j + 2 == n_max) mma_commit(bars + 8 * L::kBarQEmpty);  // last score MMA
        }
      }
      base += 2 * static_cast<uint32_t>(n_max);
    }
  }
done:
  // Every MMA this thread issued completes before tensor memory is freed.
  mma_commit(bars + 8 * L::kBarDone);
  mbar_wait(bars + 8 * L::kBarDone, 0u, nullptr, p.wait_limit_ns);
}

template <int D, bool kF8 = false>
__global__ void __launch_bounds__(kPrefillThreads, 1)
fa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using L = PrefillLayout<D, kF8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbortOff);
  const uint32_t bars = sbase + L::kBarOff;
  if (threadIdx.x == 0) {
    mbar_init(bars + 8 * L::kBarQ, 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(bars + 8 * (L::kBarKvFull + s), 1);
      mbar_init(bars + 8 * (L::kBarKvEmpty + s), 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(bars + 8 * (L::kBarSFull + w), 1);
      mbar_init(bars + 8 * (L::kBarPFull + 2 * w), 4);  // one arrival per softmax warp
      mbar_init(bars + 8 * (L::kBarPFull + 2 * w + 1), 4);
      mbar_init(bars + 8 * (L::kBarOFull + w), 1);
    }
    mbar_init(bars + 8 * L::kBarDone, 1);
    mbar_init(bars + 8 * L::kBarQEmpty, 1);
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
    warpgroup_reg_alloc<kSoftmaxRegs>();
    const int w = warp >> 2;
    prefill_softmax<D, kF8>(p, tmem, bars + 8 * (L::kBarSFull + w), bars + 8 * (L::kBarPFull + 2 * w),
                       bars + 8 * (L::kBarOFull + w), w, abort_flag);
  } else {
    warpgroup_reg_dealloc<kControlRegs>();
    if (warp == 8) {
      if (lane == 0)
        prefill_producer<D, kF8>(&tm_q, &tm_k, &tm_v, p, sbase, abort_flag);
    } else if (warp == 9) {
      if (lane == 0) prefill_mma<D, kF8>(p, sbase, tmem, abort_flag);
    }
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
