// fa_api.cu -- the C ABI of libfa.so (declared in include/fa.h): argument
// checks, TMA tensor-map encoding and kernel launches.  Every kernel of the
// library lives in this one translation unit.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "sm100.cuh"
#include "prefill_sm100.cuh"
#include "decode_sm100.cuh"
#include "backward_sm100.cuh"
#include "ffn_sm100.cuh"

namespace {

constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s per mbarrier wait
// Backward CTA order: groups of (batch, kv-head) pairs worth this many waves
// of CTAs (see fa::bwd_tile).
constexpr int kBwdGroupWaves = 4;
// The interleaved backward order is used while a group's K, V, Q and dO stay
// within this many bytes (two groups in flight fit the 126 MB L2 with room).
constexpr double kBwdInterleaveBytes = 48.0 * 1024 * 1024;
constexpr int kMaxDevices = 64;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// --- driver entry point for the tensor-map encoder (no link to libcuda) ----
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// [planes, rows, d] bf16 tensor as a 3-D map with 64 x 128 x 1 boxes, 128B
// swizzle; rows beyond `rows` read as zeros.
bool encode_bhsd(CUtensorMap* map, const void* base, int d, int rows, long long planes) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t r = static_cast<cuuint64_t>(rows > 0 ? rows : 1);
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), r, static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, r * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [planes, rows, d] E4M3 (one byte per element) tensor as a 3-D map with
// 128 x 128 x 1 boxes (128-byte rows), 128B swizzle; rows beyond `rows` read
// as zeros.
bool encode_bhsd_e4m3(CUtensorMap* map, const void* base, int d, int rows, long long planes) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t r = static_cast<cuuint64_t>(rows > 0 ? rows : 1);
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), r, static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d), r * static_cast<cuuint64_t>(d)};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, cols] bf16 matrix (a weight, K = cols contiguous) as a 3-D map with
// 64 x 256 x 1 boxes, 128B swizzle.
bool encode_rows256(CUtensorMap* map, const void* base, int cols, int rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), 1};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2,
                           static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[3] = {64, 256, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One-time per-device opt-in to the prefill kernels' dynamic shared memory,
// and the device's SM count (the persistent grid size).
std::once_flag g_attr_once[kMaxDevices];
cudaError_t g_attr_err[kMaxDevices];
int g_prefill_sms[kMaxDevices];

// The prefill kernel moves registers between its warpgroups (setmaxnreg);
// that is only safe when every thread was launched with the register count
// the split was computed for, so a build that compiled to another count is
// refused instead of launched.
template <int D, bool kF8 = false>
cudaError_t check_prefill_regs() {
  cudaFuncAttributes a;
  cudaError_t e = cudaFuncGetAttributes(&a, fa::fa_prefill_kernel<D, kF8>);
  if (e != cudaSuccess) return e;
  return a.numRegs == fa::kPrefillLaunchRegs ? cudaSuccess : cudaErrorInvalidKernelImage;
}

cudaError_t prepare_prefill(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_attr_once[dev], [dev] {
    cudaError_t e = cudaDeviceGetAttribute(&g_prefill_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = check_prefill_regs<64>();
    if (e == cudaSuccess) e = check_prefill_regs<128>();
    if (e == cudaSuccess) e = check_prefill_regs<128, true>();
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::fa_prefill_kernel<128, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fa::PrefillLayout<128, true>::kBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::fa_prefill_kernel<64>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fa::PrefillLayout<64>::kBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::fa_prefill_kernel<128>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fa::PrefillLayout<128>::kBytes);
    g_attr_err[dev] = e;
  });
  return g_attr_err[dev];
}

// Which query tiles a prefill launch computes and where its outputs go: a
// whole forward is tiles [0, ceil(Sq/128)) into o [B,Hq,Sq,d], lse [B,Hq,Sq].
struct PrefillRange {
  int q_tile0, q_tile_end;
  int o_rows, o_row0, lse_rows, lse_row0;
};

template <int D, bool kF8 = false>
fa_status launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int Hq, int Hkv, int Sq, int Skv, int causal, float scale,
                         cudaStream_t stream, const float* descale_q = nullptr,
                         const float* descale_k = nullptr, const float* descale_v = nullptr,
                         const PrefillRange* range = nullptr) {
  CUtensorMap tq, tk, tv;
  auto encode = kF8 ? encode_bhsd_e4m3 : encode_bhsd;
  if (Skv == 0) k = v = q;  // no key tile is ever loaded; any valid address will do
  if (!encode(&tq, q, D, Sq, static_cast<long long>(B) * Hq) ||
      !encode(&tk, k, D, Skv, static_cast<long long>(B) * Hkv) ||
      !encode(&tv, v, D, Skv, static_cast<long long>(B) * Hkv))
    return FA_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (prepare_prefill(dev) != cudaSuccess) return FA_ERR_CUDA;

  fa::PrefillParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_align32 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Sq = Sq;
  p.Skv = Skv;
  p.group = Hq / Hkv;
  p.causal = causal ? 1 : 0;
  const int q_tiles = (Sq + fa::kBM - 1) / fa::kBM;
  const PrefillRange whole{0, q_tiles, Sq, 0, Sq, 0};
  const PrefillRange& rg = range ? *range : whole;
  p.q_tile0 = rg.q_tile0;
  p.q_tile_end = rg.q_tile_end;
  p.o_rows = rg.o_rows;
  p.o_row0 = rg.o_row0;
  p.lse_rows = rg.lse_rows;
  p.lse_row0 = rg.lse_row0;
  p.n_qpairs = (rg.q_tile_end - rg.q_tile0 + 1) / 2;
  p.n_items = p.n_qpairs * B * Hq;
  if (p.n_items <= 0) return FA_OK;
  p.n_kv_tiles = (Skv + fa::kBN - 1) / fa::kBN;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = kWaitLimitNs;
  p.descale_q = descale_q;
  p.descale_k = descale_k;
  p.descale_v = descale_v;
  const int sms = g_prefill_sms[dev] > 0 ? g_prefill_sms[dev] : 1;
  const int grid = p.n_items < sms ? p.n_items : sms;  // persistent: one CTA per SM
  fa::fa_prefill_kernel<D, kF8><<<static_cast<unsigned>(grid), fa::kPrefillThreads,
                                  fa::PrefillLayout<D, kF8>::kBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Per device: SM count, and the decode kernels' shared-memory opt-in.
std::once_flag g_dec_once[kMaxDevices];
cudaError_t g_dec_err[kMaxDevices];
int g_num_sms[kMaxDevices];

template <int D>
cudaError_t decode_attr() {
  cudaError_t e = cudaSuccess;
  auto set = [&e](const void* fn) {
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fa::DecodeLayout<D>::kBytes);
  };
  set(reinterpret_cast<const void*>(fa::fa_decode_split_kernel<D, 1>));
  set(reinterpret_cast<const void*>(fa::fa_decode_split_kernel<D, 2>));
  set(reinterpret_cast<const void*>(fa::fa_decode_split_kernel<D, 4>));
  set(reinterpret_cast<const void*>(fa::fa_decode_split_kernel<D, 8>));
  return e;
}

cudaError_t prepare_decode(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_dec_once[dev], [dev] {
    cudaError_t e = cudaDeviceGetAttribute(&g_num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = decode_attr<64>();
    if (e == cudaSuccess) e = decode_attr<128>();
    g_dec_err[dev] = e;
  });
  return g_dec_err[dev];
}

// [planes, rows, d] bf16 cache as a 3-D map with 64 x box_rows x 1 boxes.
bool encode_cache(CUtensorMap* map, const void* base, int d, int rows, long long planes,
                  int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t r = static_cast<cuuint64_t>(rows > 0 ? rows : 1);
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), r, static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, r * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A paged pool [planes, P, 128] bf16 (P = page_size, a multiple of 8) as the
// 5-D view (64 columns, 8 rows, 2 column halves, P/8 row groups, planes) with
// boxes of box_rows rows: shared memory receives [group][half][8 rows][64],
// the interleaved tile layout of the decode kernel at d = 128.
bool encode_pool_interleaved(CUtensorMap* map, const void* base, int page_size, long long planes,
                             int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[5] = {64, 8, 2, static_cast<cuuint64_t>(page_size / 8),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[4] = {256, 128, 2048, static_cast<cuuint64_t>(page_size) * 256};
  cuuint32_t box[5] = {64, 8, 2, static_cast<cuuint32_t>(box_rows / 8), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, d] bf16 query matrix as a 2-D map with 64 x 16 boxes.
bool encode_query(CUtensorMap* map, const void* base, int d, long long rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(fa::kDecNPad)};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A paged cache: [num_pages, Hkv, page_size, d] plus a [B, max_pages] block table.
struct PagedCache {
  const int32_t* block_table;
  int num_pages, page_size, max_pages;
};

template <int D, int G>
fa_status launch_decode(const void* q, const void* kc, const void* vc, const int32_t* seqlens,
                        float* o_part, float* lse_part, int B, int Hq, int Hkv, int Lmax,
                        int num_splits, float scale, int num_sms, cudaStream_t stream,
                        const PagedCache* pg) {
  CUtensorMap tk, tv, tk32, tv32, tq;
  // Contiguous: planes (b, g) of Lmax rows.  Paged: planes (page, g) of page_size rows.
  const long long planes = pg ? static_cast<long long>(pg->num_pages) * Hkv
                              : static_cast<long long>(B) * Hkv;
  const int rows = pg ? pg->page_size : Lmax;
  const int box_main = pg ? std::min(pg->page_size, fa::kDecBN) : fa::kDecBN;
  const int box_tail = pg ? std::min(pg->page_size, fa::kDecSubRows) : fa::kDecSubRows;
  // paged at d = 128: one box per page slice, both column halves
  // (interleaved); should the driver refuse that view, two boxes per slice
  bool interleaved = (pg != nullptr) && D == 128;
  if (interleaved)
    interleaved = encode_pool_interleaved(&tk, kc, pg->page_size, planes, box_main) &&
                  encode_pool_interleaved(&tv, vc, pg->page_size, planes, box_main) &&
                  encode_pool_interleaved(&tk32, kc, pg->page_size, planes, box_tail) &&
                  encode_pool_interleaved(&tv32, vc, pg->page_size, planes, box_tail);
  if (interleaved) {
  } else if (!encode_cache(&tk, kc, D, rows, planes, box_main) ||
             !encode_cache(&tv, vc, D, rows, planes, box_main) ||
             !encode_cache(&tk32, kc, D, rows, planes, box_tail) ||
             !encode_cache(&tv32, vc, D, rows, planes, box_tail)) {
    return FA_ERR_CUDA;
  }
  if (!encode_query(&tq, q, D, static_cast<long long>(B) * Hq)) return FA_ERR_CUDA;
  fa::DecodeParams p;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.seqlens = seqlens;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Lmax = Lmax;
  p.n_splits = num_splits;
  p.n_items = B * Hkv * num_splits;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = kWaitLimitNs;
  p.block_table = pg ? pg->block_table : nullptr;
  p.max_pages = pg ? pg->max_pages : 0;
  int shift = 0;
  while (pg && (1 << shift) < pg->page_size) ++shift;
  p.page_shift = shift;
  p.rows_main = box_main;
  p.rows_tail = box_tail;
  p.interleaved = interleaved ? 1 : 0;
  p.chunk_align = pg ? fa::kDecBN : 1;
  const int grid = p.n_items < num_sms ? p.n_items : num_sms;
  fa::fa_decode_split_kernel<D, G><<<grid, fa::kDecThreads, fa::DecodeLayout<D>::kBytes,
                                     stream>>>(tk, tv, tk32, tv32, tq, p);
  return FA_OK;
}

template <int D>
fa_status dispatch_decode_group(int G, const void* q, const void* kc, const void* vc,
                                const int32_t* seqlens, float* o_part, float* lse_part, int B,
                                int Hq, int Hkv, int Lmax, int num_splits, float scale,
                                int num_sms, cudaStream_t stream, const PagedCache* pg) {
  switch (G) {
    case 1: return launch_decode<D, 1>(q, kc, vc, seqlens, o_part, lse_part, B, Hq, Hkv, Lmax, num_splits, scale, num_sms, stream, pg);
    case 2: return launch_decode<D, 2>(q, kc, vc, seqlens, o_part, lse_part, B, Hq, Hkv, Lmax, num_splits, scale, num_sms, stream, pg);
    case 4: return launch_decode<D, 4>(q, kc, vc, seqlens, o_part, lse_part, B, Hq, Hkv, Lmax, num_splits, scale, num_sms, stream, pg);
    case 8: return launch_decode<D, 8>(q, kc, vc, seqlens, o_part, lse_part, B, Hq, Hkv, Lmax, num_splits, scale, num_sms, stream, pg);
    default: return FA_ERR_UNSUPPORTED;
  }
}

__global__ void timeout_probe_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = fa::smem_addr(&bar);
  if (threadIdx.x == 0) {
    fa::mbar_init(b, 1);
    abort_flag = 0;
    fa::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on this barrier: the bounded wait must give up.
    fa::mbar_wait(b, 0u, &abort_flag, limit_ns);
  }
}

// ---------------------------------------------------------------------------
// Fixed, library-owned scratch for fa_decode_noalloc.
// ---------------------------------------------------------------------------
// FA_DECODE_NOALLOC_BYTES (32 MiB) on every device that loads this library,
// held until the process exits.  The name is only a host-side stand-in: host code obtains the
// device address with cudaGetSymbolAddress (once per device, that device
// current) and passes that address to the kernels.
constexpr size_t kNoAllocScratchBytes = FA_DECODE_NOALLOC_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices];  // device address per device; null until set up

cudaError_t noalloc_scratch_address(int dev, void** addr) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  return cudaSuccess;
}

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = fa::exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = fa::exp2_poly2(make_float2(x[i], 0.f)).x;
  }
}

}  // namespace

// Backward: per-device shared-memory opt-in.
std::once_flag g_bwd_once[kMaxDevices];
cudaError_t g_bwd_err[kMaxDevices];
int g_bwd_sms[kMaxDevices];

cudaError_t prepare_backward(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_bwd_once[dev], [dev] {
    cudaError_t e = cudaDeviceGetAttribute(&g_bwd_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::fa_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fa::bwd_smem_bytes<64>());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::fa_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fa::bwd_smem_bytes<128>());
    g_bwd_err[dev] = e;
  });
  return g_bwd_err[dev];
}

// CTA order of the backward launch (fa::bwd_tile).  Work of a CTA in tile
// steps: a dK/dV CTA on key tile j visits group * (query tiles from the first
// that sees j); a dQ CTA on query tile i visits the key tiles i sees.
struct BwdOrder {
  bool interleave;
  int heads_per_group, q_heads_per_group;
};
BwdOrder backward_order(int B, int Hq, int Hkv, int Sq, int Skv, int d, bool causal,
                        int n_kv_tiles, int n_q_tiles, int sms) {
  const int group = Hq / Hkv;
  const long long off = static_cast<long long>(Skv) - Sq;
  long long pair_steps = 0, longest = 1;  // per (batch, kv-head) pair
  for (int j = 0; j < n_kv_tiles; ++j) {
    long long first = 0;
    if (causal) {
      const long long need = static_cast<long long>(j) * fa::kBwdBM - off;
      first = need <= 0 ? 0 : need / fa::kBwdBN;
    }
    const long long steps = group * std::max(0LL, n_q_tiles - first);
    pair_steps += steps;
    longest = std::max(longest, steps);
  }
  for (int i = 0; i < n_q_tiles; ++i) {
    long long keys = n_kv_tiles;
    if (causal) {
      const long long q_last = std::min(static_cast<long long>(i) * fa::kBwdBN + fa::kBwdBN - 1,
                                        static_cast<long long>(Sq) - 1);
      const long long k_last = q_last + off;
      keys = k_last < 0 ? 0 : std::min<long long>(n_kv_tiles, k_last / fa::kBwdBM + 1);
    }
    pair_steps += group * keys;
    longest = std::max(longest, keys);
  }
  const int pairs = B * Hkv;
  const int ctas_per_pair = n_kv_tiles + group * n_q_tiles;
  BwdOrder o;
  // interleaved: about kBwdGroupWaves waves per group, and enough pairs that a
  // group's span on the SMs is at least twice its longest CTA
  long long g = std::max<long long>(1, kBwdGroupWaves * static_cast<long long>(sms) / ctas_per_pair);
  if (pair_steps > 0)
    g = std::max(g, (2 * longest * sms + pair_steps - 1) / pair_steps);
  g = std::min<long long>(g, pairs);
  // bytes a group streams: K, V of its pairs and Q, dO of their query heads
  const double pair_bytes = 2.0 * 2.0 * d * (static_cast<double>(Skv) + group * static_cast<double>(Sq));
  o.interleave = g * pair_bytes <= kBwdInterleaveBytes;
  if (o.interleave) {
    o.heads_per_group = static_cast<int>(g);
    o.q_heads_per_group = 1;  // unused
  } else {
    o.heads_per_group = std::max(1, std::min(pairs, kBwdGroupWaves * sms / std::max(1, n_kv_tiles)));
    o.q_heads_per_group = std::max(1, std::min(B * Hq, kBwdGroupWaves * sms / std::max(1, n_q_tiles)));
  }
  return o;
}

// Sets the order fields of p (whose sizes are set) and returns the grid: the
// dK/dV CTAs (one per batch, kv head and key tile) plus the dQ CTAs (one per
// batch, query head and query tile).
long long fill_backward_order(fa::BwdParams& p, int d, int sms) {
  const BwdOrder order = backward_order(p.B, p.Hq, p.Hkv, p.Sq, p.Skv, d, p.causal != 0,
                                        p.n_kv_tiles, p.n_q_tiles, sms);
  p.interleave = order.interleave ? 1 : 0;
  p.heads_per_group = order.heads_per_group;
  p.q_heads_per_group = order.q_heads_per_group;
  const long long kv_ctas = static_cast<long long>(p.B) * p.Hkv * p.n_kv_tiles;
  p.n_kv_ctas = static_cast<int>(kv_ctas);
  return kv_ctas + static_cast<long long>(p.B) * p.Hq * p.n_q_tiles;
}

// D = rowsum(dO * O) into the workspace, then the dK/dV kernel (one CTA per
// key tile) and the dQ kernel (one CTA per query tile); neither writes what
// the other reads, and each gradient is written once.
template <int D>
fa_status launch_backward(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* d_o, void* dq, void* dk, void* dv,
                          float* workspace, int B, int Hq, int Hkv, int Sq, int Skv, int causal,
                          float scale, cudaStream_t stream) {
  const int n_q_tiles = (Sq + fa::kBwdBN - 1) / fa::kBwdBN;
  const long long rows_padded = static_cast<long long>(B) * Hq * n_q_tiles * fa::kBwdBN;
  float* ld = workspace;
  // no key tile is loaded or stored without keys; any valid address will do
  if (Skv == 0) {
    k = v = q;
    dk = dv = dq;
  }
  fa::fa_bwd_dsum_kernel<D><<<static_cast<unsigned>(rows_padded / fa::kDsumRowsPerBlock), 256, 0,
                               stream>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(d_o), lse, ld, Sq,
      n_q_tiles, rows_padded);
  const int n_kv_tiles = (Skv + fa::kBwdBM - 1) / fa::kBwdBM;
  CUtensorMap tq, tk, tv, tdo, tdq, tdk, tdv;
  if (!encode_bhsd(&tq, q, D, Sq, static_cast<long long>(B) * Hq) ||
      !encode_bhsd(&tdo, d_o, D, Sq, static_cast<long long>(B) * Hq) ||
      !encode_bhsd(&tdq, dq, D, Sq, static_cast<long long>(B) * Hq) ||
      !encode_bhsd(&tk, k, D, Skv, static_cast<long long>(B) * Hkv) ||
      !encode_bhsd(&tv, v, D, Skv, static_cast<long long>(B) * Hkv) ||
      !encode_bhsd(&tdk, dk, D, Skv, static_cast<long long>(B) * Hkv) ||
      !encode_bhsd(&tdv, dv, D, Skv, static_cast<long long>(B) * Hkv))
    return FA_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (prepare_backward(dev) != cudaSuccess) return FA_ERR_CUDA;
  fa::BwdParams p;
  p.ld = ld;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Sq = Sq;
  p.Skv = Skv;
  p.group = Hq / Hkv;
  p.causal = causal ? 1 : 0;
  p.n_kv_tiles = n_kv_tiles;
  p.n_q_tiles = n_q_tiles;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = kWaitLimitNs;
  const unsigned grid = static_cast<unsigned>(fill_backward_order(p, D, g_bwd_sms[dev]));
  // programmatic dependent launch: the CTAs' setup and their K, V, Q and dO
  // loads overlap the D kernel's tail; the reads of its output wait for it
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(fa::kBwdThreads);
  cfg.dynamicSmemBytes = fa::bwd_smem_bytes<D>();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fa::fa_bwd_kernel<D>, tq, tk, tv, tdo, tdq, tdk, tdv, p) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Feed-forward network after attention: per-device shared-memory opt-in.
std::once_flag g_ffn_once[kMaxDevices];
cudaError_t g_ffn_err[kMaxDevices];
int g_ffn_sms[kMaxDevices];

cudaError_t prepare_ffn(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_ffn_once[dev], [dev] {
    cudaError_t e = cudaDeviceGetAttribute(&g_ffn_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fa::fa_ffn_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fa::FfnLayout::kBytes);
    g_ffn_err[dev] = e;
  });
  return g_ffn_err[dev];
}

// One persistent launch of the feed-forward GEMM over row_tiles query tiles
// (one CTA per SM, at most one per output tile).
void launch_ffn(const CUtensorMap& tm_a, const CUtensorMap& tm_b, fa::FfnParams p, int row_tiles,
                int dev, cudaStream_t s) {
  p.n_row_tiles = row_tiles;
  const int tiles = row_tiles * (p.N / fa::kFfnBN);
  const int grid = std::max(1, std::min(tiles, g_ffn_sms[dev]));
  // programmatic dependent launch: the CTAs' setup overlaps the previous
  // kernel's end; the kernel waits for it before its first load
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(fa::kFfnThreads);
  cfg.dynamicSmemBytes = fa::FfnLayout::kBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  (void)cudaLaunchKernelEx(&cfg, fa::fa_ffn_gemm_kernel, tm_a, tm_b, p);
}

extern "C" {

size_t fa_bwd_workspace_bytes(int B, int Hq, int Sq, int d) {
  if (B <= 0 || Hq <= 0 || Sq <= 0 || d <= 0) return 0;
  // per 128-row query tile: 128 values of -LSE*log2(e) and 128 of D, fp32
  const size_t tiles = (static_cast<size_t>(Sq) + 127) / 128;
  return static_cast<size_t>(B) * Hq * tiles * 256 * sizeof(float);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* d_o, void* dq, void* dk, void* dv, float* workspace, int B, int Hq,
                 int Hkv, int Sq, int Skv, int d, int causal, float scale, fa_stream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Sq < 0 || Skv < 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || (Sq == 0 && Skv == 0)) return FA_OK;
  // the query-side buffers may be null with no query rows, the key-side ones
  // with no keys (nothing is read from or written to them)
  if ((Sq > 0 && (q == nullptr || o == nullptr || lse == nullptr || d_o == nullptr ||
                  dq == nullptr || workspace == nullptr)) ||
      (Skv > 0 && (k == nullptr || v == nullptr || dk == nullptr || dv == nullptr)))
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(d_o) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      !aligned16(workspace))
    return FA_ERR_ALIGNMENT;
  const long long n_kv_tiles = (static_cast<long long>(Skv) + fa::kBwdBM - 1) / fa::kBwdBM;
  const long long n_q_tiles = (static_cast<long long>(Sq) + fa::kBwdBN - 1) / fa::kBwdBN;
  // one grid of dK/dV and dQ CTAs; the D kernel's grid has 16 blocks per query tile
  if (static_cast<long long>(B) * Hkv * n_kv_tiles + static_cast<long long>(B) * Hq * n_q_tiles >
          0x7fffffffLL ||
      static_cast<long long>(B) * Hq * n_q_tiles * 16 > 0x7fffffffLL ||
      static_cast<long long>(B) * Hkv > 0x7fffffffLL)
    return FA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (Sq == 0) {  // no query rows: every key gets zero gradients
    const size_t kv_bytes = static_cast<size_t>(B) * Hkv * Skv * d * 2;
    if (cudaMemsetAsync(dk, 0, kv_bytes, s) != cudaSuccess ||
        cudaMemsetAsync(dv, 0, kv_bytes, s) != cudaSuccess)
      return FA_ERR_CUDA;
    return FA_OK;
  }
  return d == 64 ? launch_backward<64>(q, k, v, o, lse, d_o, dq, dk, dv, workspace, B, Hq, Hkv,
                                       Sq, Skv, causal, scale, s)
                 : launch_backward<128>(q, k, v, o, lse, d_o, dq, dk, dv, workspace, B, Hq, Hkv,
                                        Sq, Skv, causal, scale, s);
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                 int Hkv, int Sq, int Skv, int d, int causal, float scale, fa_stream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Sq < 0 || Skv < 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (scale < 0.f) return FA_ERR_UNSUPPORTED;  // softmax follows the largest raw score
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || Sq == 0) return FA_OK;  // nothing to compute
  // no keys: k and v may be null (nothing is read from them)
  if (q == nullptr || o == nullptr || lse == nullptr ||
      (Skv > 0 && (k == nullptr || v == nullptr)))
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_ALIGNMENT;
  const long long q_tiles = (static_cast<long long>(Sq) + fa::kBM - 1) / fa::kBM;
  const long long grid = (q_tiles + 1) / 2 * B * static_cast<long long>(Hq);
  if (grid > 0x7fffffffLL || static_cast<long long>(B) * Hq > 0x7fffffffLL ||
      static_cast<long long>(B) * Hkv > 0x7fffffffLL)
    return FA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? launch_prefill<64>(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, causal, scale, s)
                 : launch_prefill<128>(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, causal, scale, s);
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, const float* descale_q,
                     const float* descale_k, const float* descale_v, void* o, float* lse, int B,
                     int Hq, int Hkv, int Sq, int Skv, int d, int causal, float scale,
                     fa_stream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Sq < 0 || Skv < 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (scale < 0.f) return FA_ERR_UNSUPPORTED;  // softmax follows the largest raw score
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || Sq == 0) return FA_OK;  // nothing to compute
  // no keys: k and v may be null (nothing is read from them)
  if (q == nullptr || o == nullptr || lse == nullptr ||
      (Skv > 0 && (k == nullptr || v == nullptr)))
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_ALIGNMENT;
  auto aligned4 = [](const float* f) { return (reinterpret_cast<uintptr_t>(f) & 3u) == 0; };
  if (!aligned4(descale_q) || !aligned4(descale_k) || !aligned4(descale_v))
    return FA_ERR_ALIGNMENT;
  const long long q_tiles = (static_cast<long long>(Sq) + fa::kBM - 1) / fa::kBM;
  const long long grid = (q_tiles + 1) / 2 * B * static_cast<long long>(Hq);
  if (grid > 0x7fffffffLL || static_cast<long long>(B) * Hq > 0x7fffffffLL ||
      static_cast<long long>(B) * Hkv > 0x7fffffffLL)
    return FA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return launch_prefill<128, true>(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, causal, scale, s,
                                   descale_q, descale_k, descale_v);
}

size_t fa_bpt_workspace_bytes(int F, int chunk_tiles) {
  if (F < 1 || chunk_tiles < 1) return 0;
  return static_cast<size_t>(chunk_tiles) * fa::kFfnBM * static_cast<size_t>(F) * 2;
}

fa_status fa_bpt_ffn(const void* o, const void* w1, const void* w2, void* y,
                                void* workspace, int B, int Hq, int S, int d, int F,
                                int chunk_tiles, fa_stream_t stream) {
  if (B < 0 || Hq < 1 || S < 0 || F < 1 || chunk_tiles < 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long D = static_cast<long long>(Hq) * d;
  if (D % fa::kFfnBN != 0 || F % fa::kFfnBN != 0 || D > (1 << 20) || F > (1 << 20))
    return FA_ERR_UNSUPPORTED;
  if (B == 0 || S == 0) return FA_OK;  // nothing to compute
  if (o == nullptr || w1 == nullptr || w2 == nullptr || y == nullptr || workspace == nullptr)
    return FA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(w1) || !aligned16(w2) || !aligned16(y) || !aligned16(workspace))
    return FA_ERR_ALIGNMENT;
  const long long tiles_per_seq = (static_cast<long long>(S) + fa::kFfnBM - 1) / fa::kFfnBM;
  const long long total_tiles = tiles_per_seq * B;
  if (total_tiles > 0x7fffffffLL || static_cast<long long>(B) * Hq > 0x7fffffffLL ||
      static_cast<long long>(B) * S * D > (1LL << 40) || chunk_tiles > 65535)
    return FA_ERR_UNSUPPORTED;
  CUtensorMap tm_o, tm_w1, tm_w2, tm_h;
  if (!encode_bhsd(&tm_o, o, d, S, static_cast<long long>(B) * Hq) ||
      !encode_rows256(&tm_w1, w1, static_cast<int>(D), F) ||
      !encode_rows256(&tm_w2, w2, F, static_cast<int>(D)) ||
      !encode_bhsd(&tm_h, workspace, F, chunk_tiles * fa::kFfnBM, 1))
    return FA_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (prepare_ffn(dev) != cudaSuccess) return FA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  fa::FfnParams p1;  // H = gelu(X W1^T), X read from the attention output
  p1.c = static_cast<__nv_bfloat16*>(workspace);
  p1.N = F;
  p1.K = static_cast<int>(D);
  p1.S = S;
  p1.Hq = Hq;
  p1.d = d;
  p1.tiles_per_seq = static_cast<int>(tiles_per_seq);
  p1.a_heads = 1;
  p1.c_tokens = 0;
  p1.S_out = S;
  p1.tok0 = 0;
  p1.gelu = 1;
  p1.wait_limit_ns = kWaitLimitNs;
  fa::FfnParams p2 = p1;  // Y = H W2^T, rows back to their tokens
  p2.c = static_cast<__nv_bfloat16*>(y);
  p2.N = static_cast<int>(D);
  p2.K = F;
  p2.a_heads = 0;
  p2.c_tokens = 1;
  p2.gelu = 0;
  for (long long mt0 = 0; mt0 < total_tiles; mt0 += chunk_tiles) {
    const int n = static_cast<int>(std::min<long long>(chunk_tiles, total_tiles - mt0));
    p1.mt0 = p2.mt0 = static_cast<int>(mt0);
    launch_ffn(tm_o, tm_w1, p1, n, dev, s);
    launch_ffn(tm_h, tm_w2, p2, n, dev, s);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

size_t fa_bpt_layer_workspace_bytes(int B, int Hq, int d, int F, int chunk_tiles) {
  if (B < 1 || Hq < 1 || d < 1 || F < 1 || chunk_tiles < 1) return 0;
  const size_t rows = static_cast<size_t>(chunk_tiles) * fa::kBM;
  const size_t o_bytes = static_cast<size_t>(B) * Hq * rows * d * 2;
  return ((o_bytes + 255) & ~static_cast<size_t>(255)) + static_cast<size_t>(B) * rows * F * 2;
}

fa_status fa_bpt_layer(const void* q, const void* k, const void* v, const void* w1,
                       const void* w2, void* y, float* lse, void* workspace, int B, int Hq,
                       int Hkv, int S, int d, int F, int causal, float scale, int chunk_tiles,
                       fa_stream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || S < 0 || F < 1 || chunk_tiles < 1) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (scale < 0.f) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long D = static_cast<long long>(Hq) * d;
  if (D % fa::kFfnBN != 0 || F % fa::kFfnBN != 0 || D > (1 << 20) || F > (1 << 20))
    return FA_ERR_UNSUPPORTED;
  if (B == 0 || S == 0) return FA_OK;
  if (q == nullptr || k == nullptr || v == nullptr || w1 == nullptr || w2 == nullptr ||
      y == nullptr || lse == nullptr || workspace == nullptr)
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(w1) || !aligned16(w2) ||
      !aligned16(y) || !aligned16(lse) || !aligned16(workspace))
    return FA_ERR_ALIGNMENT;
  const long long tiles_per_seq = (static_cast<long long>(S) + fa::kBM - 1) / fa::kBM;
  if (chunk_tiles > tiles_per_seq) chunk_tiles = static_cast<int>(tiles_per_seq);
  const long long rows = static_cast<long long>(chunk_tiles) * fa::kBM;  // chunk rows per head
  if (static_cast<long long>(B) * Hq * rows > 0x7fffffffLL ||
      static_cast<long long>(B) * chunk_tiles > 65535 ||
      static_cast<long long>(B) * S * D > (1LL << 40) || static_cast<long long>(B) * Hq > 0x7fffffffLL)
    return FA_ERR_UNSUPPORTED;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  void* o_chunk = ws;
  const size_t o_bytes = static_cast<size_t>(B) * Hq * rows * d * 2;
  void* h_chunk = ws + ((o_bytes + 255) & ~static_cast<size_t>(255));
  CUtensorMap tm_o, tm_w1, tm_w2, tm_h;
  if (!encode_bhsd(&tm_o, o_chunk, d, static_cast<int>(rows), static_cast<long long>(B) * Hq) ||
      !encode_rows256(&tm_w1, w1, static_cast<int>(D), F) ||
      !encode_rows256(&tm_w2, w2, F, static_cast<int>(D)) ||
      !encode_bhsd(&tm_h, h_chunk, F, static_cast<int>(B * rows), 1))
    return FA_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (prepare_ffn(dev) != cudaSuccess) return FA_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (long long c0 = 0; c0 < tiles_per_seq; c0 += chunk_tiles) {
    const int tiles = static_cast<int>(std::min<long long>(chunk_tiles, tiles_per_seq - c0));
    const int tok0 = static_cast<int>(c0 * fa::kBM);
    // 1. attention for query tiles [c0, c0 + tiles) of every (b, h): O into
    //    the chunk buffer (its row 0 is query row tok0), LSE into lse
    const PrefillRange rg{static_cast<int>(c0), static_cast<int>(c0) + tiles,
                          static_cast<int>(rows), tok0, S, 0};
    const fa_status st =
        d == 64 ? launch_prefill<64>(q, k, v, o_chunk, lse, B, Hq, Hkv, S, S, causal, scale, s,
                                     nullptr, nullptr, nullptr, &rg)
                : launch_prefill<128>(q, k, v, o_chunk, lse, B, Hq, Hkv, S, S, causal, scale, s,
                                      nullptr, nullptr, nullptr, &rg);
    if (st != FA_OK) return st;
    // 2. H = gelu(X W1^T) of the chunk's tokens; 3. y = H W2^T at their tokens
    fa::FfnParams p1;
    p1.c = static_cast<__nv_bfloat16*>(h_chunk);
    p1.N = F;
    p1.K = static_cast<int>(D);
    p1.S = static_cast<int>(std::min<long long>(rows, S - tok0));
    p1.Hq = Hq;
    p1.d = d;
    p1.tiles_per_seq = tiles;
    p1.mt0 = 0;
    p1.a_heads = 1;
    p1.c_tokens = 0;
    p1.S_out = S;
    p1.tok0 = tok0;
    p1.gelu = 1;
    p1.wait_limit_ns = kWaitLimitNs;
    fa::FfnParams p2 = p1;
    p2.c = static_cast<__nv_bfloat16*>(y);
    p2.N = static_cast<int>(D);
    p2.K = F;
    p2.a_heads = 0;
    p2.c_tokens = 1;
    p2.gelu = 0;
    launch_ffn(tm_o, tm_w1, p1, B * tiles, dev, s);
    launch_ffn(tm_h, tm_w2, p2, B * tiles, dev, s);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

fa_status fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* seqlens_k, float* o_partial, float* lse_partial, int B,
                            int Hq, int Hkv, int Lmax, int d, int num_splits, float scale,
                            fa_stream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Lmax < 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > 256) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (scale < 0.f) return FA_ERR_UNSUPPORTED;  // softmax follows the largest raw score
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || seqlens_k == nullptr ||
      o_partial == nullptr || lse_partial == nullptr)
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(seqlens_k) & 3u) != 0 ||
      !aligned16(o_partial) || !aligned16(lse_partial))
    return FA_ERR_ALIGNMENT;
  if (static_cast<long long>(B) * Hkv * num_splits > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (prepare_decode(dev) != cudaSuccess) return FA_ERR_CUDA;
  const int sms = g_num_sms[dev];
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const fa_status st =
      d == 64 ? dispatch_decode_group<64>(G, q, k_cache, v_cache, seqlens_k, o_partial,
                                          lse_partial, B, Hq, Hkv, Lmax, num_splits, scale, sms, s,
                                          nullptr)
              : dispatch_decode_group<128>(G, q, k_cache, v_cache, seqlens_k, o_partial,
                                           lse_partial, B, Hq, Hkv, Lmax, num_splits, scale, sms,
                                           s, nullptr);
  if (st != FA_OK) return st;
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_decode_paged_splitkv(const void* q, const void* k_pages, const void* v_pages,
                                  const int32_t* block_table, const int32_t* seqlens_k,
                                  float* o_partial, float* lse_partial, int B, int Hq, int Hkv,
                                  int num_pages, int page_size, int max_pages, int d,
                                  int num_splits, float scale, fa_stream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || num_pages < 1 || max_pages < 1) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > 256) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (scale < 0.f) return FA_ERR_UNSUPPORTED;  // softmax follows the largest raw score
  if (page_size < 16 || page_size > 256 || (page_size & (page_size - 1)) != 0)
    return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return FA_ERR_UNSUPPORTED;
  const long long lmax = static_cast<long long>(max_pages) * page_size;
  if (lmax > 0x7fffffffLL - fa::kDecBN ||
      static_cast<long long>(num_pages) * Hkv > 0x7fffffffLL ||
      static_cast<long long>(B) * max_pages > 0x7fffffffLL ||
      static_cast<long long>(B) * Hkv * num_splits > 0x7fffffffLL)
    return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  if (q == nullptr || k_pages == nullptr || v_pages == nullptr || block_table == nullptr ||
      seqlens_k == nullptr || o_partial == nullptr || lse_partial == nullptr)
    return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) ||
      (reinterpret_cast<uintptr_t>(seqlens_k) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) != 0 ||
      !aligned16(o_partial) || !aligned16(lse_partial))
    return FA_ERR_ALIGNMENT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (prepare_decode(dev) != cudaSuccess) return FA_ERR_CUDA;
  const int sms = g_num_sms[dev];
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const PagedCache pg{block_table, num_pages, page_size, max_pages};
  const int Lmax = static_cast<int>(lmax);
  const fa_status st =
      d == 64 ? dispatch_decode_group<64>(G, q, k_pages, v_pages, seqlens_k, o_partial,
                                          lse_partial, B, Hq, Hkv, Lmax, num_splits, scale, sms, s,
                                          &pg)
              : dispatch_decode_group<128>(G, q, k_pages, v_pages, seqlens_k, o_partial,
                                           lse_partial, B, Hq, Hkv, Lmax, num_splits, scale, sms,
                                           s, &pg);
  if (st != FA_OK) return st;
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_combine(const float* o_partial, const float* lse_partial, void* o, float* lse, int B,
                     int Hq, int num_splits, int d, fa_stream_t stream) {
  if (B < 0 || Hq < 1) return FA_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > 256) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  if (o_partial == nullptr || lse_partial == nullptr || o == nullptr || lse == nullptr)
    return FA_ERR_INVALID_ARG;
  if (!aligned16(o_partial) || !aligned16(lse_partial) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_ALIGNMENT;
  const long long rows = static_cast<long long>(B) * Hq;
  if (rows > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  const unsigned blocks = static_cast<unsigned>((rows + 3) / 4);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // programmatic dependent launch: scheduled while the previous kernel (the
  // split) finishes; the kernel waits for it before reading the partials
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(o);
  const int nrows = static_cast<int>(rows);
  const cudaError_t e =
      d == 64 ? cudaLaunchKernelEx(&cfg, fa::fa_combine_kernel<64>, o_partial, lse_partial, ob, lse,
                                   nrows, num_splits)
              : cudaLaunchKernelEx(&cfg, fa::fa_combine_kernel<128>, o_partial, lse_partial, ob,
                                   lse, nrows, num_splits);
  if (e != cudaSuccess) return FA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_decode_default_splits(int B, int Hkv, int Lmax, int num_sms) {
  if (B < 1 || Hkv < 1 || Lmax < 1) return 1;
  if (num_sms < 1) num_sms = 1;
  // About 1024 keys per chunk, and at least 8 CTAs per SM overall.
  long long n = (Lmax + 1023) / 1024;
  const long long units = static_cast<long long>(B) * Hkv;
  const long long want = (8LL * num_sms + units - 1) / units;
  if (n < want) n = want;
  const long long max_useful = (Lmax + 63) / 64;  // keep chunks >= 64 keys
  if (n > max_useful) n = max_useful;
  if (n < 1) n = 1;
  if (n > 256) n = 256;
  return static_cast<int>(n);
}

fa_status fa_shard_units(int B, int Hkv, int n_shards, int shard, int* first, int* count) {
  if (B < 1 || Hkv < 1 || n_shards < 1 || shard < 0 || shard >= n_shards || first == nullptr ||
      count == nullptr)
    return FA_ERR_INVALID_ARG;
  const long long units = static_cast<long long>(B) * Hkv;
  const long long a = units * shard / n_shards, b = units * (shard + 1) / n_shards;
  *first = static_cast<int>(a);
  *count = static_cast<int>(b - a);
  return FA_OK;
}

fa_status fa_shard_sequences(const int32_t* seqlens_k, int B, int n_shards, int32_t* bounds) {
  if (B < 1 || n_shards < 1 || seqlens_k == nullptr || bounds == nullptr)
    return FA_ERR_INVALID_ARG;
  long long total = 0;
  for (int b = 0; b < B; ++b) total += std::max(seqlens_k[b], 1);
  // bounds[s] = smallest b' whose prefix [0, b') holds at least s/n of the
  // total; prefix counts are non-decreasing, so the bounds are too.
  long long run = 0;
  int s = 1;
  bounds[0] = 0;
  for (int b = 0; b < B && s < n_shards; ++b) {
    run += std::max(seqlens_k[b], 1);
    while (s < n_shards && run * n_shards >= total * s) bounds[s++] = b + 1;
  }
  while (s < n_shards) bounds[s++] = B;
  bounds[n_shards] = B;
  return FA_OK;
}

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: null pointer or bad size";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: shape or head size not implemented";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA call or kernel launch failed";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT: a kernel gave up a bounded wait";
  }
  return "unknown fa_status";
}

fa_status fa_get_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_device_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(fa::g_device_status, &zero, sizeof(int)) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  return static_cast<fa_status>(v);
}

fa_status fa_debug_exp2_poly(const float* x, float* y, int n, fa_stream_t stream) {
  if (n < 0) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (x == nullptr || y == nullptr) return FA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return FA_ERR_ALIGNMENT;
  const int pairs = (n + 1) / 2;
  exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_debug_bwd_tiles(int B, int Hq, int Hkv, int Sq, int Skv, int d, int causal, int sms,
                             int* tiles, long long capacity, long long* n_ctas, int* interleave) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Skv < 0 || sms < 1 || Hq % Hkv != 0 ||
      n_ctas == nullptr || interleave == nullptr || capacity < 0)
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  fa::BwdParams p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Sq = Sq;
  p.Skv = Skv;
  p.group = Hq / Hkv;
  p.causal = causal ? 1 : 0;
  p.n_kv_tiles = (Skv + fa::kBwdBM - 1) / fa::kBwdBM;
  p.n_q_tiles = (Sq + fa::kBwdBN - 1) / fa::kBwdBN;
  const long long grid = fill_backward_order(p, d, sms);
  *n_ctas = grid;
  *interleave = p.interleave;
  if (tiles == nullptr) return FA_OK;
  if (capacity < grid) return FA_ERR_INVALID_ARG;
  for (long long blk = 0; blk < grid; ++blk) {
    const fa::BwdTile t = fa::bwd_tile_of(p, static_cast<int>(blk));
    tiles[4 * blk + 0] = t.kv ? 1 : 0;
    tiles[4 * blk + 1] = t.b;
    tiles[4 * blk + 2] = t.hg;
    tiles[4 * blk + 3] = t.t;
  }
  return FA_OK;
}

fa_status fa_debug_timeout_probe(unsigned int limit_us, fa_stream_t stream) {
  if (limit_us == 0 || limit_us > 10000000u) return FA_ERR_INVALID_ARG;
  timeout_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* seqlens_k, void* o, float* lse, int B, int Hq,
                            int Hkv, int Lmax, int d, int num_splits, float scale,
                            fa_stream_t stream) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Lmax < 0) return FA_ERR_INVALID_ARG;
  if (num_splits < 1 || num_splits > 256) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  // Split partials: o_part [B,Hq,n,d] fp32 at offset 0, lse_part [B,Hq,n] fp32
  // at the next 256-byte boundary.  Larger than the fixed array: refuse.
  const unsigned long long rows = static_cast<unsigned long long>(B) * Hq * num_splits;
  const unsigned long long o_bytes = rows * static_cast<unsigned long long>(d) * 4ull;
  const unsigned long long lse_off = (o_bytes + 255ull) & ~255ull;
  if (lse_off + rows * 4ull > kNoAllocScratchBytes) return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  if (o == nullptr || lse == nullptr) return FA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGNMENT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  void* base = nullptr;
  if (noalloc_scratch_address(dev, &base) != cudaSuccess) return FA_ERR_CUDA;
  float* o_part = static_cast<float*>(base);
  float* lse_part = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + lse_off);
  // Every partial the merge reads is written by the split pass first, so the
  // array's previous contents never matter and nothing is cleared.
  const fa_status st = fa_decode_splitkv(q, k_cache, v_cache, seqlens_k, o_part, lse_part, B,
                                         Hq, Hkv, Lmax, d, num_splits, scale, stream);
  if (st != FA_OK) return st;
  return fa_combine(o_part, lse_part, o, lse, B, Hq, num_splits, d, stream);
}

}  // extern "C"
