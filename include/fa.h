/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library libfa.so.
 *
 * The library computes exact softmax attention without writing the score
 * matrix to HBM: query blocks stay on chip while key/value blocks stream past
 * them, and an online softmax keeps a running max and sum per row, rescaling
 * the partial output whenever the max grows ("I/O-Aware Kernels", section
 * "FlashAttention"; "FlashAttention & IO-aware attention", section "Direct
 * answer").  Single-query decode splits the key/value length across SMs and
 * merges the pieces by their log-sum-exp ("FlashAttention & IO-aware
 * attention", sections "Deep dive" and "Interviewer follow-ups").
 *
 * Conventions shared by every entry point
 *  - Pointers are DEVICE pointers of the current CUDA device, unless stated.
 *    The caller owns every buffer; the library allocates no device memory and
 *    keeps no per-call state.  All tensors are contiguous, row-major.
 *  - bf16 is IEEE-754 binary16-bfloat (the bit pattern of __nv_bfloat16).
 *  - Calls only enqueue work on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and return without synchronising.  A fault during
 *    execution surfaces at the caller's next synchronisation.
 *  - Errors are returned, never printed and never trapped.  Argument checks
 *    run before any CUDA call; a call that fails them launches nothing.
 *  - A kernel that gives up one of its bounded waits (see
 *    fa_get_device_status) returns early: the outputs of that call are then
 *    undefined (partly written, or holding what the buffers held before), and
 *    only fa_get_device_status() tells.  Check it before trusting outputs of
 *    a run in which anything went wrong.
 *  - Unsupported head sizes are rejected with FA_ERR_UNSUPPORTED: there is no
 *    slower fallback path ("FlashAttention & IO-aware attention", section
 *    "Interviewer follow-ups", warns that a silent fallback to a materialising
 *    kernel is why a "flash" path can fail to be fast).
 *  - Thread safety: calls hold no shared mutable state apart from the
 *    one-time lookup of the driver's tensor-map encoder, which is guarded.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque stream handle; pass a cudaStream_t. */
typedef struct CUstream_st *fa_stream_t;

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,     /* null pointer, negative or inconsistent size */
    FA_ERR_UNSUPPORTED = 2,     /* valid but not implemented (e.g. head size) */
    FA_ERR_ALIGNMENT = 3,       /* a pointer is not 16-byte aligned */
    FA_ERR_CUDA = 4,            /* a CUDA runtime/driver call or launch failed */
    FA_ERR_DEVICE_TIMEOUT = 5   /* a kernel gave up a bounded wait (see below) */
} fa_status;

/*
 * fa_fwd -- fused exact attention forward (prefill).
 *
 *   O[b,h,i,:] = sum_j softmax_j(scale * q[b,h,i,:] . k[b,g,j,:]) * v[b,g,j,:]
 *   LSE[b,h,i] = ln sum_j exp(scale * q[b,h,i,:] . k[b,g,j,:])
 *
 * over the visible keys j, with g = h / (Hq / Hkv) (grouped-query heads share
 * a key/value head; MHA when Hq == Hkv).  The naive form of this computation
 * is the one "I/O-Aware Kernels", section "The Memory Bottleneck", describes;
 * this call never materialises the score matrix.
 *
 *   q    [B, Hq,  Sq,  d] bf16      o   [B, Hq, Sq, d] bf16 (written)
 *   k, v [B, Hkv, Skv, d] bf16      lse [B, Hq, Sq]    fp32 (written, natural log)
 *   causal != 0: key j is visible to query i iff j <= i + (Skv - Sq)
 *       (bottom-right alignment).  A query row that sees no key gets
 *       O = 0 and LSE = -inf.
 *   scale: multiplies q.k before the softmax (normally 1/sqrt(d)); must be
 *       >= 0 (the kernel follows the largest raw score q.k, which is the
 *       softmax's largest only for a non-negative scale), else
 *       FA_ERR_UNSUPPORTED.
 *
 * Supported: d in {64, 128}; Hq % Hkv == 0; B, Hq, Hkv >= 1; Sq, Skv >= 0
 * (Sq == 0 or B == 0 is a no-op).  All five pointers 16-byte aligned.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT before any
 * CUDA call; FA_ERR_CUDA if the tensor-map encoder or the launch fails.
 */
fa_status fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                 int B, int Hq, int Hkv, int Sq, int Skv, int d, int causal,
                 float scale, fa_stream_t stream);

/*
 * fa_fwd_fp8 -- fa_fwd on 8-bit inputs (the FP8 variant of FlashAttention-3
 * that "FlashAttention & IO-aware attention", section "Deep dive", names; the
 * page fixes no format or scaling, so this call defines its own):
 *
 *   q, k, v hold E4M3 codes (OCP 8-bit float: 4 exponent bits with bias 7,
 *   3 mantissa bits, no infinities, NaN = S.1111.111), one byte per element,
 *   in the layouts of fa_fwd.  descale_q, descale_k, descale_v are device
 *   arrays of B * Hkv fp32 factors, [b * Hkv + g]; the real input of head h
 *   of batch b is factor[b, g] * value(code) with g = h / (Hq / Hkv) for the
 *   queries and g = h for keys and values.  A null factor pointer means 1.
 *   Factors must be positive and finite (the kernel cannot check device
 *   memory; a negative Q or K factor gives meaningless results, as a
 *   negative scale would).
 *   o and lse are those of fa_fwd on the real inputs (o bf16, lse fp32).
 *
 * Arithmetic: both products on the tensor cores in E4M3 with fp32
 * accumulation; the softmax weights are quantised to E4M3 for P V (as
 * p * 2^6, p relative to a reference max that lags the row max by at most
 * 2^2), while the normaliser l and LSE use the unquantised fp32 weights.
 * Per output element the error against exact attention of the real inputs is
 * at most 2^-4 * sum_j w_j |v_j| (w = softmax weights; E4M3 keeps 3 mantissa
 * bits) + n * 2^-16 * max|v| (n visible keys; E4M3 subnormals) + the bf16
 * rounding of o.  LSE is as accurate as fa_fwd's.
 *
 * Supported: d == 128 (other d: FA_ERR_UNSUPPORTED); otherwise as fa_fwd.
 * q, k, v, o, lse 16-byte aligned; factor arrays 4-byte aligned
 * (FA_ERR_ALIGNMENT).  Errors as fa_fwd.
 */
fa_status fa_fwd_fp8(const void *q, const void *k, const void *v, const float *descale_q,
                     const float *descale_k, const float *descale_v, void *o, float *lse,
                     int B, int Hq, int Hkv, int Sq, int Skv, int d, int causal,
                     float scale, fa_stream_t stream);

/*
 * fa_bwd -- gradients of fa_fwd by recomputation.
 *
 * "Tracing Tiled QKV Data Movement in FlashAttention's Memory Hierarchy"
 * (closing takeaways) notes that the backward pass recomputes the attention
 * matrix from the inputs instead of storing it.  With the forward's LSE,
 * P_ij = exp(scale * q_i.k_j - LSE_i) over the visible keys, D_i = dO_i . O_i
 * and dS_ij = P_ij * (dO_i . v_j - D_i):
 *
 *   dq_i = scale * sum_j dS_ij k_j
 *   dk_j = scale * sum_i dS_ij q_i   (summed over the query heads of j's group)
 *   dv_j = sum_i P_ij dO_i           (likewise)
 *
 *   q, o, d_o, dq [B, Hq, Sq, d] bf16     k, v, dk, dv [B, Hkv, Skv, d] bf16
 *   lse           [B, Hq, Sq] fp32 (natural log, as fa_fwd writes it)
 *   workspace     fa_bwd_workspace_bytes(B, Hq, Sq, d) bytes, 16-byte aligned,
 *                 caller-owned scratch (per 128-row query tile, -LSE*log2(e)
 *                 and D = dO . O of each row, fp32); its contents on entry
 *                 do not matter
 *   causal, scale: as passed to fa_fwd.
 *
 * dq, dk, dv are written once each (dk = dv = 0 for keys no query sees, dq = 0
 * for queries that see no key) by one kernel with two kinds of CTA: one per
 * key tile for dk, dv and one per query tile for dq, each accumulating in
 * tensor memory, so the result does not depend on scheduling.  A first,
 * bandwidth-bound kernel writes the workspace; the second is launched with
 * programmatic stream serialisation, so its setup and its loads of q, k, v,
 * d_o overlap the first's end, and it reads the workspace only after the
 * first has completed.  P and dS enter the tensor-core products as bf16;
 * accumulation is fp32.
 * Supported: d in {64, 128}; Hq % Hkv == 0.  All pointers 16-byte aligned;
 * dq, dk, dv and workspace must not overlap the inputs or one another.
 * k, v, dk, dv may be null when Skv = 0, and q, o, lse, d_o, dq, workspace
 * when Sq = 0.  Errors as for fa_fwd.
 */
fa_status fa_bwd(const void *q, const void *k, const void *v, const void *o,
                 const float *lse, const void *d_o, void *dq, void *dk, void *dv,
                 float *workspace, int B, int Hq, int Hkv, int Sq, int Skv, int d,
                 int causal, float scale, fa_stream_t stream);

/* Bytes of scratch fa_bwd needs: B * Hq * ceil(Sq / 128) * 256 floats (0 for
 * empty); d is unused. */
size_t fa_bwd_workspace_bytes(int B, int Hq, int Sq, int d);

/*
 * fa_bpt_ffn -- the feed-forward network after attention, run blockwise
 * ("I/O-Aware Kernels", section "Blockwise Parallel Transformers": the
 * network acts on each token alone, so it runs on blocks of query rows and
 * only one block's activations are materialised).  The page fixes no network;
 * this call defines it:
 *
 *   x_t = (o[b,0,t,:], ..., o[b,Hq-1,t,:])       (concatenation over heads, D = Hq*d)
 *   y[b,t,:] = W2 gelu(W1 x_t)                    (gelu(h) = h/2 (1 + erf(h/sqrt 2)))
 *
 *   o   [B, Hq, S, d] bf16 (an attention output, as fa_fwd writes it)
 *   w1  [F, D] bf16, w2 [D, F] bf16 (row-major; no biases)
 *   y   [B, S, D] bf16 (written)
 *   workspace  fa_bpt_workspace_bytes(F, chunk_tiles) bytes, caller-owned
 *
 * The query rows are taken in chunks of chunk_tiles tiles of 128 rows (over
 * all sequences, in order).  Per chunk, one launch writes the chunk's hidden
 * activations gelu(X W1^T) to the workspace (chunk_tiles * 128 * F bf16) and
 * a second writes Y = H W2^T.  So the F-wide activations exist for one chunk
 * at a time; chunk_tiles trades that memory against launches.  Both products
 * run on the tensor cores with fp32 accumulation; H and y are rounded to
 * bf16 once each.
 *
 * Supported: d in {64, 128}; D and F multiples of 256; chunk_tiles in
 * [1, 65535].  Pointers 16-byte aligned.  B == 0 or S == 0 is a no-op.
 * Errors as for fa_fwd (FA_ERR_UNSUPPORTED for other sizes).
 */
fa_status fa_bpt_ffn(const void *o, const void *w1, const void *w2, void *y, void *workspace,
                     int B, int Hq, int S, int d, int F, int chunk_tiles, fa_stream_t stream);

/* Bytes of scratch fa_bpt_ffn needs: chunk_tiles * 128 * F bf16 values. */
size_t fa_bpt_workspace_bytes(int F, int chunk_tiles);

/*
 * fa_bpt_layer -- attention and the feed-forward network after it, run block
 * by block ("I/O-Aware Kernels", section "Blockwise Parallel Transformers":
 * a block of query rows goes through the network as soon as its attention
 * output exists, so no sequence-wide activation is ever materialised).
 *
 * For each chunk of chunk_tiles query tiles (rows [c*R, c*R + R) of every
 * sequence and head, R = chunk_tiles * 128), in order:
 *   1. the attention of those rows (as fa_fwd computes them) into a chunk
 *      buffer of the workspace, their LSE into lse;
 *   2. H = gelu(X W1^T) of the chunk's tokens into the workspace;
 *   3. y at those tokens = H W2^T.
 * So the attention output and the F-wide activations exist for one chunk at a
 * time: the workspace is B*Hq*R*d + B*R*F bf16 values, against B*S*Hq*d +
 * B*S*F when the attention runs over the whole sequence first.
 *
 *   q [B,Hq,S,d], k, v [B,Hkv,S,d] bf16 (self-attention: Sq = Skv = S)
 *   w1 [F, D], w2 [D, F] bf16 with D = Hq*d (as fa_bpt_ffn)
 *   y  [B, S, D] bf16 (written: the network's output per token)
 *   lse [B, Hq, S] fp32 (written: the attention's LSE, as fa_fwd)
 *   workspace  fa_bpt_layer_workspace_bytes(B, Hq, d, F, chunk_tiles) bytes,
 *              caller-owned scratch; contents on entry do not matter
 *   causal, scale: as for fa_fwd.  chunk_tiles >= 1 (larger than the
 *              sequence's tile count means one chunk).
 *
 * y equals fa_bpt_ffn applied to fa_fwd's output, bit for bit: every query
 * tile's attention and every token's network are computed by the same
 * kernels with the same arithmetic whatever the chunking.
 * Supported: d in {64, 128}; D and F multiples of 256; B * chunk_tiles
 * <= 65535.  Pointers 16-byte aligned.  Errors as for fa_fwd and fa_bpt_ffn.
 */
fa_status fa_bpt_layer(const void *q, const void *k, const void *v, const void *w1,
                       const void *w2, void *y, float *lse, void *workspace, int B, int Hq,
                       int Hkv, int S, int d, int F, int causal, float scale, int chunk_tiles,
                       fa_stream_t stream);

/* Bytes of scratch fa_bpt_layer needs (0 for invalid sizes). */
size_t fa_bpt_layer_workspace_bytes(int B, int Hq, int d, int F, int chunk_tiles);

/*
 * fa_decode_splitkv -- first half of single-query decode (Sq = 1, no mask).
 *
 * The key/value length L_b = seqlens_k[b] of sequence b is cut into
 * num_splits chunks of cs = ceil(L_b / num_splits) keys; chunk c covers keys
 * [c*cs, min(L_b, (c+1)*cs)).  For every (b, query head h, chunk c) the call
 * writes the chunk's normalised partial output and its log-sum-exp:
 *
 *   o_partial[b,h,c,:] = softmax over the chunk's keys, times their values
 *   lse_partial[b,h,c] = ln sum over the chunk's keys of exp(scale * q.k)
 *
 * An empty chunk writes o_partial = 0 and lse_partial = -inf.  Cache
 * positions >= L_b never contribute to any output, but they may be read:
 * a chunk's last key tile is fetched in boxes of 32 rows, so up to 31 rows
 * past the chunk's end (still inside the cache's Lmax rows) can be loaded
 * and are then zeroed or masked on chip.
 *
 *   q            [B, Hq, d]           bf16
 *   k_cache,
 *   v_cache      [B, Hkv, Lmax, d]    bf16
 *   seqlens_k    [B]                  int32, device (4-byte aligned), 0 <= L_b <= Lmax
 *                                     (values outside that range are clamped)
 *   o_partial    [B, Hq, num_splits, d] fp32 (written; caller-owned scratch)
 *   lse_partial  [B, Hq, num_splits]    fp32 (written; caller-owned scratch)
 *
 * Supported: d in {64, 128}; Hq / Hkv in {1, 2, 4, 8}; 1 <= num_splits <= 256;
 * scale >= 0 (as for fa_fwd; a negative scale is FA_ERR_UNSUPPORTED).
 */
fa_status fa_decode_splitkv(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *seqlens_k, float *o_partial,
                            float *lse_partial, int B, int Hq, int Hkv, int Lmax,
                            int d, int num_splits, float scale, fa_stream_t stream);

/*
 * fa_decode_paged_splitkv -- fa_decode_splitkv over a paged key/value cache.
 *
 * "I/O-Aware Kernels", section "FlashAttention", names paged KV management
 * (PagedAttention) as what inference kernels built on FlashAttention read
 * from; the pages fix no layout.  Here the cache is a pool of fixed-size
 * pages and each sequence owns a row of a block table: key t of sequence b
 * (and its value) is row t % page_size of physical page
 * block_table[b, t / page_size].
 *
 *   q            [B, Hq, d]                           bf16
 *   k_pages,
 *   v_pages      [num_pages, Hkv, page_size, d]       bf16 (a page holds every
 *                                                     key/value head's rows)
 *   block_table  [B, max_pages]   int32, device (4-byte aligned); entries
 *                t / page_size for t < L_b must name pages in [0, num_pages);
 *                later entries are never read
 *   seqlens_k    [B]  int32, device; 0 <= L_b <= max_pages * page_size
 *                (values outside that range are clamped)
 *   o_partial    [B, Hq, num_splits, d] fp32 (written; caller-owned scratch)
 *   lse_partial  [B, Hq, num_splits]    fp32 (written; caller-owned scratch)
 *
 * Chunks differ from fa_decode_splitkv in one way: the chunk size
 * ceil(L_b / num_splits) is rounded up to a multiple of 128, so chunk c covers
 * keys [c*cs, min(L_b, (c+1)*cs)) with cs = 128 * ceil(ceil(L_b/num_splits)/128)
 * (key tiles then start on tile boundaries and never straddle pages).  Chunks
 * past L_b are empty (o_partial = 0, lse_partial = -inf); fa_combine merges
 * the partials exactly as for the contiguous cache.  Rows of a page past L_b
 * may be read but never contribute.  An out-of-range page index reads zeros
 * or another page (never outside the cache), so the result is then
 * meaningless but memory stays safe.
 *
 * Supported: page_size a power of two in [16, 256]; d in {64, 128};
 * Hq / Hkv in {1, 2, 4, 8}; 1 <= num_splits <= 256.  Errors as for
 * fa_decode_splitkv; FA_ERR_UNSUPPORTED for another page size.
 */
fa_status fa_decode_paged_splitkv(const void *q, const void *k_pages, const void *v_pages,
                                  const int32_t *block_table, const int32_t *seqlens_k,
                                  float *o_partial, float *lse_partial, int B, int Hq,
                                  int Hkv, int num_pages, int page_size, int max_pages,
                                  int d, int num_splits, float scale, fa_stream_t stream);

/*
 * fa_combine -- second half of decode: merge split partials by their LSE.
 *
 * With M = max_c lse_partial[b,h,c]:
 *   lse[b,h] = M + ln sum_c exp(lse_partial[b,h,c] - M)
 *   o[b,h,:] = sum_c exp(lse_partial[b,h,c] - lse[b,h]) * o_partial[b,h,c,:]
 * which is the online softmax's e^(m - m_new) rescale applied between chunks
 * ("FlashAttention & IO-aware attention", section "Direct answer").  All
 * chunks empty gives o = 0, lse = -inf.
 *
 *   o_partial [B, Hq, num_splits, d] fp32,  lse_partial [B, Hq, num_splits] fp32
 *   o         [B, Hq, d] bf16 (written),    lse [B, Hq] fp32 (written)
 *
 * Supported: d in {64, 128}; 1 <= num_splits <= 256.
 */
fa_status fa_combine(const float *o_partial, const float *lse_partial, void *o,
                     float *lse, int B, int Hq, int num_splits, int d,
                     fa_stream_t stream);

/*
 * Host-only helper: a split count for fa_decode_splitkv that gives the GPU's
 * num_sms SMs enough independent chunks.  Never fails; returns >= 1.
 */
int fa_decode_default_splits(int B, int Hkv, int Lmax, int num_sms);

/*
 * Host-only: partition of one fa_fwd / fa_bwd problem over n_shards devices
 * or processes.  The work units are the B * Hkv (batch, key/value head)
 * pairs in row-major order; a unit together with its Hq / Hkv query heads is
 * an attention problem of its own (no query head reads another unit's keys),
 * so the shards need no exchange of data: each computes its units' rows of
 * o and lse, and the union of the shards is the whole result.
 *
 * Shard `shard` (0 <= shard < n_shards) gets units [*first, *first + *count):
 * contiguous, in order, sizes differing by at most one (every unit has the
 * same work).  In the [B * Hkv, Hq / Hkv, S, d] view of q and o and the
 * [B * Hkv, 1, S, d] view of k and v, a shard is one contiguous slice, i.e.
 * one fa_fwd call with B' = *count, Hq' = Hq / Hkv, Hkv' = 1.  A shard may be
 * empty (*count = 0) when n_shards > B * Hkv.
 * Errors: FA_ERR_INVALID_ARG for B, Hkv, n_shards < 1, shard out of range or
 * null outputs.  first and count are host pointers.
 */
fa_status fa_shard_units(int B, int Hkv, int n_shards, int shard, int *first, int *count);

/*
 * Host-only: partition of a decode batch over n_shards devices or processes.
 * Sequences are independent problems; shard s gets sequences
 * [bounds[s], bounds[s+1]), contiguous and in order, chosen so that the
 * shards' key counts (sum of max(L_b, 1) over their sequences, the decode's
 * work) are as even as a contiguous split allows: bounds[s] is the smallest
 * b' such that sequences [0, b') hold at least s / n_shards of the total.
 *   seqlens_k  [B] int32, HOST memory (values < 0 count as 0)
 *   bounds     [n_shards + 1] int32, HOST memory (written; bounds[0] = 0,
 *              bounds[n_shards] = B, non-decreasing)
 * Errors: FA_ERR_INVALID_ARG for B < 1, n_shards < 1 or null pointers.
 */
fa_status fa_shard_sequences(const int32_t *seqlens_k, int B, int n_shards, int32_t *bounds);

/* Host-only: a static, human-readable name for a status code. */
const char *fa_status_string(fa_status s);

/*
 * Reads and clears the device status word of the current device.  Every
 * wait inside the kernels (on an mbarrier) is bounded in time; a kernel whose
 * wait runs out records FA_ERR_DEVICE_TIMEOUT there, drains its own copies,
 * frees its tensor memory and returns instead of hanging.  Synchronises the
 * device.  Returns FA_OK when nothing was recorded.
 */
fa_status fa_get_device_status(void);

/*
 * Test hook for the bounded waits: launches one CTA that waits on an
 * mbarrier nothing will complete, with a time limit of limit_us
 * microseconds, then returns.  The wait must run out, so a following
 * fa_get_device_status() reports FA_ERR_DEVICE_TIMEOUT.  Enqueued on stream.
 */
fa_status fa_debug_timeout_probe(unsigned int limit_us, fa_stream_t stream);

/*
 * Test hook for the backward's CTA order (host only; no CUDA call).  For the
 * backward problem the sizes describe and a device of `sms` SMs, writes the
 * number of CTAs fa_bwd launches to *n_ctas, whether it runs them
 * interleaved by head group (1) or by role (0) to *interleave, and, when
 * tiles is not null, the unit of every CTA in launch order: tiles[4*c ..
 * 4*c+3] = {1 for a dK/dV CTA or 0 for a dQ CTA, batch, kv head (dK/dV) or
 * query head (dQ), key tile (dK/dV) or query tile (dQ)}.  capacity is the
 * number of 4-int entries tiles holds (FA_ERR_INVALID_ARG if fewer than
 * *n_ctas).  Sizes as for fa_bwd with Sq >= 1; d in {64, 128}.
 */
fa_status fa_debug_bwd_tiles(int B, int Hq, int Hkv, int Sq, int Skv, int d, int causal, int sms,
                             int *tiles, long long capacity, long long *n_ctas, int *interleave);

/*
 * Test hook for the polynomial 2^x that the prefill kernel evaluates on the
 * FMA pipe for part of its softmax (the rest uses the hardware exp2):
 * y[i] = 2^n * p(x[i] - n), n = round(x[i]), p the degree-3 minimax fit of
 * 2^f on [-1/2, 1/2] (arguments clamped to >= -126).  x and y are device
 * arrays of n floats (16-byte aligned); n >= 0.  Enqueued on stream.
 */
fa_status fa_debug_exp2_poly(const float *x, float *y, int n, fa_stream_t stream);

/*
 * fa_decode_noalloc -- single-query decode that allocates nothing.
 *
 * The pages have no counterpart to this call.  It computes exactly what
 * fa_decode_splitkv followed by fa_combine computes, with the same arguments
 * and the same meaning of q, k_cache, v_cache, seqlens_k, o and lse, but the
 * split partials live in a fixed array inside the library instead of a
 * buffer from the caller.  It is meant for callers that can neither call
 * cudaMalloc nor hand the library a workspace: a plugin whose host framework
 * owns every device allocation and passes an op nothing but its own tensors,
 * or a serving loop that must not allocate once it runs, because cudaMalloc
 * can synchronise the device and stall all of its streams.
 *
 * Limits and behaviour:
 *  - The array is FA_DECODE_NOALLOC_BYTES (32 MiB) on every device that loads
 *    libfa.so, held until the process exits.  The partials need
 *    B*Hq*num_splits*d*4 bytes, rounded up to 256, plus B*Hq*num_splits*4; a
 *    call that needs more returns FA_ERR_UNSUPPORTED before any CUDA call
 *    (use fewer splits, or fa_decode_splitkv with a caller buffer).
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and keeps it for the
 *    life of the process; make that first call before any stream capture.
 *    The kept address belongs to the device's primary context: after
 *    cudaDeviceReset, or with another context current on that device, it is
 *    stale and this call must not be used.  No call allocates device or host
 *    memory: no cudaMalloc, no cudaFree, no allocating library routine.
 *  - If the split kernel gives up a bounded wait, the merge may combine the
 *    previous call's partials still held in the array, so o and lse are
 *    undefined unless fa_get_device_status() returns FA_OK.
 *  - All calls on a device share the one array, which keeps the previous
 *    call's partials.  Calls whose kernels overlap on the GPU (other streams,
 *    other host threads) race on it; order them on one stream.  Nothing in it
 *    needs to start at zero: every partial the merge reads is written first.
 *  - Supported shapes and the other errors are those of fa_decode_splitkv and
 *    fa_combine.
 */
/* Size in bytes of fa_decode_noalloc's fixed partials array, per device. */
#define FA_DECODE_NOALLOC_BYTES (32u << 20)

fa_status fa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *seqlens_k, void *o, float *lse, int B, int Hq,
                            int Hkv, int Lmax, int d, int num_splits, float scale,
                            fa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
