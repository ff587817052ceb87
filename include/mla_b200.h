/*
 * mla_b200.h — C ABI of libmla_b200.so: Multi-head Latent Attention (MLA)
 * decode over a paged, compressed latent KV cache, on one NVIDIA B200
 * (sm_100a).
 *
 * The operation.  "MLA 和 MHA 的 Kernel 区别" (sealessland.top), sections
 * "内存布局和 KV Cache 大小 / MLA" and "Decode 阶段的 HBM 访问模式 / MLA Decode":
 * the cache holds one compressed latent vector per token; a decode step scores
 * the new query against every cached token, applies a softmax and sums the
 * values.  In absorbed form each cached token is one 576-element bf16 row
 * (512 latent dims, then 64 rope dims); each query head is a 576-element row;
 * the score is softmax_scale * <q, k_j> over all 576 dims and the value is the
 * first 512 dims of the same row.  For batch row i, query token t, head h:
 *
 *     z_j  = softmax_scale * <q[i][t][h][:], kv_row(i, j)>,   j visible
 *     lse  = ln sum_j exp(z_j)
 *     out  = sum_j exp(z_j - lse) * kv_row(i, j)[0:512]
 *
 * "FlashMLA overview" (nullthought.net FlashMLA walkthrough): bf16 cache,
 * paged in blocks of 64 tokens, variable-length rows.  Token j of row i lives
 * in page block_table[i][j / 64], slot j % 64.  Visible tokens are j < L_i;
 * with causal = 1 query token t sees j <= L_i - s_q + t (the s_q new tokens
 * are the last s_q cache positions).  A query with no visible token returns
 * out = 0 and lse = -inf.
 *
 * The two calls follow the same page's account of the FlashMLA API
 * ("flash_api.cpp"): a metadata call prepares the tile-scheduler plan once per
 * decode step and is reused for every layer; then the attention call runs once
 * per layer.  Splitting long rows across processors and merging the pieces by
 * log-sum-exp is the flash-decoding scheme of "Unlocking GPU Potential: The
 * Impact of FlashAttention and KV Cache Optimization in Long-Text Inference"
 * (decode has query length 1, so a small batch leaves most SMs idle).
 *
 * Conventions for every function below.
 *   - Pointers marked [device] are CUDA device pointers owned by the caller;
 *     the library never allocates, frees or keeps them.  Tensors are dense
 *     and row-major in the stated shape.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls enqueue work asynchronously and never synchronise the
 *     host, except mla_check_device_error.
 *   - Argument errors are found on the host, before anything is enqueued, and
 *     returned as a negative status.  Errors only the GPU can see (a length
 *     past the block table, a page id outside the pool, a plan that does not
 *     match the call, a wait that ran past its time limit) set bits in an error
 *     word inside `metadata`; the kernels skip the offending work instead of
 *     faulting, and mla_check_device_error reports the word.
 *   - No exception or C++ type crosses the ABI.  The functions are
 *     thread-compatible: concurrent calls must use distinct metadata and
 *     workspace buffers.
 *   - Per device, the library caches the kernels' launch geometry (looked up
 *     on the first call there) and the device address of its fixed scratch
 *     array (mla_decode_noalloc); per host thread, the TMA descriptors of
 *     recently used (pointer, size) pairs.  None of these survive a device
 *     reset (cudaDeviceReset) or the destruction of the device's primary
 *     context: the library must not be used on a device after either.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every int-valued function. */
#define MLA_OK 0
#define MLA_ERR_ARG (-1)         /* NULL pointer, bad size, bad alignment  */
#define MLA_ERR_UNSUPPORTED (-2) /* shape outside what the kernels handle  */
#define MLA_ERR_CUDA (-3)        /* a CUDA runtime or driver call failed   */
#define MLA_ERR_WORKSPACE (-4)   /* workspace smaller than required        */
#define MLA_ERR_DEVICE (-5)      /* the device error word is non-zero      */
#define MLA_ERR_SCRATCH (-6)     /* needs more than the fixed scratch holds */

/* Bits of the device error word (see mla_check_device_error). */
#define MLA_DEVERR_SEQLEN 0x1u   /* L_i < 0 or L_i > 64 * max_pages_per_seq */
#define MLA_DEVERR_PAGE 0x2u     /* block-table entry outside [0, num_pages) */
#define MLA_DEVERR_TIMEOUT 0x4u  /* a bounded wait inside a kernel gave up   */
#define MLA_DEVERR_PLAN 0x8u     /* metadata does not match this call (its
                                    shape, or lengths that changed since it
                                    was built)                               */
#define MLA_DEVERR_FP8_RANGE 0x10u /* mla_decode_fp8: a visible token's scale
                                      exponent outside [-15, 7], or a query
                                      value past the f16 range              */

/* Fixed dimensions of the absorbed cache row and of a page. */
#define MLA_D_QK 576
#define MLA_D_V 512
#define MLA_PAGE 64

/*
 * Bytes of the metadata buffer mla_get_metadata fills for this shape.
 * batch >= 1, 1 <= h_q <= 128, 1 <= s_q <= 16; returns 0 otherwise.
 */
size_t mla_metadata_bytes(int batch, int h_q, int s_q);

/*
 * Bytes of scratch ("workspace") mla_decode needs for this shape on the
 * current CUDA device: the fp32 partial outputs and log-sum-exps of rows that
 * the plan splits across SM pairs.  Returns 0 for an unsupported shape.  When
 * no CUDA device can be queried the bound for the largest supported GPU is
 * returned, which is never too small.
 */
size_t mla_workspace_bytes(int batch, int h_q, int s_q);

/*
 * Number of 2-CTA clusters (SM pairs) the decode kernel runs on the current
 * device; the plan is cut into this many pieces.  Negative status on error.
 */
int mla_num_sm_pairs(void);

/*
 * Build the split-KV tile-scheduler plan for one decode step ("FlashMLA
 * overview", flash_api.cpp: get_mla_metadata).
 *
 *   seqlens   [device] int32 [batch]: cached tokens L_i of each row.
 *   batch, h_q, s_q: as for mla_decode.
 *   metadata  [device] mla_metadata_bytes(batch, h_q, s_q) bytes, 16-byte
 *             aligned; overwritten by the plan, and its error word cleared.
 *
 * One kernel on `stream`; no host synchronisation.  The same metadata serves
 * any number of mla_decode calls (one per layer) with the same seqlens.
 */
int mla_get_metadata(const int32_t* seqlens, int batch, int h_q, int s_q, void* metadata, void* stream);

/*
 * MLA decode ("FlashMLA overview", flash_api.cpp: flash_mla_with_kvcache).
 *
 *   q            [device] bf16 [batch][s_q][h_q][576], 16-byte aligned.
 *   kv_cache     [device] bf16 [num_pages][64][1][576], 16-byte aligned;
 *                one latent-plus-rope row per cached token, h_kv = 1.
 *   num_pages    pages in the pool, 1 <= num_pages <= 2^25.
 *   block_table  [device] int32 [batch][max_pages_per_seq]; entries past a
 *                row's ceil(L_i / 64) pages are never read.
 *   seqlens      [device] int32 [batch], 0 <= L_i <= 64 * max_pages_per_seq;
 *                must hold the values the metadata was built from: the
 *                kernels work from the lengths the plan read, and a length
 *                that differs from them sets MLA_DEVERR_PLAN.
 *   softmax_scale  multiplies <q, k>; finite and >= 0.
 *   causal       0 or 1 (see the header comment).
 *   out          [device] bf16 [batch][s_q][h_q][512], 16-byte aligned.
 *   lse          [device] fp32 [batch][h_q][s_q]: natural log of
 *                sum_j exp(softmax_scale * <q, k_j>).
 *   metadata     [device] from mla_get_metadata for (seqlens, batch, h_q, s_q);
 *                its error word may be set by this call.
 *   workspace    [device] at least mla_workspace_bytes(batch, h_q, s_q)
 *                bytes, 16-byte aligned; workspace_bytes says how many.
 *
 * Enqueues the split-KV decode kernel and the log-sum-exp combine kernel on
 * `stream`.  Supported: 1 <= h_q <= 128, 1 <= s_q <= 16, batch >= 1.
 */
int mla_decode(const void* q, const void* kv_cache, int64_t num_pages, const int32_t* block_table,
               int max_pages_per_seq, const int32_t* seqlens, int batch, int s_q, int h_q, float softmax_scale,
               int causal, void* out, float* lse, void* metadata, void* workspace, size_t workspace_bytes,
               void* stream);

/*
 * mla_decode with an fp32 output: the same attention, with out written as
 * fp32 [batch][s_q][h_q][512] (16-byte aligned) instead of bf16, unrounded.
 * For results that are merged again before they are rounded: the split of
 * one long row across GPUs ("Unlocking GPU Potential: The Impact of
 * FlashAttention and KV Cache Optimization in Long-Text Inference": each
 * chunk of the keys is attended to separately, and the partial results are
 * rescaled by their log-sum-exp), whose per-GPU results go to
 * mla_merge_splits_f32.  Every other argument, the limits and the errors are
 * those of mla_decode.
 */
int mla_decode_f32(const void* q, const void* kv_cache, int64_t num_pages, const int32_t* block_table,
                   int max_pages_per_seq, const int32_t* seqlens, int batch, int s_q, int h_q, float softmax_scale,
                   int causal, float* out, float* lse, void* metadata, void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * MLA decode over an FP8 latent cache.  "MLA 和 MHA 的 Kernel 区别", section
 * "量化友好性": the compressed latent c_KV tolerates FP8 (or INT8) storage,
 * with the dequantisation fused into the load, which halves the bytes a
 * memory-bound decode reads.  The pages fix no format; this call takes:
 *
 *   latent_codes [device] uint8 [num_pages][64][512]: OCP FP8 E4M3 codes of
 *                the 512 latent dims of each cached token (1 sign, 4
 *                exponent bits with bias 7, 3 mantissa bits; largest finite
 *                value 448), 16-byte aligned;
 *   rope         [device] bf16 [num_pages][64][64]: the 64 rope dims, which
 *                are not part of c_KV and stay bf16, 16-byte aligned;
 *   exps         [device] int8 [num_pages][64]: each token's scale exponent
 *                e, 16-byte aligned.
 *
 * Cached token j of a page is the 576-wide row [code_value(latent_codes[j])
 * * 2^exps[j], rope[j]], and the result is mla_decode's over those rows:
 * every other argument, the plan (one mla_get_metadata serves both calls),
 * the outputs and the errors are those of mla_decode.  Every E4M3 value
 * times 2^e with -15 <= e <= 7 is exact in f16; the kernel computes the
 * latent products in f16 (the latent part of q converted to f16, the rope
 * part in bf16) and accumulates in fp32.  A visible token whose exponent is
 * outside [-15, 7], or a query value past the f16 range (|q| >= 65520), sets
 * MLA_DEVERR_FP8_RANGE in the device error word (its results are then not
 * those of the definition); query values below 2^-14 in magnitude keep an
 * absolute precision of 2^-25.
 */
int mla_decode_fp8(const void* q, const void* latent_codes, const void* rope, const int8_t* exps, int64_t num_pages,
                   const int32_t* block_table, int max_pages_per_seq, const int32_t* seqlens, int batch, int s_q,
                   int h_q, float softmax_scale, int causal, void* out, float* lse, void* metadata, void* workspace,
                   size_t workspace_bytes, void* stream);

/* mla_decode_fp8 with events around its split-KV decode kernel, as
   mla_decode_timed. */
int mla_decode_fp8_timed(const void* q, const void* latent_codes, const void* rope, const int8_t* exps,
                         int64_t num_pages, const int32_t* block_table, int max_pages_per_seq, const int32_t* seqlens,
                         int batch, int s_q, int h_q, float softmax_scale, int causal, void* out, float* lse,
                         void* metadata, void* workspace, size_t workspace_bytes, void* stream,
                         void* event_before_decode, void* event_after_decode);

/*
 * mla_decode, plus CUDA events recorded on `stream` immediately before and
 * after the split-KV decode kernel (either may be NULL), so that a caller can
 * time that kernel alone.  The events are cudaEvent_t passed as void*.
 */
int mla_decode_timed(const void* q, const void* kv_cache, int64_t num_pages, const int32_t* block_table,
                     int max_pages_per_seq, const int32_t* seqlens, int batch, int s_q, int h_q,
                     float softmax_scale, int causal, void* out, float* lse, void* metadata, void* workspace,
                     size_t workspace_bytes, void* stream, void* event_before_decode, void* event_after_decode);

/*
 * Size in bytes of the library's fixed, statically allocated scratch buffer
 * used by mla_decode_noalloc: 40 MiB.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (40u * 1024u * 1024u)

/*
 * mla_decode without a caller-supplied workspace, for callers that cannot
 * allocate device memory at the point of the call: code running inside a
 * framework that owns the device allocator, a fixed-footprint inference
 * engine that sizes all its memory before it starts serving, or a capture or
 * replay of a graph whose memory plan is frozen.  None of these can call
 * cudaMalloc (nor ask torch for a tensor) in the decode loop, but all of them
 * can pass the inputs, outputs and metadata they already own.  (The pages
 * this library follows have no counterpart to this call; it only changes
 * where the scratch lives.)
 *
 * Arguments and results are those of mla_decode, without workspace and
 * workspace_bytes.  The scratch that mla_decode takes from the caller (the
 * fp32 partial outputs of rows the plan splits) lives instead in one
 * statically allocated device array of MLA_NOALLOC_SCRATCH_BYTES, which every
 * GPU that loads the library holds until the process exits.
 *
 *   - Returns MLA_ERR_SCRATCH, before enqueueing anything, when this shape
 *     could need more scratch than that (mla_workspace_bytes(batch, h_q, s_q)
 *     > MLA_NOALLOC_SCRATCH_BYTES); then use mla_decode with a workspace.
 *     On B200 every supported shape fits.
 *   - The first call on each device looks up the array's device address (no
 *     allocation); make that first call before any stream capture.
 *   - Nothing in the array needs to start at zero: the decode kernel writes
 *     every partial it assigns before the combine kernel reads it, so the
 *     contents left by an earlier call are never used.
 *   - All calls on a device share the one array: calls whose kernels overlap
 *     on the GPU (different streams, or different host threads, without an
 *     ordering between them) race on it and give wrong results.  Order them
 *     on one stream, or use mla_decode with separate workspaces.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine.
 */
int mla_decode_noalloc(const void* q, const void* kv_cache, int64_t num_pages, const int32_t* block_table,
                       int max_pages_per_seq, const int32_t* seqlens, int batch, int s_q, int h_q,
                       float softmax_scale, int causal, void* out, float* lse, void* metadata, void* stream);

/*
 * The projections either side of the absorbed decode.  "MLA 和 MHA 的 Kernel
 * 区别", section "内存布局和 KV Cache 大小 / MLA": a head's keys and values are
 * up-projections of the cached latent, K^h = c W_UK^h and V^h = c W_UV^h.
 * Since <q_nope^h, c W_UK^h> = <W_UK^h q_nope^h, c> (W_UK^h taken as [512][128]
 * with the latent index first) and sum_j p_j c_j W_UV^h = (sum_j p_j c_j)
 * W_UV^h, both matrices move off the cache: onto the query before the decode
 * (mla_absorb_q) and onto the latent output after it (mla_up_project), which
 * leaves the decode above reading each cached row once.  Both are batched
 * GEMMs over the heads on the tensor cores (fp32 accumulation, bf16 results).
 *
 * mla_absorb_q: for every token t and head h
 *     q_out[t][h][0:512]   = W_UK^h q_nope[t][h]      (sum over 128 columns)
 *     q_out[t][h][512:576] = q_rope[t][h]             (copied)
 * so that q_out is mla_decode's q (t = i * s_q + token).
 *   q_nope  [device] bf16 [tokens][h_q][128].
 *   q_rope  [device] bf16 [tokens][h_q][64].
 *   w_uk    [device] bf16 [h_q][512][128]: w_uk[h][c][n] is W_UK^h's entry for
 *           latent dim c and no-position dim n.
 *   tokens  >= 1 rows of every tensor; at most 65535 * 128.
 *   h_q     1..128.
 *   q_out   [device] bf16 [tokens][h_q][576].
 * Every pointer 16-byte aligned.  Returns MLA_ERR_ARG for a NULL or misaligned
 * pointer or a count below 1, MLA_ERR_UNSUPPORTED for h_q or tokens past the
 * limits, MLA_ERR_UNSUPPORTED / MLA_ERR_CUDA if the device is not sm_100 or a
 * launch failed.  A kernel wait that ran past its time limit leaves q_out
 * unwritten for that head and token tile and sets MLA_DEVERR_TIMEOUT in the
 * bits mla_take_device_errors reports.
 */
int mla_absorb_q(const void* q_nope, const void* q_rope, const void* w_uk, int tokens, int h_q, void* q_out,
                 void* stream);

/*
 * mla_up_project: for every token t and head h
 *     o_out[t][h][v] = sum_c o_latent[t][h][c] * W_UV^h[c][v]
 * where o_latent is mla_decode's out (t = i * s_q + token).
 *   o_latent [device] bf16 [tokens][h_q][512].
 *   w_uv     [device] bf16 [h_q][512][128]: w_uv[h][c][v] is W_UV^h's entry
 *            for latent dim c and value dim v.
 *   h_q      1..128.
 *   o_out    [device] bf16 [tokens][h_q][128].
 * tokens may be at most 65535 * 64 (the kernel's token tiles are 64 wide);
 * the other limits and errors are those of mla_absorb_q.
 */
int mla_up_project(const void* o_latent, const void* w_uv, int tokens, int h_q, void* o_out, void* stream);

/*
 * Merge decode results computed over disjoint token ranges of the same rows:
 * one long row split across GPUs, each decoding (mla_get_metadata and
 * mla_decode on its own cache, block table and lengths) the pages it holds,
 * then exchanging (out, lse).  "Unlocking GPU Potential: The Impact of
 * FlashAttention and KV Cache Optimization in Long-Text Inference": attend to
 * each chunk of the keys separately, then rescale the partial results by
 * their log-sum-exp.  For each query row, over splits k:
 *     lse = ln sum_k exp(lse_k),   out = sum_k exp(lse_k - lse) * out_k
 * in fp32; a split with lse_k = -inf adds nothing, and a row with no visible
 * token in any split gets out = 0, lse = -inf.  The result equals one
 * mla_decode over the union of the ranges when every split saw the query rows'
 * visible tokens of its range (for a causal step: all splits but the one
 * holding the row's last tokens run with causal = 0).
 *   outs   [device] bf16 [splits][batch][s_q][h_q][512]: the splits' `out`,
 *          stacked; 16-byte aligned.
 *   lses   [device] fp32 [splits][batch][h_q][s_q]: the splits' `lse`.
 *   splits >= 1; batch, s_q, h_q as for mla_decode.
 *   out    [device] bf16 [batch][s_q][h_q][512], 16-byte aligned; lse [device]
 *          fp32 [batch][h_q][s_q].  Neither may overlap the inputs.
 * Returns MLA_ERR_ARG for a NULL or misaligned pointer or a count below 1,
 * MLA_ERR_UNSUPPORTED for shapes mla_decode refuses, MLA_ERR_CUDA if the
 * launch failed.  One small kernel; no device error bits.
 */
int mla_merge_splits(const void* outs, const float* lses, int splits, int batch, int s_q, int h_q, void* out,
                     float* lse, void* stream);

/*
 * mla_merge_splits over fp32 partial outputs (mla_decode_f32's `out`): outs
 * is fp32 [splits][batch][s_q][h_q][512], 16-byte aligned; the result `out` is
 * bf16 as for mla_merge_splits, rounded once after the merge.  Arguments,
 * limits and errors as for mla_merge_splits.
 */
int mla_merge_splits_f32(const float* outs, const float* lses, int splits, int batch, int s_q, int h_q, void* out,
                         float* lse, void* stream);

/*
 * Synchronise `stream` and read the device error word from `metadata`.
 * Writes the word to *error_word (if not NULL).  Returns MLA_OK when it is
 * zero, MLA_ERR_DEVICE when not, MLA_ERR_CUDA if the copy or sync failed.
 */
int mla_check_device_error(const void* metadata, void* stream, uint32_t* error_word);

/*
 * The error bits any call raised on the current device since the last
 * mla_take_device_errors, whatever metadata buffer it used (and those of
 * mla_absorb_q and mla_up_project, which have none): unlike the word in
 * `metadata`, which the next mla_get_metadata on that buffer rewrites, these
 * bits stay set until taken.  For callers that replay many steps (a captured
 * graph, a benchmark loop) and check once at the end.  Enqueues an atomic
 * read-and-clear on `stream` (one tiny kernel), synchronises the stream and
 * writes the bits to *error_word (if not NULL).  Returns MLA_OK when they are
 * zero, MLA_ERR_DEVICE when not, MLA_ERR_CUDA if the launch, copy or sync
 * failed.
 */
int mla_take_device_errors(void* stream, uint32_t* error_word);

/*
 * Self-test of the kernels' bounded waits, for failure-detection tests: one
 * tiny kernel waits on a barrier that nothing arrives at, with the limit the
 * projection kernels use (1 s of %globaltimer).  The wait gives up, sets
 * MLA_DEVERR_TIMEOUT in the bits mla_take_device_errors reports, and the
 * kernel returns: no fault, and the context stays usable.  Enqueued on
 * `stream`; returns MLA_OK, or MLA_ERR_UNSUPPORTED / MLA_ERR_CUDA if the
 * device is not sm_100 or the launch failed.
 */
int mla_selftest_bounded_wait(void* stream);

/* Static text for a status code. */
const char* mla_error_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H */
