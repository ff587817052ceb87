// Internal layout shared by the host code and the three kernels of the
// decode path: the metadata (tile-scheduler plan) word layout, the workspace
// layout, and the kernels' launch entry points.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "mla_b200.h"

namespace mla {

constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kPage = 64;
constexpr int kMTile = 128;       // query rows per work row (UMMA M)
constexpr int kMaxPairs = 160;    // upper bound on SM pairs of any sm_100 part
constexpr int kMaxHq = 128;
constexpr int kMaxSq = 16;
constexpr int kKappa = 5;         // fixed per-piece cost of the plan, in pages
constexpr uint32_t kMagic = 0x314C4D42u;  // "BML1"

// ---------------------------------------------------------------------------
// Metadata: int32 words.
//   header [kHdrWords]
//   pair_off  [kMaxPairs + 1]           segment range of each pair
//   pair_rec  [kMaxPairs][8]            per pair: its first segment's record
//                                       (words 0-4, as in segs; work row -1 if
//                                       it has none) and its first segment
//                                       index (word 5), so a pair starts from
//                                       one load
//   segs      [W + kMaxPairs][8]        (work row, first page, end page, slot,
//                                       length, 0, 0, 0)
//   row_info  [W][2]                    (first slot or -1, pieces)
//   split_rows [W]                      work rows cut into >1 pieces
//   empty_rows [W]                      work rows with no pages
//   tasks     [W][4]                    per split row: (work row, first slot, pieces, 0),
//                                       so the combine finds a row's pieces in one load
// A work row is (batch row i, m-tile mt) with index w = mt * batch + i.
// ---------------------------------------------------------------------------
enum HeaderWord : int {
  kHMagic = 0,
  kHError = 1,
  kHPairs = 2,
  kHWorkRows = 3,
  kHSegments = 4,
  kHSlots = 5,
  kHRows = 6,      // R = s_q * h_q
  kHMTiles = 7,
  kHBatch = 8,
  kHKappa = 9,
  kHSplitRows = 10,
  kHEmptyRows = 11,
  kHHq = 12,
  kHSq = 13,
  kHCap = 14,
  kHdrWords = 32,
};

constexpr int kSegWords = 8;  // words of a segment record (pair_rec and segs)

struct MetaLayout {
  int W;
  size_t pair_off, pair_rec, segs, row_info, split_rows, empty_rows, tasks, words;
};

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

__host__ __device__ inline MetaLayout meta_layout(int batch, int h_q, int s_q) {
  MetaLayout L;
  L.W = batch * ceil_div(s_q * h_q, kMTile);
  L.pair_off = kHdrWords;
  L.pair_rec = (L.pair_off + kMaxPairs + 1 + 7) & ~size_t(7);
  L.segs = L.pair_rec + size_t(kSegWords) * kMaxPairs;
  L.row_info = L.segs + size_t(kSegWords) * (L.W + kMaxPairs);
  L.split_rows = L.row_info + size_t(2) * L.W;
  L.empty_rows = L.split_rows + L.W;
  L.tasks = (L.empty_rows + L.W + 3) & ~size_t(3);
  L.words = L.tasks + size_t(4) * L.W;
  return L;
}

// Rows of a work row that hold real query rows: min(R, 128).
__host__ __device__ inline int tile_rows(int h_q, int s_q) {
  int R = s_q * h_q;
  return R < kMTile ? R : kMTile;
}

// Workspace: o_part [slots][tile_rows][512] fp32, then lse_part [slots][tile_rows].
// A plan over P pairs cuts rows at most P - 1 times, and every cut row has one
// more piece than cuts, so at most 2 (P - 1) slots are used.
__host__ __device__ inline int max_slots(int pairs) { return pairs > 1 ? 2 * (pairs - 1) : 0; }

__host__ __device__ inline size_t workspace_bytes_for(int pairs, int h_q, int s_q) {
  size_t rows = size_t(max_slots(pairs)) * tile_rows(h_q, s_q);
  return rows * (kDv + 1) * sizeof(float);
}

// ---------------------------------------------------------------------------
// Split-KV decode kernel parameters.
// ---------------------------------------------------------------------------
struct DecodeParams {
  // All three view a [rows][576] bf16 tensor as (64 cols, rows, 9 panels),
  // strides (1152 B, 128 B), so that a 3-D box lands as panels of 64
  // columns x box rows, 128B-swizzled.
  CUtensorMap tm_k;  // cache: box (64, 64, 1), one panel of a page's 64 tokens
  // cache as (64 cols, rows, 4 panels of a 256-column half, 2 halves), strides
  // (1152 B, 128 B, 512 B): box (64, 64, 2, 2) is one CTA's value tile of a
  // page (its 128 columns of each half), panels in [half][panel] order.
  CUtensorMap tm_v;
  CUtensorMap tm_q;  // q: box (64, 64, 9), 64 query rows
  // bf16 out [batch][R][512] as (512 cols, R rows, batch), strides (1024 B,
  // R * 1024 B), 128B-swizzled: box (64, 32, 1) is 32 rows x 64 columns of a
  // work row's output (rows past R are not written).  Unused for fp32 out.
  CUtensorMap tm_out;
  // FP8 cache only (fp8 = 1; tm_k and tm_v unused then):
  //   latent codes [rows][512] u8 as (512 cols, rows), box (64, 64), no
  //   swizzle: 64 codes of a page's 64 tokens;
  //   rope [rows][64] bf16 as (64 cols, rows), box (64, 64), 128B-swizzled.
  CUtensorMap tm_codes;
  CUtensorMap tm_rope;
  //   the same codes as (128 cols, rows, 2 blocks c, 2 halves h), strides
  //   (512 B, 128 B, 256 B): box (128, 64, 1, 2) at (0, y, c, 0) is CTA c's
  //   value columns [256h + 128c, +128) of 64 tokens, [h][token][128].
  CUtensorMap tm_vcodes;
  const uint8_t* codes;    // [rows][512] E4M3 (value tiles are built from it)
  const int8_t* exps;      // [rows]: token scale 2^exp
  int fp8;
  const int32_t* block_table;
  const int32_t* seqlens;
  void* out;               // bf16
  float* lse;
  float* o_part;
  float* lse_part;
  int32_t* meta;
  long long num_pages;
  int max_pages;
  int batch, s_q, h_q, R, n_mt, causal, tile_rows, max_slots;
  int out_f32;             // 1: out is fp32 [batch][s_q][h_q][512] (mla_decode_f32), 0: bf16
  float scale_log2;        // softmax_scale * log2(e)
};

struct CombineParams {
  const int32_t* meta;
  const float* o_part;
  const float* lse_part;
  void* out;
  float* lse;
  int batch, s_q, h_q, R, tile_rows, pairs, max_slots;
  int slices;  // warps per query row (1, 2, 4 or 8), each merging 512 / slices columns
  int out_f32;  // as DecodeParams::out_f32
};

// Launch wrappers (each returns a cudaError_t).
cudaError_t launch_sched(const int32_t* seqlens, int batch, int h_q, int s_q, int pairs, int32_t* meta,
                         cudaStream_t stream);
cudaError_t decode_kernel_prepare();
cudaError_t decode_kernel_pairs(int* pairs);
size_t decode_kernel_smem_bytes(bool fp8);
// Reads and clears (atomically, on `stream`) the device's sticky error bits.
cudaError_t take_sticky_error(cudaStream_t stream, uint32_t* word);
cudaError_t launch_decode(const DecodeParams& p, int pairs, cudaStream_t stream);
cudaError_t launch_combine(const CombineParams& p, int grid, cudaStream_t stream);
// Warps per query row of the combine (CombineParams::slices) for this many
// work rows of tile_rows query rows on a device with `sms` SMs.
int combine_slices(int work_rows, int tile_rows, int sms);

}  // namespace mla
