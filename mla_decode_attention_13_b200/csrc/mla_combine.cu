// Log-sum-exp combine of split-KV pieces, and the output of empty rows.
//
// "Unlocking GPU Potential: The Impact of FlashAttention and KV Cache
// Optimization in Long-Text Inference": once long rows are split across SMs,
// the per-piece results must be merged.  Each piece k of a row holds its
// normalised output o_k and lse_k = ln sum_{j in piece} exp(z_j); the merge is
//     lse = ln sum_k exp(lse_k),    out = sum_k exp(lse_k - lse) * o_k,
// computed with the maximum lse_k subtracted first.  Work rows the plan gave
// no pages (L = 0) produce out = 0 and lse = -inf here.
//
// Grid-stride over items (work row, group of 8 query rows); one warp per query
// row, each lane owning 16 of the 512 output columns as 4 float4 strips, so a
// warp reads and writes whole contiguous rows.  Memory-light, CUDA cores.
#include <cuda_bf16.h>

#include "mla_internal.h"

namespace mla {
namespace {

constexpr int kCombineThreads = 256;
constexpr int kRowsPerItem = kCombineThreads / 32;

__global__ void __launch_bounds__(kCombineThreads) mla_combine_kernel(const CombineParams p) {
  const int32_t* meta = p.meta;
  const MetaLayout lo = meta_layout(p.batch, p.h_q, p.s_q);
  // Only a plan built for this call's shape on this many pairs is used.
  if (meta[kHMagic] != static_cast<int32_t>(kMagic) || meta[kHBatch] != p.batch || meta[kHHq] != p.h_q ||
      meta[kHSq] != p.s_q || meta[kHPairs] != p.pairs)
    return;
  const int n_split = meta[kHSplitRows];
  const int n_empty = meta[kHEmptyRows];
  const int W = lo.W;
  if (n_split < 0 || n_split > W || n_empty < 0 || n_empty > W) return;
  const int groups = ceil_div(p.tile_rows, kRowsPerItem);
  const int n_items = (n_split + n_empty) * groups;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int k = item / groups;
    const int grp = item - k * groups;
    const bool empty = k >= n_split;
    const int w = empty ? meta[lo.empty_rows + (k - n_split)] : meta[lo.split_rows + k];
    if (w < 0 || w >= W) continue;
    const int i = w % p.batch;
    const int mt = w / p.batch;
    const int r = grp * kRowsPerItem + warp;
    const int row_g = mt * kMTile + r;
    if (r >= p.tile_rows || row_g >= p.R) continue;
    const int t = row_g / p.h_q;
    const int hh = row_g - t * p.h_q;
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + (static_cast<long long>(i) * p.R + row_g) * kDv;
    float* lse_out = p.lse + (static_cast<long long>(i) * p.h_q + hh) * p.s_q + t;

    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
    float lse = -INFINITY;
    if (!empty) {
      const int base = meta[lo.row_info + 2 * w + 0];
      const int pieces = meta[lo.row_info + 2 * w + 1];
      if (base < 0 || pieces < 2 || base + pieces > p.max_slots) continue;
      float mx = -INFINITY;
      for (int q = lane; q < pieces; q += 32) {
        mx = fmaxf(mx, p.lse_part[static_cast<long long>(base + q) * p.tile_rows + r]);
      }
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (mx != -INFINITY) {
        float sum = 0.0f;
        for (int q = lane; q < pieces; q += 32) {
          sum += __expf(p.lse_part[static_cast<long long>(base + q) * p.tile_rows + r] - mx);
        }
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        lse = mx + __logf(sum);
        for (int q = 0; q < pieces; ++q) {
          const long long slot_row = static_cast<long long>(base + q) * p.tile_rows + r;
          const float wgt = __expf(p.lse_part[slot_row] - lse);
          const float4* src = reinterpret_cast<const float4*>(p.o_part + slot_row * kDv);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float4 v = src[c * 32 + lane];
            acc[4 * c + 0] += wgt * v.x;
            acc[4 * c + 1] += wgt * v.y;
            acc[4 * c + 2] += wgt * v.z;
            acc[4 * c + 3] += wgt * v.w;
          }
        }
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      __nv_bfloat162 a = __floats2bfloat162_rn(acc[4 * c + 0], acc[4 * c + 1]);
      __nv_bfloat162 b = __floats2bfloat162_rn(acc[4 * c + 2], acc[4 * c + 3]);
      uint2 v;
      v.x = *reinterpret_cast<uint32_t*>(&a);
      v.y = *reinterpret_cast<uint32_t*>(&b);
      *reinterpret_cast<uint2*>(orow + (c * 32 + lane) * 4) = v;
    }
    if (lane == 0) *lse_out = lse;
  }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, int grid, cudaStream_t stream) {
  mla_combine_kernel<<<grid, kCombineThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
