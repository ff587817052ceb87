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
// warp reads and writes whole contiguous rows.  Lane q reads piece q's lse
// once; the pieces' rows are then fetched kBatch at a time with all their
// loads in flight together, because the kernel is bound by memory latency,
// not bandwidth.  Launched as the decode kernel's programmatic dependent: it
// waits for the decode kernel's completion before reading the partials.
#include <cuda_bf16.h>

#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kCombineThreads = 256;
constexpr int kRowsPerItem = kCombineThreads / 32;
constexpr int kBatch = 4;  // pieces whose rows are in flight at once

__global__ void __launch_bounds__(kCombineThreads) mla_combine_kernel(const CombineParams p) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // the decode kernel's partials and the plan are complete
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
      if (base < 0 || pieces < 2 || pieces > 32 * 8 || base + pieces > p.max_slots) continue;
      // lse of piece lane + 32 k, held by that lane.
      float lv[8];
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int q = lane + 32 * k;
        lv[k] = q < pieces ? p.lse_part[static_cast<long long>(base + q) * p.tile_rows + r] : -INFINITY;
        mx = fmaxf(mx, lv[k]);
      }
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (mx != -INFINITY) {
        float sum = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) sum += __expf(lv[k] - mx);  // exp(-inf) = 0 for absent pieces
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        lse = mx + __logf(sum);
        float wl[8];  // weight of piece lane + 32 k
#pragma unroll
        for (int k = 0; k < 8; ++k) wl[k] = __expf(lv[k] - lse);
        for (int q0 = 0; q0 < pieces; q0 += kBatch) {
          float4 v[kBatch][4];
#pragma unroll
          for (int b = 0; b < kBatch; ++b) {
            const int q = q0 + b < pieces ? q0 + b : pieces - 1;  // clamp; weight 0 below
            const float4* src =
                reinterpret_cast<const float4*>(p.o_part + (static_cast<long long>(base + q) * p.tile_rows + r) * kDv);
#pragma unroll
            for (int c = 0; c < 4; ++c) v[b][c] = src[c * 32 + lane];
          }
#pragma unroll
          for (int b = 0; b < kBatch; ++b) {
            const int q = q0 + b;
            float wgt = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float wk = __shfl_sync(0xffffffffu, wl[k], q & 31);
              if ((q >> 5) == k) wgt = wk;
            }
            if (q >= pieces) wgt = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              acc[4 * c + 0] += wgt * v[b][c].x;
              acc[4 * c + 1] += wgt * v[b][c].y;
              acc[4 * c + 2] += wgt * v[b][c].z;
              acc[4 * c + 3] += wgt * v[b][c].w;
            }
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kCombineThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mla_combine_kernel, p);
}

}  // namespace mla
