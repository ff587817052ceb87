// Log-sum-exp combine of split-KV pieces, and the output of empty rows.
//
// "Unlocking GPU Potential: The Impact of FlashAttention and KV Cache
// Optimization in Long-Text Inference": once long rows are split across SMs,
// the per-piece results must be merged.  Each piece k of a row holds its
// normalised output o_k and lse_k = ln sum_{j in piece} exp(z_j); the merge is
//     lse = ln sum_k exp(lse_k),    out = sum_k exp(lse_k - lse) * o_k,
// computed with the maximum lse_k subtracted first.  Work rows the plan gave
// no pages (L = 0) produce out = 0 and lse = -inf here.  out is bf16, or fp32
// for mla_decode_f32.
//
// Grid-stride over items (work row, query row, slice of the 512 output
// columns); one warp per item.  The host picks the slices per query row (1,
// 2, 4 or 8) from the number of query rows, so that the items fill the GPU:
// many rows take one warp each (fewer, longer dependent chains), few rows (a
// small h_q with one very long, many-piece row) spread each row over up to 8
// warps.  The pieces are merged online: a batch of pieces' lse values and
// rows is loaded with all loads in flight together (the kernel is bound by
// memory latency, not bandwidth), the running maximum moves to the batch's,
// and the running sum and the accumulated row are rescaled by the
// difference, so no pass over the lse values has to come first.  A split
// row's pieces are found from one task record written by the plan.
// Launched as the decode kernel's programmatic dependent: it waits for the
// decode kernel's completion before reading the partials.
#include <cuda_bf16.h>

#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {

#ifdef MLA_DECODE_TRACE
// Profiling builds only: [first block entry, first block past the grid dependency, last block exit] (globaltimer).
__device__ unsigned long long g_mla_comb_times[3];
#endif

namespace {

constexpr int kCombineThreads = 128;
constexpr int kWarpsPerCta = kCombineThreads / 32;

// A lane's share of one piece's slice of a row: 16 / S floats, as float4s
// (S <= 4) spread 32 lanes apart so that each load instruction of the warp
// reads 512 contiguous bytes, or one float2 (S = 8).
template <int S>
struct Slice {
  static constexpr int kFloats = 16 / S;
  static constexpr int kVec = S == 8 ? 2 : 4;
  static constexpr int kNVec = kFloats / kVec;
  static constexpr int kBatch = S < 4 ? 4 * S : 16;  // pieces in flight: up to 64 floats per lane
  // Float offset (within a 512-float row) of the lane's vector j.
  __device__ static int col(int slice, int lane, int j) {
    return slice * (kDv / S) + (j * 32 + lane) * kVec;
  }
  __device__ static void load(const float* row, int slice, int lane, float (&v)[kFloats]) {
#pragma unroll
    for (int j = 0; j < kNVec; ++j) {
      if constexpr (kVec == 4) {
        const float4 x = *reinterpret_cast<const float4*>(row + col(slice, lane, j));
        v[4 * j] = x.x;
        v[4 * j + 1] = x.y;
        v[4 * j + 2] = x.z;
        v[4 * j + 3] = x.w;
      } else {
        const float2 x = *reinterpret_cast<const float2*>(row + col(slice, lane, j));
        v[2 * j] = x.x;
        v[2 * j + 1] = x.y;
      }
    }
  }
  __device__ static void store(__nv_bfloat16* orow, int slice, int lane, const float (&a)[kFloats], float scale) {
#pragma unroll
    for (int j = 0; j < kNVec; ++j) {
      if constexpr (kVec == 4) {
        __nv_bfloat162 x = __floats2bfloat162_rn(a[4 * j] * scale, a[4 * j + 1] * scale);
        __nv_bfloat162 y = __floats2bfloat162_rn(a[4 * j + 2] * scale, a[4 * j + 3] * scale);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t*>(&x);
        u.y = *reinterpret_cast<uint32_t*>(&y);
        *reinterpret_cast<uint2*>(orow + col(slice, lane, j)) = u;
      } else {
        __nv_bfloat162 x = __floats2bfloat162_rn(a[2 * j] * scale, a[2 * j + 1] * scale);
        *reinterpret_cast<__nv_bfloat162*>(orow + col(slice, lane, j)) = x;
      }
    }
  }
  __device__ static void store(float* orow, int slice, int lane, const float (&a)[kFloats], float scale) {
#pragma unroll
    for (int j = 0; j < kNVec; ++j) {
      if constexpr (kVec == 4) {
        *reinterpret_cast<float4*>(orow + col(slice, lane, j)) =
            make_float4(a[4 * j] * scale, a[4 * j + 1] * scale, a[4 * j + 2] * scale, a[4 * j + 3] * scale);
      } else {
        *reinterpret_cast<float2*>(orow + col(slice, lane, j)) = make_float2(a[2 * j] * scale, a[2 * j + 1] * scale);
      }
    }
  }
};

template <int S>
__global__ void __launch_bounds__(kCombineThreads, 4) mla_combine_kernel(const CombineParams p) {
  using Sl = Slice<S>;
  constexpr int kF = Sl::kFloats;
  constexpr int kB = Sl::kBatch;
#ifdef MLA_DECODE_TRACE
  if (threadIdx.x == 0) atomicMin(&g_mla_comb_times[0], ptx::globaltimer());
#endif
  ptx::griddep_launch_dependents();
  // The plan is complete before this grid launches (the decode kernel lets it
  // launch only after its own wait for the plan), so the plan's words and this
  // warp's first task are read now; only the partials wait for the decode
  // kernel's completion.
  const int32_t* meta = p.meta;
  const MetaLayout lo = meta_layout(p.batch, p.h_q, p.s_q);
  // Only a plan built for this call's shape on this many pairs is used.
  const bool plan_ok = meta[kHMagic] == static_cast<int32_t>(kMagic) && meta[kHBatch] == p.batch &&
                       meta[kHHq] == p.h_q && meta[kHSq] == p.s_q && meta[kHPairs] == p.pairs;
  const int n_split = meta[kHSplitRows];
  const int n_empty = meta[kHEmptyRows];
  const int W = lo.W;
  const int per_row = p.tile_rows * S;
  const int lane = threadIdx.x & 31;
  const int warp_g = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int stride = gridDim.x * kWarpsPerCta;
  const bool counts_ok = plan_ok && n_split >= 0 && n_split <= W && n_empty >= 0 && n_empty <= W;
  const int n_items = counts_ok ? (n_split + n_empty) * per_row : 0;
  // A work row's task: (work row, first slot, pieces) for a split row, or the
  // work row alone for an empty one.
  auto task_of = [&](int k) -> int4 {
    if (k < n_split) return *reinterpret_cast<const int4*>(meta + lo.tasks + 4 * k);
    return make_int4(meta[lo.empty_rows + (k - n_split)], 0, 0, 0);
  };
  int4 first_task = make_int4(-1, 0, 0, 0);
  if (warp_g < n_items) first_task = task_of(warp_g / per_row);
  ptx::griddep_wait();  // the decode kernel's partials are complete
#ifdef MLA_DECODE_TRACE
  if (threadIdx.x == 0) atomicMin(&g_mla_comb_times[1], ptx::globaltimer());
#endif

  for (int item = warp_g; item < n_items; item += stride) {
    const int k = item / per_row;
    const int rem = item - k * per_row;
    const int r = rem / S;
    const int slice = rem - r * S;
    const int4 task = item == warp_g ? first_task : task_of(k);
    const int w = task.x, base = task.y, pieces = task.z;
    if (k < n_split && (base < 0 || pieces < 2 || base + pieces > p.max_slots)) continue;
    if (w < 0 || w >= W) continue;
    const int i = w % p.batch;
    const int mt = w / p.batch;
    const int row_g = mt * kMTile + r;
    if (row_g >= p.R) continue;
    const int t = row_g / p.h_q;
    const int hh = row_g - t * p.h_q;
    const long long orow_off = (static_cast<long long>(i) * p.R + row_g) * kDv;

    // Online merge: m = running max of lse_k, s = sum exp(lse_k - m),
    // acc = sum exp(lse_k - m) o_k.
    float acc[kF];
#pragma unroll
    for (int e = 0; e < kF; ++e) acc[e] = 0.0f;
    float m = -INFINITY, s = 0.0f;
    for (int q0 = 0; q0 < pieces; q0 += kB) {
      float lv[kB];
      float v[kB][kF];
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const int q = q0 + b < pieces ? q0 + b : pieces - 1;  // clamp; weight 0 below
        const long long prow = static_cast<long long>(base + q) * p.tile_rows + r;
        lv[b] = p.lse_part[prow];
        Sl::load(p.o_part + prow * kDv, slice, lane, v[b]);
      }
      float mb = -INFINITY;
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        if (q0 + b >= pieces) lv[b] = -INFINITY;
        mb = fmaxf(mb, lv[b]);
      }
      const float m_new = fmaxf(m, mb);
      if (m_new == -INFINITY) continue;  // no piece with a visible token yet
      const float rs = __expf(m - m_new);  // 0 while m is -inf
      s *= rs;
#pragma unroll
      for (int e = 0; e < kF; ++e) acc[e] *= rs;
#pragma unroll
      for (int b = 0; b < kB; ++b) {
        const float wb = __expf(lv[b] - m_new);  // 0 for absent pieces
        s += wb;
#pragma unroll
        for (int e = 0; e < kF; ++e) acc[e] += wb * v[b][e];
      }
      m = m_new;
    }
    const bool any = s > 0.0f;
    if (p.out_f32)
      Sl::store(static_cast<float*>(p.out) + orow_off, slice, lane, acc, any ? 1.0f / s : 0.0f);
    else
      Sl::store(static_cast<__nv_bfloat16*>(p.out) + orow_off, slice, lane, acc, any ? 1.0f / s : 0.0f);
    if (slice == 0 && lane == 0)
      p.lse[(static_cast<long long>(i) * p.h_q + hh) * p.s_q + t] = any ? m + __logf(s) : -INFINITY;
  }
#ifdef MLA_DECODE_TRACE
  __syncthreads();
  if (threadIdx.x == 0) atomicMax(&g_mla_comb_times[2], ptx::globaltimer());
#endif
}

}  // namespace

#ifdef MLA_DECODE_TRACE
extern "C" __attribute__((visibility("default"))) int mla_trace_comb_times(void* host, int clear) {
  cudaError_t e = cudaMemcpyFromSymbol(host, g_mla_comb_times, sizeof(g_mla_comb_times));
  if (e == cudaSuccess && clear) {
    const unsigned long long init[3] = {~0ull, ~0ull, 0ull};
    e = cudaMemcpyToSymbol(g_mla_comb_times, init, sizeof(init));
  }
  return static_cast<int>(e);
}
#endif

// Warps per query row: the largest of 1, 2, 4, 8 whose items (an upper bound:
// every work row split) still fit in the resident warps of one wave.
int combine_slices(int work_rows, int tile_rows, int sms) {
  const long long resident = static_cast<long long>(sms) * 4 * kWarpsPerCta;
  const long long rows = static_cast<long long>(work_rows) * tile_rows;
  int sl = 1;
  while (sl < 8 && rows * sl * 2 <= resident) sl *= 2;
  return sl;
}

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
  switch (p.slices) {
    case 1: return cudaLaunchKernelEx(&cfg, mla_combine_kernel<1>, p);
    case 2: return cudaLaunchKernelEx(&cfg, mla_combine_kernel<2>, p);
    case 4: return cudaLaunchKernelEx(&cfg, mla_combine_kernel<4>, p);
    case 8: return cudaLaunchKernelEx(&cfg, mla_combine_kernel<8>, p);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mla
