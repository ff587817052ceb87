// Merge of decode results computed over disjoint token ranges of the same
// rows: the multi-GPU split of one long row, where each GPU decodes the pages
// it holds and the (out, lse) pairs are exchanged.
//
// "Unlocking GPU Potential: The Impact of FlashAttention and KV Cache
// Optimization in Long-Text Inference": the flash-decoding scheme splits the
// keys into chunks, attends to each chunk separately and rescales the partial
// results by their log-sum-exp.  Here a split is one GPU's share of a row.  For
// each query row, with splits k = 0..S-1:
//     lse = ln sum_k exp(lse_k)
//     out = sum_k exp(lse_k - lse) * out_k
// computed online in fp32: m' = max(m, lse_k), s <- s e^(m - m') + e^(lse_k - m'),
// acc <- acc e^(m - m') + e^(lse_k - m') out_k; then lse = m + ln s, out = acc / s.
// A split whose lse is -inf (no visible token there) adds nothing; a row with
// no visible token in any split gets out = 0 and lse = -inf.
//
// One warp per query row; each lane holds 16 of the 512 columns (two 16-byte
// loads per split of bf16 partial outputs, four of fp32 ones from
// mla_decode_f32).  The loads of the next split are issued before the current
// one is folded in.
#include <cuda_bf16.h>

#include <cmath>

#include "mla_layer.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kMergeWarps = 8;

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 v = __bfloat1622float2(b[k]);
    f[2 * k] = v.x;
    f[2 * k + 1] = v.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * k], f[2 * k + 1]);
    w[k] = *reinterpret_cast<uint32_t*>(&b);
  }
  return u;
}

// A lane's 16 columns of one split's row: [8 lane, +8) and [256 + 8 lane, +8),
// from bf16 (two 16-byte loads) or fp32 (four) partial outputs.
template <bool kF32>
struct Part {
  uint4 u[kF32 ? 4 : 2];
  __device__ void load(const void* outs, long long row_elem, int lane) {
    if constexpr (kF32) {
      const uint4* b = static_cast<const uint4*>(outs);
      const long long c0 = (row_elem + 8 * lane) / 4, c1 = (row_elem + 256 + 8 * lane) / 4;
      u[0] = b[c0];
      u[1] = b[c0 + 1];
      u[2] = b[c1];
      u[3] = b[c1 + 1];
    } else {
      const uint4* b = static_cast<const uint4*>(outs);
      u[0] = b[(row_elem + 8 * lane) / 8];
      u[1] = b[(row_elem + 256 + 8 * lane) / 8];
    }
  }
  __device__ void unpack(float* f) const {
    if constexpr (kF32) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        f[4 * k] = __uint_as_float(u[k].x);
        f[4 * k + 1] = __uint_as_float(u[k].y);
        f[4 * k + 2] = __uint_as_float(u[k].z);
        f[4 * k + 3] = __uint_as_float(u[k].w);
      }
    } else {
      unpack8(u[0], f);
      unpack8(u[1], f + 8);
    }
  }
};

template <bool kF32>
__global__ void __launch_bounds__(32 * kMergeWarps) mla_merge_kernel(const MergeParams p) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();  // the partial results may come from the previous kernels
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(p.batch) * p.s_q * p.h_q;
  const long long split_stride = rows * kDv;  // elements per split
  const long long lse_split_stride = rows;
  for (long long r = static_cast<long long>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5); r < rows;
       r += static_cast<long long>(gridDim.x) * kMergeWarps) {
    // out rows are [batch][s_q][h_q]; lse is [batch][h_q][s_q]
    const int h = static_cast<int>(r % p.h_q);
    const long long it = r / p.h_q;
    const int t = static_cast<int>(it % p.s_q);
    const long long i = it / p.s_q;
    const long long lse_idx = (i * p.h_q + h) * p.s_q + t;
    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = 0.0f;
    float m = -INFINITY, s = 0.0f;
    Part<kF32> cur;
    cur.load(p.outs, r * kDv, lane);
    float l = p.lses[lse_idx];
    for (int k = 0; k < p.splits; ++k) {
      Part<kF32> nxt = cur;
      float nl = l;
      if (k + 1 < p.splits) {  // next split's loads before this one is folded in
        nxt.load(p.outs, (k + 1) * split_stride + r * kDv, lane);
        nl = p.lses[(k + 1) * lse_split_stride + lse_idx];
      }
      if (l != -INFINITY) {
        const float m2 = fmaxf(m, l);
        const float a = __expf(m - m2);  // 0 when m is -inf
        const float b = __expf(l - m2);
        float f[16];
        cur.unpack(f);
        s = s * a + b;
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c] = acc[c] * a + b * f[c];
        m = m2;
      }
      cur = nxt;
      l = nl;
    }
    uint4* out = static_cast<uint4*>(p.out);
    if (m == -INFINITY) {
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      out[(r * kDv + 8 * lane) / 8] = z;
      out[(r * kDv + 256 + 8 * lane) / 8] = z;
      if (lane == 0) p.lse[lse_idx] = -INFINITY;
    } else {
      const float inv = 1.0f / s;
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[c] *= inv;
      out[(r * kDv + 8 * lane) / 8] = pack8(acc);
      out[(r * kDv + 256 + 8 * lane) / 8] = pack8(acc + 8);
      if (lane == 0) p.lse[lse_idx] = m + logf(s);
    }
  }
}

}  // namespace

cudaError_t launch_merge(const MergeParams& p, int sms, cudaStream_t stream) {
  const long long rows = static_cast<long long>(p.batch) * p.s_q * p.h_q;
  long long blocks = (rows + kMergeWarps - 1) / kMergeWarps;
  const long long cap = 8LL * sms;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(32 * kMergeWarps, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return p.in_f32 ? cudaLaunchKernelEx(&cfg, mla_merge_kernel<true>, p)
                  : cudaLaunchKernelEx(&cfg, mla_merge_kernel<false>, p);
}

}  // namespace mla
