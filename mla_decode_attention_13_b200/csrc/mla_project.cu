// The projections either side of the absorbed decode, on sm_100a.
//
// "MLA 和 MHA 的 Kernel 区别", sections "内存布局和 KV Cache 大小 / MLA" and
// "MLA 的 FlashAttention": keys and values are up-projections of the cached
// latent, K^h = c W_UK^h and V^h = c W_UV^h.  Moving W_UK^h onto the query and
// W_UV^h onto the output (the absorbed form the decode kernel computes) leaves
// two small products per head around it:
//   absorb:      q~[t][h] = [W_UK^h q_nope[t][h], q_rope[t][h]]    (512 + 64)
//   up-project:  o[t][h]  = o~[t][h] W_UV^h                        (128)
// with W_UK^h and W_UV^h stored [512 latent rows][128 columns] per head.
//
// Both are batched GEMMs over the heads whose bytes are the weights (128 KB
// per head and product) and the tokens' rows; with decode's few tokens per
// head they are bound by memory.  One CTA takes one head and a tile of up to
// 128 tokens: the tokens are the MMA's M (so each TMEM lane holds one token's
// output row, stored whole with 16-byte stores), the head's weight rows its N.
//   * absorb: A = the tokens' q_nope (128 x 128, K-major), B = W_UK^h (512 x
//     128, K-major), D = 128 tokens x 512 fp32 in all 512 TMEM columns, as two
//     N = 256 products over 8 K steps.
//   * up-project: A = the tokens' latent output (128 x 512, K-major), B =
//     W_UV^h (K = 512 rows, N = 128 columns, MN-major), D = 128 x 128 fp32, over
//     32 K steps streamed through two 64 KB stages.
// One thread issues the TMA loads and the MMAs; four warps read TMEM out.  Every
// wait is bounded by %globaltimer; on expiry the kernel raises
// MLA_DEVERR_TIMEOUT in this file's sticky error word (taken with the decode
// kernel's by mla_take_device_errors), waits for its copies, frees TMEM and
// returns without writing.
#include <cuda_bf16.h>

#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {

__device__ unsigned int g_mla_project_sticky_error;

namespace {

using namespace ptx;

constexpr int kProjThreads = 128;
constexpr int kTokTile = 128;
constexpr uint64_t kProjTimeoutNs = 1000ull * 1000ull * 1000ull;

// K-major 128B-swizzled panel of 64 bf16 columns: rows x 128 bytes.
constexpr uint32_t kPanelTok = kTokTile * 128;  // 128 token rows: 16 KB

// absorb: A = 2 panels (K = 128), B = 2 N-halves x 2 panels of 256 rows.
constexpr uint32_t kAbsA = 2 * kPanelTok;          // 32 KB
constexpr uint32_t kAbsBPanel = 256 * 128;         // 32 KB
constexpr uint32_t kAbsB = 4 * kAbsBPanel;         // 128 KB
constexpr uint32_t kAbsBar = kAbsA + kAbsB;
constexpr uint32_t kAbsSmem = kAbsBar + 64 + 1024;

// up-project: 2 stages of (A: 2 panels of 128 tokens, B: 2 column panels of
// 128 latent rows), one stage per 128 latent columns.
constexpr uint32_t kUpStage = 2 * kPanelTok + 2 * (128 * 128);  // 64 KB
constexpr uint32_t kUpBar = 2 * kUpStage;
constexpr uint32_t kUpSmem = kUpBar + 64 + 1024;

constexpr uint32_t kIdescAbs = idesc_bf16_f32(128, 256, false);
constexpr uint32_t kIdescUp = idesc_bf16_f32(128, 128, true);

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int32_t x, int32_t y,
                                            int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Bounded wait on an mbarrier phase: false when it ran out, and then, if
// `raise`, the sticky timeout bit is set (a drain after a failure waits
// quietly).
__device__ bool wait_proj(uint32_t bar, uint32_t parity, bool raise = true) {
  uint64_t t0 = 0;
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++spins & 63u) == 0) {
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kProjTimeoutNs) {
        if (raise) atomicOr(&g_mla_project_sticky_error, MLA_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Four warps, one token per thread: row t of D (its TMEM lane), columns
// [c0, c0 + 32), as bf16 to dst (32 contiguous elements, 16-byte stores).
__device__ __forceinline__ void store_row32(uint32_t taddr, __nv_bfloat16* dst, bool ok) {
  float v[32];
  tmem_ld32(taddr, v);
  tmem_wait_ld();
  if (!ok) return;
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[8 * j + 0], v[8 * j + 1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[8 * j + 2], v[8 * j + 3]);
    __nv_bfloat162 c = __floats2bfloat162_rn(v[8 * j + 4], v[8 * j + 5]);
    __nv_bfloat162 e = __floats2bfloat162_rn(v[8 * j + 6], v[8 * j + 7]);
    uint4 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    u.z = *reinterpret_cast<uint32_t*>(&c);
    u.w = *reinterpret_cast<uint32_t*>(&e);
    d4[j] = u;
  }
}

__global__ void __launch_bounds__(kProjThreads, 1) mla_absorb_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int h = blockIdx.x;
  const int t0 = blockIdx.y * kTokTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_full = base + kAbsBar, bar_done = base + kAbsBar + 8;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + kAbsBar + 16);
  volatile uint32_t* ok_flag = reinterpret_cast<volatile uint32_t*>(gbase + kAbsBar + 20);
  if (threadIdx.x == 0) {
    mbar_init(bar_full, 1);
    mbar_init(bar_done, 1);
    *ok_flag = 1u;
    fence_mbar_init_cluster();
  }
  if (warp == 0) {
    tmem_alloc(base + kAbsBar + 16, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();
  griddep_wait();  // the tokens' q_nope may come from the previous kernel

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar_full, kAbsA + kAbsB);
    tma_load_4d(base, &p.tm_a, bar_full, 0, t0, 0, h);  // q_nope: 2 panels x 128 tokens
#pragma unroll
    for (int nh = 0; nh < 2; ++nh)  // W_UK^h rows [256 nh, +256): 2 panels
      tma_load_3d(base + kAbsA + nh * 2 * kAbsBPanel, &p.tm_b, bar_full, 0, h * 512 + nh * 256, 0);
    bool good = wait_proj(bar_full, 0);
    if (good) {
      tc_fence_after();
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t a = smem_desc(base + (ks >> 2) * kPanelTok + (ks & 3) * 32, 16, 1024, kSwizzle128B);
          const uint64_t b = smem_desc(base + kAbsA + (2 * nh + (ks >> 2)) * kAbsBPanel + (ks & 3) * 32, 16, 1024,
                                       kSwizzle128B);
          umma_ss(tmem + 256 * nh, a, b, kIdescAbs, ks > 0 ? 1u : 0u);
        }
      }
      umma_commit(bar_done);
      if (!wait_proj(bar_done, 0)) {
        good = false;
        wait_proj(bar_done, 0, false);  // drain the MMAs before TMEM is freed
      }
    } else {
      wait_proj(bar_full, 0, false);  // drain the copies before the CTA exits
    }
    if (!good) *ok_flag = 0u;
  }
  __syncthreads();
  tc_fence_after();
  const bool ok = *ok_flag != 0u;
  const int t = t0 + 32 * warp + lane;
  const bool row_ok = ok && t < p.tokens;
  __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + (static_cast<long long>(t) * p.h_q + h) * kDqk;
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * warp) << 16);
  if (ok) {
#pragma unroll 1
    for (int c0 = 0; c0 < 512; c0 += 32) store_row32(lane_addr + c0, orow + c0, row_ok);
    if (row_ok) {  // the rope part passes through
      const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.extra) +
                                                        (static_cast<long long>(t) * p.h_q + h) * 64);
      uint4* dst = reinterpret_cast<uint4*>(orow + 512);
#pragma unroll
      for (int j = 0; j < 8; ++j) dst[j] = src[j];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

__global__ void __launch_bounds__(kProjThreads, 1) mla_up_project_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int h = blockIdx.x;
  const int t0 = blockIdx.y * kTokTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar_full = base + kUpBar, bar_empty = base + kUpBar + 16, bar_done = base + kUpBar + 32;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + kUpBar + 40);
  volatile uint32_t* ok_flag = reinterpret_cast<volatile uint32_t*>(gbase + kUpBar + 44);
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_done, 1);
    *ok_flag = 1u;
    fence_mbar_init_cluster();
  }
  if (warp == 0) {
    tmem_alloc(base + kUpBar + 40, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();
  griddep_wait();  // the latent output comes from the decode (combine) kernel

  if (threadIdx.x == 0) {
    // Stage s holds latent columns [128 c, +128) of chunk c: the tokens' rows
    // (2 panels) and W_UV^h's rows (2 panels of 64 output columns).
    auto load = [&](int c) {
      const int s = c & 1;
      const uint32_t st = base + s * kUpStage;
      mbar_arrive_expect_tx(bar_full + 8 * s, kUpStage);
      tma_load_4d(st, &p.tm_a, bar_full + 8 * s, 0, t0, 2 * c, h);
      tma_load_3d(st + 2 * kPanelTok, &p.tm_b, bar_full + 8 * s, 0, h * 512 + c * 128, 0);
    };
    int issued = 0, landed = 0;  // chunks loaded, chunks whose load was waited for
    load(0);
    load(1);
    issued = 2;
    bool good = true;
    for (int c = 0; c < 4 && good; ++c) {
      const int s = c & 1;
      const uint32_t st = base + s * kUpStage;
      good = wait_proj(bar_full + 8 * s, (c >> 1) & 1);
      if (!good) break;
      landed = c + 1;
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t a = smem_desc(st + (ks >> 2) * kPanelTok + (ks & 3) * 32, 16, 1024, kSwizzle128B);
        // MN-major: 16 latent rows of both 64-column panels (leading byte
        // offset = one panel of 128 rows)
        const uint64_t b = smem_desc(st + 2 * kPanelTok + ks * 16 * 128, 128 * 128, 1024, kSwizzle128B);
        umma_ss(tmem, a, b, kIdescUp, (c > 0 || ks > 0) ? 1u : 0u);
      }
      if (c + 2 < 4) {  // refill the stage once this chunk's MMAs are done with it
        umma_commit(bar_empty + 8 * s);
        good = wait_proj(bar_empty + 8 * s, (c >> 1) & 1);
        if (good) {
          load(c + 2);
          issued = c + 3;
        }
      }
    }
    umma_commit(bar_done);  // every MMA issued so far
    if (!wait_proj(bar_done, 0, good)) {
      good = false;
      wait_proj(bar_done, 0, false);
    }
    if (!good)  // drain copies still in flight before the CTA exits
      for (int c = landed; c < issued; ++c) wait_proj(bar_full + 8 * (c & 1), (c >> 1) & 1, false);
    if (!good) *ok_flag = 0u;
  }
  __syncthreads();
  tc_fence_after();
  const bool ok = *ok_flag != 0u;
  const int t = t0 + 32 * warp + lane;
  const bool row_ok = ok && t < p.tokens;
  __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + (static_cast<long long>(t) * p.h_q + h) * 128;
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * warp) << 16);
  if (ok) {
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) store_row32(lane_addr + c0, orow + c0, row_ok);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace

cudaError_t launch_projection(const ProjParams& p, bool absorb, cudaStream_t stream) {
  const void* fn = absorb ? reinterpret_cast<const void*>(mla_absorb_kernel)
                          : reinterpret_cast<const void*>(mla_up_project_kernel);
  const int smem = static_cast<int>(absorb ? kAbsSmem : kUpSmem);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.h_q), static_cast<unsigned>((p.tokens + kTokTile - 1) / kTokTile), 1);
  cfg.blockDim = dim3(kProjThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return absorb ? cudaLaunchKernelEx(&cfg, mla_absorb_kernel, p) : cudaLaunchKernelEx(&cfg, mla_up_project_kernel, p);
}

__device__ unsigned int g_mla_project_taken;

__global__ void take_project_sticky_kernel() {
  g_mla_project_taken = atomicExch(&g_mla_project_sticky_error, 0u);
}

cudaError_t take_project_sticky_error(cudaStream_t stream, uint32_t* word) {
  take_project_sticky_kernel<<<1, 1, 0, stream>>>();
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess)
    e = cudaMemcpyFromSymbolAsync(word, g_mla_project_taken, sizeof(unsigned int), 0, cudaMemcpyDeviceToHost,
                                  stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  return e;
}

}  // namespace mla
