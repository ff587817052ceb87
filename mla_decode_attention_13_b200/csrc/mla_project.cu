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
// per head and product); a decode step has few tokens (16 to a few hundred),
// so they are bound by memory.  The weight rows are the MMA's M and the tokens
// its N (N = the token box, a multiple of 16), so a short token list costs no
// padded MMA rows, each TMEM lane holds one output dimension, and a warp
// stores 32 consecutive dimensions of a token (64 bytes) per instruction.
//   * absorb: one CTA per (head, 128-row chunk of W_UK^h, tile of up to 128
//     tokens): one M = 128 product of the chunk (K-major, 32 KB) with the
//     tokens' q_nope (K-major), 8 K steps.  Small CTAs (32 KB + the token box)
//     let several share an SM, the next launch's included.
//   * up-project: one CTA per (head, tile of up to 64 tokens): one M = 128
//     product over K = 512: A = W_UV^h seen as 128 value dims x 512 latent
//     dims (MN-major: the value dim is contiguous in memory), B = the tokens'
//     latent output (K-major), in four 128-deep K chunks, each with a barrier
//     of its own, all in flight at once, each chunk's MMAs issued as it lands.
// Shared memory is sized by the token box, and TMEM is read out 16 columns at
// a time so that both kernels fit in 64 registers a thread: up to five absorb
// CTAs (at 16 tokens) share an SM, which leaves room for the next launch's
// CTAs to start early.  Before waiting for the previous
// kernel on the stream (programmatic dependent launch) each CTA asks L2 to
// fetch its weights, which no kernel of the decode writes; a prefetch is only
// a hint and L2 is the point of coherence, so it cannot return stale data.  One
// thread issues the TMA loads and the MMAs; four warps read TMEM out.  Every
// wait is bounded by %globaltimer; on expiry the kernel raises
// MLA_DEVERR_TIMEOUT in this file's sticky error word (taken with the decode
// kernel's by mla_take_device_errors), skips the affected stores, waits for
// its copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "mla_layer.h"
#include "sm100_ptx.cuh"

namespace mla {

__device__ unsigned int g_mla_project_sticky_error;

namespace {

using namespace ptx;

constexpr int kProjThreads = 128;
constexpr uint64_t kProjTimeoutNs = 1000ull * 1000ull * 1000ull;
constexpr int kChunks = 4;                      // 128-row weight chunks per head
constexpr uint32_t kWChunk = 128 * 256;         // 128 rows x 128 bf16 columns: 32 KB
constexpr uint32_t kAMajorMN = 1u << 15;        // instruction descriptor: A is MN-major

// Shared memory (sized by the token box nb at launch), then barriers:
//   absorb:     one 32 KB chunk of W_UK^h, then q_nope (2 panels x nb rows x 128 B)
//   up-project: 4 x 32 KB of W_UV^h, then 4 chunks of the latent output
//               (2 panels x nb rows x 128 B each)
constexpr uint32_t kAbsTokens = kProjAbsorbTile;
constexpr uint32_t kUpTokens = kProjUpTile;
constexpr uint32_t kBarBytes = 128;
__host__ __device__ constexpr uint32_t absorb_bar_offset(int nb) { return kWChunk + 2u * nb * 128u; }
__host__ __device__ constexpr uint32_t up_bar_offset(int nb) { return kChunks * kWChunk + kChunks * 2u * nb * 128u; }
__host__ __device__ constexpr uint32_t absorb_smem(int nb) { return absorb_bar_offset(nb) + kBarBytes + 1024; }
__host__ __device__ constexpr uint32_t up_smem(int nb) { return up_bar_offset(nb) + kBarBytes + 1024; }
static_assert(absorb_smem(kProjAbsorbTile) <= 227 * 1024 && up_smem(kProjUpTile) <= 227 * 1024, "shared memory");

// Barrier words (byte offsets from the barrier area): w[c] at 8c (data of
// chunk c; absorb uses w[0]), accumulator ready at 40, final drain at 72;
// TMEM address at 80; ok flag at 84.
constexpr uint32_t kBW = 0, kBD = 40, kBFin = 72, kTmemSlot = 80, kOkFlag = 84;

// Ask L2 to fetch [ptr, ptr + bytes) from memory (no shared-memory write).
__device__ __forceinline__ void prefetch_l2(const void* ptr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(bytes) : "memory");
}

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

// Width of one accumulator of nb token columns: nb rounded up to 32 (the
// smallest TMEM allocation); the read-out's 16-column loads stay inside it.
__device__ __forceinline__ uint32_t slot_width(int nb) { return (static_cast<uint32_t>(nb) + 31u) & ~31u; }

// TMEM columns to allocate for `slots` accumulators: a power of two from 32 to
// 512 (4 x 128 at most).
__device__ __forceinline__ uint32_t tmem_cols(int slots, int nb) {
  const uint32_t need = static_cast<uint32_t>(slots) * slot_width(nb);
  uint32_t c = 32;
  while (c < need) c <<= 1;
  return c;
}

// Each thread of the warp reads its own lane, 16 consecutive fp32 columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Four warps, one output dimension per thread (its TMEM lane): columns
// [j0, j0 + 16) of the accumulator at `taddr` are the tile's tokens j0 + j;
// token j is stored as bf16 at dst + j * row_stride, for j below `count`.
__device__ __forceinline__ void store_tokens16(uint32_t taddr, __nv_bfloat16* dst, long long row_stride, int j0,
                                               int count) {
  float v[16];
  tmem_ld16(taddr, v);
  tmem_wait_ld();
  __nv_bfloat16* d = dst + static_cast<long long>(j0) * row_stride;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if (j0 + j < count) *d = __float2bfloat16_rn(v[j]);
    d += row_stride;
  }
}

struct ProjSmem {
  uint32_t base;   // 1024-aligned shared address
  uint8_t* gbase;  // the same, generic
};

__device__ __forceinline__ ProjSmem proj_smem() {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  ProjSmem s;
  s.base = (raw + 1023u) & ~1023u;
  s.gbase = smem_raw + (s.base - raw);
  return s;
}

__global__ void __launch_bounds__(kProjThreads, 8) mla_absorb_kernel(const __grid_constant__ ProjParams p) {
  const ProjSmem sm = proj_smem();
  const uint32_t base = sm.base;
  const int h = blockIdx.x >> 2, c = blockIdx.x & 3;  // head, 128-row chunk of W_UK^h
  const int t0 = blockIdx.y * kAbsTokens;
  const int nb = p.nb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t q_smem = base + kWChunk;
  const uint32_t bar_area = absorb_bar_offset(nb);
  const uint32_t bars = base + bar_area;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sm.gbase + bar_area + kTmemSlot);
  volatile uint32_t* ok_flag = reinterpret_cast<volatile uint32_t*>(sm.gbase + bar_area + kOkFlag);
  const uint32_t ncols = tmem_cols(1, nb);
  const char* w_chunk = static_cast<const char*>(p.w) + (static_cast<size_t>(h) * kDv + c * 128) * 256;
  if (threadIdx.x == 0) {
    mbar_init(bars + kBW, 1);
    mbar_init(bars + kBD, 1);
    mbar_init(bars + kBFin, 1);
    *ok_flag = 1u;
    fence_mbar_init_cluster();
    // Before the dependency wait: a prefetch only warms L2, the point of
    // coherence, so it cannot return stale data whatever runs before.
    prefetch_l2(w_chunk, kWChunk);
  }
  if (warp == 0) {
    tmem_alloc(bars + kTmemSlot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();
  griddep_wait();  // q_nope may come from the previous kernel on the stream

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bars + kBW, kWChunk + 2u * nb * 128u);
    tma_load_3d(base, &p.tm_b, bars + kBW, 0, h * kDv + c * 128, 0);  // W_UK^h rows [128 c, +128): 2 panels
    tma_load_4d(q_smem, &p.tm_a, bars + kBW, 0, t0, 0, h);            // q_nope: 2 panels x nb tokens
    const uint32_t idesc = idesc_bf16_f32(128, static_cast<uint32_t>(nb), false);
    if (wait_proj(bars + kBW, 0)) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t a = smem_desc(base + (ks >> 2) * (128 * 128) + (ks & 3) * 32, 16, 1024, kSwizzle128B);
        const uint64_t b = smem_desc(q_smem + (ks >> 2) * (nb * 128) + (ks & 3) * 32, 16, 1024, kSwizzle128B);
        umma_ss(tmem, a, b, idesc, ks > 0 ? 1u : 0u);
      }
    } else {
      *ok_flag = 0u;
      wait_proj(bars + kBW, 0, false);  // drain the copies
    }
    umma_commit(bars + kBD);  // after the MMAs (or at once, with none issued)
  }
  // Every thread sees the issuer's ok flag past here (the accumulator
  // barrier's arrive comes from the tensor core and orders only its results).
  __syncthreads();

  // Read-out: the accumulator holds latent dims [128 c, +128) of the tile's
  // tokens; thread (warp, lane) owns dim 128 c + 32 warp + lane.
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
  const long long row_stride = static_cast<long long>(p.h_q) * kDqk;
  const int count = min(static_cast<int>(kAbsTokens), p.tokens - t0);
  __nv_bfloat16* tile_out = out + static_cast<long long>(t0) * row_stride + static_cast<long long>(h) * kDqk;
  const bool ready = __all_sync(0xffffffffu, wait_proj(bars + kBD, 0));  // warp-uniform, as the TMEM loads are
  tc_fence_after();
  if (ready && *ok_flag != 0u) {
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * warp) << 16);
    for (int j0 = 0; j0 < nb; j0 += 16)
      store_tokens16(lane_base + j0, tile_out + c * 128 + 32 * warp + lane, row_stride, j0, count);
    // The rope columns pass through (chunk 0's CTA): 16-byte pieces.
    if (c == 0) {
      const __nv_bfloat16* rope = reinterpret_cast<const __nv_bfloat16*>(p.extra);
      for (int k = threadIdx.x; k < count * 8; k += kProjThreads) {
        const long long t = t0 + (k >> 3);
        const uint4 v = reinterpret_cast<const uint4*>(rope + (t * p.h_q + h) * 64)[k & 7];
        reinterpret_cast<uint4*>(out + t * row_stride + static_cast<long long>(h) * kDqk + kDv)[k & 7] = v;
      }
    }
  }

  // Teardown: every MMA done before TMEM is freed.
  if (threadIdx.x == 0) {
    umma_commit(bars + kBFin);
    wait_proj(bars + kBFin, 0, false);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

__global__ void __launch_bounds__(kProjThreads, 4) mla_up_project_kernel(const __grid_constant__ ProjParams p) {
  const ProjSmem sm = proj_smem();
  const uint32_t bar_area = up_bar_offset(p.nb);
  const uint32_t base = sm.base, bars = sm.base + bar_area;
  const int h = blockIdx.x;
  const int t0 = blockIdx.y * kUpTokens;
  const int nb = p.nb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t o_smem = base + kChunks * kWChunk;  // chunk c at o_smem + c * o_chunk
  const uint32_t o_chunk = 2u * nb * 128u;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sm.gbase + bar_area + kTmemSlot);
  volatile uint32_t* ok_flag = reinterpret_cast<volatile uint32_t*>(sm.gbase + bar_area + kOkFlag);
  const uint32_t ncols = tmem_cols(1, nb);
  if (threadIdx.x == 0) {
    for (int c = 0; c < kChunks; ++c) mbar_init(bars + kBW + 8 * c, 1);
    mbar_init(bars + kBD, 1);
    mbar_init(bars + kBFin, 1);
    *ok_flag = 1u;
    fence_mbar_init_cluster();
    // W_UV^h into L2 before the dependency wait (a hint, as in the absorb)
    const char* w_head = static_cast<const char*>(p.w) + static_cast<size_t>(h) * kDv * 256;
    for (int c = 0; c < kChunks; ++c) prefetch_l2(w_head + c * kWChunk, kWChunk);
  }
  if (warp == 0) {
    tmem_alloc(bars + kTmemSlot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();
  griddep_wait();  // the latent output comes from the decode's combine kernel

  if (threadIdx.x == 0) {
    // Chunk c: latent dims [128 c, +128) of W_UV^h (2 panels of 64 value
    // dims x 128 rows) and of the tokens' output (2 panels x nb rows).
    for (int c = 0; c < kChunks; ++c) {
      mbar_arrive_expect_tx(bars + kBW + 8 * c, kWChunk + o_chunk);
      tma_load_3d(base + c * kWChunk, &p.tm_b, bars + kBW + 8 * c, 0, h * kDv + c * 128, 0);
      tma_load_4d(o_smem + c * o_chunk, &p.tm_a, bars + kBW + 8 * c, 0, t0, 2 * c, h);
    }
    const uint32_t idesc = idesc_bf16_f32(128, static_cast<uint32_t>(nb), false) | kAMajorMN;
    bool good = true;
    int landed = 0;
    for (int c = 0; c < kChunks && good; ++c) {
      good = wait_proj(bars + kBW + 8 * c, 0);
      if (!good) break;
      landed = c + 1;
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        // MN-major A: 16 latent rows of both 64-value-dim panels (leading
        // byte offset = one panel of 128 rows)
        const uint64_t a = smem_desc(base + c * kWChunk + ks * 16 * 128, 128 * 128, 1024, kSwizzle128B);
        const uint64_t b = smem_desc(o_smem + c * o_chunk + (ks >> 2) * (nb * 128) + (ks & 3) * 32, 16, 1024,
                                     kSwizzle128B);
        umma_ss(tmem, a, b, idesc, (c > 0 || ks > 0) ? 1u : 0u);
      }
    }
    umma_commit(bars + kBD);  // after the last MMA issued (or none)
    if (!good) {
      *ok_flag = 0u;
      for (int c = landed; c < kChunks; ++c) wait_proj(bars + kBW + 8 * c, 0, false);
    }
  }
  __syncthreads();  // the issuer's ok flag, as in the absorb kernel

  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
  const long long row_stride = static_cast<long long>(p.h_q) * 128;
  const int count = min(static_cast<int>(kUpTokens), p.tokens - t0);
  const bool ready = __all_sync(0xffffffffu, wait_proj(bars + kBD, 0));  // warp-uniform, as the TMEM loads are
  tc_fence_after();
  if (ready && *ok_flag != 0u) {
    __nv_bfloat16* dst = out + static_cast<long long>(t0) * row_stride + h * 128 + 32 * warp + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * warp) << 16);
    for (int j0 = 0; j0 < nb; j0 += 16) store_tokens16(lane_base + j0, dst, row_stride, j0, count);
  }

  if (threadIdx.x == 0) {
    umma_commit(bars + kBFin);
    wait_proj(bars + kBFin, 0, false);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

}  // namespace

cudaError_t launch_projection(const ProjParams& p, bool absorb, cudaStream_t stream) {
  const void* fn = absorb ? reinterpret_cast<const void*>(mla_absorb_kernel)
                          : reinterpret_cast<const void*>(mla_up_project_kernel);
  const int smem = static_cast<int>(absorb ? absorb_smem(p.nb) : up_smem(p.nb));
  const int max_smem = static_cast<int>(absorb ? absorb_smem(kProjAbsorbTile) : up_smem(kProjUpTile));
  const int tile = absorb ? kProjAbsorbTile : kProjUpTile;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(absorb ? kChunks * p.h_q : p.h_q),
                     static_cast<unsigned>((p.tokens + tile - 1) / tile), 1);
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

// Self-test of the bounded wait: one thread waits on a barrier that nothing
// arrives at; the wait gives up after its limit, raises MLA_DEVERR_TIMEOUT in
// the sticky word and the kernel returns.
__global__ void mla_wait_selftest_kernel() {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    fence_mbar_init_cluster();
    wait_proj(b, 0);
  }
}

cudaError_t launch_wait_selftest(cudaStream_t stream) {
  mla_wait_selftest_kernel<<<1, 32, 0, stream>>>();
  return cudaGetLastError();
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
