// Split-KV MLA decode kernel for sm_100a (B200).
//
// What it computes: for every query row (batch row i, query token t, head h)
// the absorbed-form attention over that row's cached latent tokens ("MLA 和
// MHA 的 Kernel 区别", sections "MLA Decode" and "MLA 的 FlashAttention": load
// each latent tile from HBM once, decompress/score it on chip, reuse it for
// every head).  Scores use all 576 dims of a cached row (512 latent + 64
// rope); values are the first 512 dims of the same row, so every cached tile
// is read once and serves as both K and V.
//
// How, per SM pair (one 2-CTA cluster, persistent over the plan's segments):
//   * The 576 columns are split between the two CTAs: CTA c owns latent
//     columns [256c, 256c + 256) and rope columns [512 + 32c, 512 + 32c + 32).
//     Each CTA TMA-loads only its 288 columns of every 64-token page, so each
//     cache byte leaves HBM once.  Pages are gathered through the block table
//     ("FlashMLA overview": paged kvcache, block size 64).
//   * QK^T: each CTA computes a partial S = Q[:, own cols] K[:, own cols]^T on
//     tcgen05 (M = 128 query rows, N = 64 tokens, 18 K-steps of 16) into TMEM.
//     The two partials are exchanged through distributed shared memory
//     (st.async with mbarrier byte counts) and added; both CTAs then hold the
//     same S and run the same online softmax (one thread per query row).
//   * PV: P (bf16, 128 x 64, written to shared memory in the 128-byte swizzled
//     K-major layout) times V (the CTA's 256 latent columns of the same tile,
//     read MN-major) accumulates into O (128 x 256 fp32) in TMEM.  Per SM the
//     TMEM holds O (256 columns) and two S buffers (2 x 64 columns).
//   * Online softmax with a lazy rescale: the running max only moves when a
//     block's max exceeds it by more than kTau (log2 units); O and the running
//     sum are rescaled together, so the result is exact.
//   * A row that the plan splits writes fp32 (O / l, lse) partials to the
//     workspace for the combine kernel; an unsplit row writes bf16 out and lse.
// Warp roles per CTA (256 threads): warp 0 = TMA producer, warp 1 = TMEM
// owner and UMMA issuer, warps 4-7 = softmax + epilogue (one thread per query
// row / TMEM lane), warps 2-3 idle.
//
// Every mbarrier wait is bounded by %globaltimer; on expiry the kernel sets
// MLA_DEVERR_TIMEOUT in the metadata error word, tells the peer CTA to stop,
// drains its own copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

using namespace ptx;

constexpr int kThreads = 256;
constexpr int kStages = 2;
constexpr float kTau = 8.0f;  // lazy-rescale threshold, log2 units
constexpr uint64_t kTimeoutNs = 500ull * 1000ull * 1000ull;

// Shared-memory layout (offsets from a 1024-byte aligned base).
constexpr uint32_t kQPanel = kMTile * 128;                // 128 rows x 64 bf16 (128B swizzle)
constexpr uint32_t kQRope = kMTile * 64;                  // 128 rows x 32 bf16 (64B swizzle)
constexpr uint32_t kQBytes = 4 * kQPanel + kQRope;        // 73728
constexpr uint32_t kKvPanel = kPage * 128;                // 64 tokens x 64 bf16
constexpr uint32_t kKvRope = kPage * 64;                  // 64 tokens x 32 bf16
constexpr uint32_t kStageBytes = 4 * kKvPanel + kKvRope;  // 36864
constexpr uint32_t kPBytes = kMTile * 128;                // 128 rows x 64 bf16
constexpr uint32_t kXBytes = kMTile * 64 * 4;             // 128 rows x 64 fp32
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKv = kOffQ + kQBytes;
constexpr uint32_t kOffP = kOffKv + kStages * kStageBytes;
constexpr uint32_t kOffX = kOffP + kPBytes;
constexpr uint32_t kOffBar = kOffX + kXBytes;
constexpr uint32_t kSmemUsed = kOffBar + 256;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // slack for aligning the base

enum Bar : uint32_t {
  kBarKvFull = 0,   // [2] TMA -> MMA (tx bytes)
  kBarKvEmpty = 2,  // [2] MMA commit -> TMA
  kBarQFull = 4,
  kBarQEmpty = 5,
  kBarSFull = 6,    // [2] MMA commit -> softmax
  kBarSEmpty = 8,   // [2] softmax (4 warps) -> MMA
  kBarPFull = 10,   // softmax (4 warps) -> MMA
  kBarPvDone = 11,  // MMA commit -> softmax
  kBarXFull = 12,   // peer st.async bytes + own expect_tx
  kBarXEmpty = 13,  // peer's 4 softmax warps -> me
  kBarOEmpty = 14,  // softmax (4 warps) -> MMA
  kBarFinal = 15,   // MMA drain at teardown
  kNumBars = 16,
};
constexpr uint32_t kOffTmemSlot = kOffBar + 8 * kNumBars;  // u32
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;           // u32

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 256;

constexpr uint32_t kIdescQK = idesc_bf16_f32(kMTile, kPage, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kMTile, 256, true);

static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Ctx {
  uint32_t base;          // shared::cta address of the aligned base
  uint8_t* gbase;         // generic pointer to the same place
  uint32_t cta, peer;
  uint32_t peer_x, peer_xfull, peer_xempty, peer_abort;
  volatile uint32_t* abort_flag;
  int32_t* meta;
  __device__ uint32_t bar(uint32_t k) const { return base + kOffBar + 8 * k; }
};

__device__ void raise_abort(const Ctx& c, uint32_t err_bits) {
  if (err_bits) atomicOr(reinterpret_cast<unsigned int*>(c.meta + kHError), err_bits);
  *c.abort_flag = 1u;
  st_cluster_u32(c.peer_abort, 1u);
}

// Bounded wait on an mbarrier phase.  Returns false when the kernel is
// aborting (this wait timed out, or another role or the peer CTA gave up).
__device__ bool wait_bar(const Ctx& c, uint32_t bar, uint32_t parity, bool cluster_scope = false) {
  uint32_t spins = 0;
  uint64_t t0 = 0;
  while (true) {
    const bool ok = cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
    if (ok) return true;
    if ((++spins & 127u) == 0) {
      if (*c.abort_flag) return false;
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kTimeoutNs) {
        raise_abort(c, MLA_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

struct Segment {
  int w, b0, b1, slot;
  int i, mt, L;
  bool bad;
};

__device__ __forceinline__ Segment load_segment(const DecodeParams& p, int s) {
  const MetaLayout lo = meta_layout(p.batch, p.h_q, p.s_q);
  const int4 v = *reinterpret_cast<const int4*>(p.meta + lo.segs + 4 * s);
  Segment g;
  g.w = v.x;
  g.b0 = v.y;
  g.b1 = v.z;
  g.slot = v.w;
  if (g.w < 0 || g.w >= p.batch * p.n_mt) {
    g.i = g.mt = g.L = 0;
    g.bad = true;
    return g;
  }
  g.i = g.w % p.batch;
  g.mt = g.w / p.batch;
  g.L = p.seqlens[g.i];
  g.bad = g.L < 0 || g.L > kPage * p.max_pages || g.b1 > ceil_div(g.L, kPage) || g.b0 < 0 || g.b0 >= g.b1 ||
          g.slot >= p.max_slots;
  return g;
}

// ------------------------------------------------------------- producer --
__device__ void producer(const DecodeParams& p, const Ctx& c, int s_begin, int s_end) {
  const uint32_t q_bytes = static_cast<uint32_t>(p.q_box_rows) * (4 * 128 + 64);  // rows x 288 bf16
  uint32_t kv_cnt = 0, seg_it = 0;
  bool ok = true;
  for (int s = s_begin; s < s_end && ok; ++s) {
    const Segment g = load_segment(p, s);
    if (g.bad) continue;
    if (seg_it > 0 && !(ok = wait_bar(c, c.bar(kBarQEmpty), (seg_it - 1) & 1))) break;
    mbar_arrive_expect_tx(c.bar(kBarQFull), q_bytes);
    const int y = g.i * p.R + g.mt * kMTile;
    for (int k = 0; k < 4; ++k)
      tma_load_2d(c.base + kOffQ + k * kQPanel, &p.tm_q_lat, c.bar(kBarQFull), c.cta * 256 + k * 64, y);
    tma_load_2d(c.base + kOffQ + 4 * kQPanel, &p.tm_q_rope, c.bar(kBarQFull), 512 + c.cta * 32, y);
    const int32_t* table = p.block_table + static_cast<long long>(g.i) * p.max_pages;
    for (int blk = g.b0; blk < g.b1; ++blk) {
      const uint32_t stage = kv_cnt & 1;
      if (!(ok = wait_bar(c, c.bar(kBarKvEmpty + stage), ((kv_cnt >> 1) & 1) ^ 1))) break;
      int page = table[blk];
      if (page < 0 || page >= p.num_pages) {
        atomicOr(reinterpret_cast<unsigned int*>(c.meta + kHError), MLA_DEVERR_PAGE);
        page = 0;  // keep the copy inside the pool; the result is flagged
      }
      const uint32_t dst = c.base + kOffKv + stage * kStageBytes;
      mbar_arrive_expect_tx(c.bar(kBarKvFull + stage), kStageBytes);
      for (int k = 0; k < 4; ++k)
        tma_load_2d(dst + k * kKvPanel, &p.tm_kv_lat, c.bar(kBarKvFull + stage), c.cta * 256 + k * 64, page * kPage);
      tma_load_2d(dst + 4 * kKvPanel, &p.tm_kv_rope, c.bar(kBarKvFull + stage), 512 + c.cta * 32, page * kPage);
      ++kv_cnt;
    }
    ++seg_it;
  }
  if (!ok) {
    // Aborting: let the copies already issued land before the CTA can exit.
    for (uint32_t k = 0; k < 2 && k < kv_cnt; ++k) {
      const uint32_t last = kv_cnt - 1 - k;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(c.bar(kBarKvFull + (last & 1)), (last >> 1) & 1) && globaltimer() - t0 < kTimeoutNs) {
      }
    }
    const uint64_t t0 = globaltimer();
    while (seg_it > 0 && !mbar_try_wait(c.bar(kBarQFull), (seg_it - 1) & 1) && globaltimer() - t0 < kTimeoutNs) {
    }
  }
}

// ------------------------------------------------------------------ MMA --
__device__ __forceinline__ void issue_qk(const Ctx& c, uint32_t tmem, uint32_t stage, uint32_t sb) {
  const uint32_t q = c.base + kOffQ;
  const uint32_t kv = c.base + kOffKv + stage * kStageBytes;
  const uint32_t d = tmem + kColS + sb * kPage;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t off = (k & 3) * 32;
    const uint64_t a = smem_desc(q + (k >> 2) * kQPanel + off, 16, 1024, kSwizzle128B);
    const uint64_t b = smem_desc(kv + (k >> 2) * kKvPanel + off, 16, 1024, kSwizzle128B);
    umma_ss(d, a, b, kIdescQK, k > 0 ? 1u : 0u);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint64_t a = smem_desc(q + 4 * kQPanel + k * 32, 16, 512, kSwizzle64B);
    const uint64_t b = smem_desc(kv + 4 * kKvPanel + k * 32, 16, 512, kSwizzle64B);
    umma_ss(d, a, b, kIdescQK, 1u);
  }
}

__device__ void mma_issuer(const DecodeParams& p, const Ctx& c, uint32_t tmem, int s_begin, int s_end) {
  uint32_t kv_cnt = 0, q_cnt = 0, pv_cnt = 0, seg_it = 0;
  for (int s = s_begin; s < s_end; ++s) {
    const Segment g = load_segment(p, s);
    if (g.bad) continue;
    const int n = g.b1 - g.b0;
    if (!wait_bar(c, c.bar(kBarQFull), seg_it & 1)) return;
    tc_fence_after();
    // QK(0)
    {
      const uint32_t stage = kv_cnt & 1, sb = q_cnt & 1;
      if (!wait_bar(c, c.bar(kBarKvFull + stage), (kv_cnt >> 1) & 1)) return;
      if (!wait_bar(c, c.bar(kBarSEmpty + sb), ((q_cnt >> 1) & 1) ^ 1)) return;
      tc_fence_after();
      issue_qk(c, tmem, stage, sb);
      umma_commit(c.bar(kBarSFull + sb));
      ++q_cnt;
    }
    for (int j = 0; j < n; ++j) {
      if (j + 1 < n) {
        const uint32_t kvi = kv_cnt + j + 1;
        const uint32_t stage = kvi & 1, sb = q_cnt & 1;
        if (!wait_bar(c, c.bar(kBarKvFull + stage), (kvi >> 1) & 1)) return;
        if (!wait_bar(c, c.bar(kBarSEmpty + sb), ((q_cnt >> 1) & 1) ^ 1)) return;
        tc_fence_after();
        issue_qk(c, tmem, stage, sb);
        umma_commit(c.bar(kBarSFull + sb));
        ++q_cnt;
      } else {
        umma_commit(c.bar(kBarQEmpty));  // Q no longer read once the last QK is done
      }
      if (!wait_bar(c, c.bar(kBarPFull), pv_cnt & 1)) return;
      if (j == 0 && seg_it > 0 && !wait_bar(c, c.bar(kBarOEmpty), (seg_it - 1) & 1)) return;
      tc_fence_after();
      const uint32_t stage = (kv_cnt + j) & 1;
      const uint32_t pbuf = c.base + kOffP;
      const uint32_t vbuf = c.base + kOffKv + stage * kStageBytes;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t a = smem_desc(pbuf + k * 32, 16, 1024, kSwizzle128B);
        // V: K = 16 tokens starting at token 16k, N = 256 latent columns
        // spread over 4 panels (leading byte offset = panel stride).
        const uint64_t b = smem_desc(vbuf + k * 16 * 128, kKvPanel, 1024, kSwizzle128B);
        umma_ss(tmem + kColO, a, b, kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
      }
      umma_commit(c.bar(kBarKvEmpty + stage));
      umma_commit(c.bar(kBarPvDone));
      ++pv_cnt;
    }
    kv_cnt += n;
    ++seg_it;
  }
}

// -------------------------------------------------------------- softmax --
__device__ void softmax_epilogue(const DecodeParams& p, const Ctx& c, uint32_t tmem, int s_begin, int s_end) {
  const int r = threadIdx.x - 128;       // query row within the tile = TMEM lane
  const int lane = threadIdx.x & 31;
  const uint32_t lane_off = static_cast<uint32_t>(r & ~31) << 16;
  const uint32_t t_s = tmem + lane_off + kColS;
  const uint32_t t_o = tmem + lane_off + kColO;
  float* xbuf = reinterpret_cast<float*>(c.gbase + kOffX);
  const uint32_t my_xfull = c.bar(kBarXFull);
  const uint32_t peer_row = c.peer_x + r * 256;
  uint32_t s_cnt = 0, pv_cnt = 0, x_cnt = 0, blk_cnt = 0;

  for (int s = s_begin; s < s_end; ++s) {
    const Segment g = load_segment(p, s);
    if (g.bad) {
      if (r == 0 && c.cta == 0) atomicOr(reinterpret_cast<unsigned int*>(c.meta + kHError), MLA_DEVERR_SEQLEN);
      continue;
    }
    const int n = g.b1 - g.b0;
    const int row_g = g.mt * kMTile + r;
    const bool row_valid = r < p.tile_rows && row_g < p.R;
    const int t = row_g / p.h_q;
    const int hh = row_g - t * p.h_q;
    int limit = 0;
    if (row_valid) {
      limit = p.causal ? g.L - p.s_q + t + 1 : g.L;
      limit = limit < 0 ? 0 : (limit > g.L ? g.L : limit);
    }
    const int last_page = ceil_div(g.L, kPage) - 1;
    // l: sum of the bf16-rounded weights actually fed to PV (normalises O, so
    // the output is an exact convex combination of those weights); le: the
    // same sum before rounding (gives lse without the bf16 rounding bias).
    float m = -INFINITY, l = 0.0f, le = 0.0f;

    for (int j = 0; j < n; ++j) {
      const int blk = g.b0 + j;
      const uint32_t sb = s_cnt & 1;
      if (!wait_bar(c, c.bar(kBarSFull + sb), (s_cnt >> 1) & 1)) return;
      tc_fence_after();
      float sv[64];
      tmem_ld32(t_s + sb * kPage, *reinterpret_cast<float(*)[32]>(&sv[0]));
      tmem_ld32(t_s + sb * kPage + 32, *reinterpret_cast<float(*)[32]>(&sv[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(c.bar(kBarSEmpty + sb));
      ++s_cnt;

      // ---- exchange the partial S with the peer CTA and add ----
      if (x_cnt > 0 && !wait_bar(c, c.bar(kBarXEmpty), (x_cnt - 1) & 1, true)) return;
      if (r == 0) mbar_arrive_expect_tx(my_xfull, kXBytes);
#pragma unroll
      for (int q4 = 0; q4 < 16; ++q4) {
        const uint32_t dst = peer_row + ((q4 ^ (r & 15)) << 4);
        st_async_v4(dst, c.peer_xfull, sv[4 * q4 + 0], sv[4 * q4 + 1], sv[4 * q4 + 2], sv[4 * q4 + 3]);
      }
      if (!wait_bar(c, my_xfull, x_cnt & 1, true)) return;
      {
        const float4* row = reinterpret_cast<const float4*>(xbuf + r * 64);
#pragma unroll
        for (int q4 = 0; q4 < 16; ++q4) {
          const float4 u = row[q4 ^ (r & 15)];
          sv[4 * q4 + 0] += u.x;
          sv[4 * q4 + 1] += u.y;
          sv[4 * q4 + 2] += u.z;
          sv[4 * q4 + 3] += u.w;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(c.peer_xempty);
      ++x_cnt;

      // ---- mask, online softmax (log2 domain) ----
      int nvalid = limit - blk * kPage;
      nvalid = nvalid < 0 ? 0 : (nvalid > kPage ? kPage : nvalid);
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        const float x = (k < nvalid) ? sv[k] * p.scale_log2 : -INFINITY;
        sv[k] = x;
        mx = fmaxf(mx, x);
      }
      float m_new = m;
      if (mx > m + kTau) m_new = mx;  // also true for the first finite block
      const float alpha = (m_new == m) ? 1.0f : ex2(m - m_new);  // 0 when m was -inf
      const float m_use = (m_new == -INFINITY) ? 0.0f : m_new;
      uint32_t packed[32];
      float psum = 0.0f, esum = 0.0f;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float a = ex2(sv[2 * k] - m_use), b = ex2(sv[2 * k + 1] - m_use);
        esum += a + b;
        const __nv_bfloat162 pr = __floats2bfloat162_rn(a, b);
        const float2 back = __bfloat1622float2(pr);
        psum += back.x + back.y;
        packed[k] = *reinterpret_cast<const uint32_t*>(&pr);
      }
      l = l * alpha + psum;
      le = le * alpha + esum;
      m = m_new;

      // ---- wait for the previous PV: P buffer free, O up to date ----
      if (j > 0) {
        if (!wait_bar(c, c.bar(kBarPvDone), pv_cnt & 1)) return;
        ++pv_cnt;
        tc_fence_after();
        const bool need = alpha < 1.0f;
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int cc = 0; cc < 256; cc += 32) {
            float o[32];
            tmem_ld32(t_o + cc, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] *= alpha;
            tmem_st32(t_o + cc, o);
          }
          tmem_wait_st();
        }
      }

      // ---- P to shared memory (128B-swizzled K-major rows) ----
      {
        uint8_t* prow = c.gbase + kOffP + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint4 v = make_uint4(packed[4 * ch + 0], packed[4 * ch + 1], packed[4 * ch + 2], packed[4 * ch + 3]);
          *reinterpret_cast<uint4*>(prow + ((ch ^ (r & 7)) << 4)) = v;
        }
      }
      // ---- the last page of a row may hold garbage (even NaN) past L: zero
      //      those V rows so that 0 * garbage cannot reach O ----
      if (blk == last_page && (g.L & (kPage - 1))) {
        const int first_bad = g.L - blk * kPage;
        const int chunks = (kPage - first_bad) * 4 * 8;  // rows x panels x 16-byte chunks
        uint8_t* stage = c.gbase + kOffKv + (blk_cnt & 1) * kStageBytes;
        for (int e = r; e < chunks; e += 128) {
          const int row = first_bad + (e >> 5);
          const int panel = (e >> 3) & 3;
          const int ch = e & 7;
          *reinterpret_cast<uint4*>(stage + panel * kKvPanel + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(c.bar(kBarPFull));
      ++blk_cnt;
    }

    // ---- epilogue ----
    if (!wait_bar(c, c.bar(kBarPvDone), pv_cnt & 1)) return;
    ++pv_cnt;
    tc_fence_after();
    const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
    if (g.slot < 0) {
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) +
                            (static_cast<long long>(g.i) * p.R + row_g) * kDv + c.cta * 256;
#pragma unroll 1
      for (int cc = 0; cc < 256; cc += 32) {
        float o[32];
        tmem_ld32(t_o + cc, o);
        tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int k = 0; k < 32; k += 8) {
            uint4 v;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(o[k + 0] * inv_l, o[k + 1] * inv_l);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(o[k + 2] * inv_l, o[k + 3] * inv_l);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(o[k + 4] * inv_l, o[k + 5] * inv_l);
            __nv_bfloat162 h3 = __floats2bfloat162_rn(o[k + 6] * inv_l, o[k + 7] * inv_l);
            v.x = *reinterpret_cast<uint32_t*>(&h0);
            v.y = *reinterpret_cast<uint32_t*>(&h1);
            v.z = *reinterpret_cast<uint32_t*>(&h2);
            v.w = *reinterpret_cast<uint32_t*>(&h3);
            *reinterpret_cast<uint4*>(orow + cc + k) = v;
          }
        }
      }
      if (row_valid && c.cta == 0) {
        const float lse = le > 0.0f ? (m + __log2f(le)) * 0.69314718055994530942f : -INFINITY;
        p.lse[(static_cast<long long>(g.i) * p.h_q + hh) * p.s_q + t] = lse;
      }
    } else {
      float* orow = p.o_part + (static_cast<long long>(g.slot) * p.tile_rows + r) * kDv + c.cta * 256;
#pragma unroll 1
      for (int cc = 0; cc < 256; cc += 32) {
        float o[32];
        tmem_ld32(t_o + cc, o);
        tmem_wait_ld();
        if (row_valid) {
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(orow + cc + k) =
                make_float4(o[k] * inv_l, o[k + 1] * inv_l, o[k + 2] * inv_l, o[k + 3] * inv_l);
        }
      }
      if (row_valid && c.cta == 0) {
        const float lse = le > 0.0f ? (m + __log2f(le)) * 0.69314718055994530942f : -INFINITY;
        p.lse_part[static_cast<long long>(g.slot) * p.tile_rows + r] = lse;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(c.bar(kBarOEmpty));
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_decode_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  Ctx c;
  c.base = base;
  c.gbase = smem_raw + (base - raw);
  c.cta = cluster_ctarank();
  c.peer = c.cta ^ 1u;
  c.meta = p.meta;
  c.abort_flag = reinterpret_cast<volatile uint32_t*>(c.gbase + kOffAbort);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(c.bar(kBarKvFull + 0), 1);
    mbar_init(c.bar(kBarKvFull + 1), 1);
    mbar_init(c.bar(kBarKvEmpty + 0), 1);
    mbar_init(c.bar(kBarKvEmpty + 1), 1);
    mbar_init(c.bar(kBarQFull), 1);
    mbar_init(c.bar(kBarQEmpty), 1);
    mbar_init(c.bar(kBarSFull + 0), 1);
    mbar_init(c.bar(kBarSFull + 1), 1);
    mbar_init(c.bar(kBarSEmpty + 0), 4);
    mbar_init(c.bar(kBarSEmpty + 1), 4);
    mbar_init(c.bar(kBarPFull), 4);
    mbar_init(c.bar(kBarPvDone), 1);
    mbar_init(c.bar(kBarXFull), 1);
    mbar_init(c.bar(kBarXEmpty), 4);
    mbar_init(c.bar(kBarOEmpty), 4);
    mbar_init(c.bar(kBarFinal), 1);
    *c.abort_flag = 0u;
    fence_mbar_init_cluster();
  }
  // Query rows past the tile's real rows are never written by TMA: zero them
  // once so that the padded MMA rows stay finite.
  if (p.q_box_rows < kMTile) {
    const int rows = kMTile - p.q_box_rows;
    const int per_panel128 = rows * 8;  // 16-byte chunks
    for (int e = threadIdx.x; e < per_panel128 * 4; e += kThreads) {
      const int panel = e / per_panel128;
      const int rem = e - panel * per_panel128;
      *reinterpret_cast<uint4*>(c.gbase + kOffQ + panel * kQPanel + (p.q_box_rows + rem / 8) * 128 + (rem & 7) * 16) =
          make_uint4(0, 0, 0, 0);
    }
    for (int e = threadIdx.x; e < rows * 4; e += kThreads) {
      *reinterpret_cast<uint4*>(c.gbase + kOffQ + 4 * kQPanel + (p.q_box_rows + e / 4) * 64 + (e & 3) * 16) =
          make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(base + kOffTmemSlot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_kv_lat);
    tma_prefetch_desc(&p.tm_kv_rope);
    tma_prefetch_desc(&p.tm_q_lat);
    tma_prefetch_desc(&p.tm_q_rope);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // the peer's barriers exist before any remote arrival
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(c.gbase + kOffTmemSlot);
  c.peer_x = map_to_rank(base + kOffX, c.peer);
  c.peer_xfull = map_to_rank(c.bar(kBarXFull), c.peer);
  c.peer_xempty = map_to_rank(c.bar(kBarXEmpty), c.peer);
  c.peer_abort = map_to_rank(base + kOffAbort, c.peer);

  // The plan must be the one built for this call's shape on this many pairs.
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int pairs = static_cast<int>(gridDim.x >> 1);
  const bool plan_ok = p.meta[kHMagic] == static_cast<int32_t>(kMagic) && p.meta[kHPairs] == pairs &&
                       p.meta[kHBatch] == p.batch && p.meta[kHHq] == p.h_q && p.meta[kHSq] == p.s_q;
  int s_begin = 0, s_end = 0;
  if (plan_ok) {
    const MetaLayout lo = meta_layout(p.batch, p.h_q, p.s_q);
    s_begin = p.meta[lo.pair_off + pair];
    s_end = p.meta[lo.pair_off + pair + 1];
  } else if (threadIdx.x == 0 && c.cta == 0 && pair == 0) {
    atomicOr(reinterpret_cast<unsigned int*>(c.meta + kHError), MLA_DEVERR_PLAN);
  }

  if (warp == 0) {
    if (lane == 0) producer(p, c, s_begin, s_end);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_issuer(p, c, tmem, s_begin, s_end);
    __syncwarp();
  } else if (warp >= 4) {
    softmax_epilogue(p, c, tmem, s_begin, s_end);
  }

  // ---- teardown: drain MMAs, wait for the peer, free TMEM ----
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      umma_commit(c.bar(kBarFinal));
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(c.bar(kBarFinal), 0) && globaltimer() - t0 < kTimeoutNs) {
      }
    }
    __syncwarp();
  }
  if (*c.abort_flag) __nanosleep(20000);  // let a peer's in-flight DSMEM stores land
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t decode_kernel_smem_bytes() { return kSmemBytes; }

cudaError_t decode_kernel_prepare() {
  return cudaFuncSetAttribute(mla_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

cudaError_t decode_kernel_pairs(int* pairs) {
  cudaError_t e = decode_kernel_prepare();
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  e = cudaOccupancyMaxActiveClusters(&clusters, mla_decode_kernel, &cfg);
  if (e != cudaSuccess) return e;
  *pairs = clusters < kMaxPairs ? clusters : kMaxPairs;
  return cudaSuccess;
}

cudaError_t launch_decode(const DecodeParams& p, int pairs, cudaStream_t stream) {
  mla_decode_kernel<<<dim3(2 * pairs), dim3(kThreads), kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
