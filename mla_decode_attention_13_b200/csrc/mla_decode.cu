// Split-KV MLA decode kernel for sm_100a (B200).
//
// What it computes: for every query row (batch row i, query token t, head h)
// the absorbed-form attention over that row's cached latent tokens ("MLA 和
// MHA 的 Kernel 区别", sections "MLA Decode" and "MLA 的 FlashAttention": load
// each latent tile from HBM once, score it on chip, reuse it for every head).
// Scores use all 576 dims of a cached row (512 latent + 64 rope); values are
// the first 512 dims of the same row.
//
// How: one persistent 2-CTA cluster per SM pair walks the plan's segments.
// The pair works on a tile of 128 query rows (a work row); CTA c owns query
// rows [64c, 64c + 64).  Both products run as pair MMAs (tcgen05.mma
// cta_group::2, M = 128), issued by the leader CTA: each CTA supplies its 64
// rows of the A operand and half of the B operand's columns from its own
// shared memory at the same offsets; the tensor cores share the B halves, and
// each CTA's 64 rows of the result land in its own TMEM spread over all 128
// lanes (lanes 0-63 hold the first N/2 columns, lanes 64-127 the rest).
//   * QK^T: A = Q (64 rows x 576, shared memory, loaded once per segment),
//     B = the page's cache rows: CTA c TMA-loads tokens [32c, 32c + 32) of each
//     64-token page, all 576 columns, so the page's keys are read once for
//     the pair.  S (64 rows x 64 tokens per CTA) lands in 32 TMEM columns:
//     lane r < 64 holds tokens 0-31 of row r, lane r + 64 tokens 32-63.
//   * Softmax: thread r (= TMEM lane r) handles row r mod 64, 32 tokens; the
//     two threads of a row trade their block maxima through shared memory.
//     Online softmax in the log2 domain with a lazy rescale (the running max
//     only moves when a block's max exceeds it by more than kTau; O and the
//     running sums are rescaled together, so the result is exact).  The
//     bf16-rounded weights P go to shared memory (A operand of PV); the
//     normaliser and lse use their unrounded fp32 sum.
//   * PV: O (64 rows x 512 per CTA, 256 TMEM columns) += P V in two MMAs of
//     N = 256; for each, CTA c supplies latent columns [128c, 128c + 128) of
//     that half for all 64 tokens (its own TMA load of the page's V columns).
//   Pages are gathered through the block table ("FlashMLA overview": paged
//   kvcache, block size 64); the producer warp reads page ids 32 at a time.
// A row the plan splits writes fp32 (O / l, lse) partials to the workspace
// for the combine kernel; an unsplit row writes bf16 out and lse.
// Warp roles per CTA (256 threads): warp 0 = TMA producer, warp 1 = TMEM
// owner and (leader only) MMA issuer, warps 4-7 = softmax and epilogue.
//
// Every mbarrier wait is bounded by %globaltimer; on expiry the kernel sets
// MLA_DEVERR_TIMEOUT in the metadata error word, tells the peer CTA to stop,
// drains its own MMAs, frees TMEM and returns.
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
constexpr int kRowsCta = kMTile / 2;  // 64 query rows per CTA

// Shared-memory layout (offsets from a 1024-byte aligned base).  All operand
// tiles are 128-byte swizzled panels of 64 bf16 columns.
constexpr uint32_t kQPanel = kRowsCta * 128;               // 64 rows x 64 cols
constexpr uint32_t kQBytes = 9 * kQPanel;                  // 576 cols
constexpr uint32_t kKPanel = (kPage / 2) * 128;            // 32 tokens x 64 cols
constexpr uint32_t kKBytes = 9 * kKPanel;                  // this CTA's 32 tokens, 576 cols
constexpr uint32_t kVPanel = kPage * 128;                  // 64 tokens x 64 cols
constexpr uint32_t kVBytes = 4 * kVPanel;                  // 64 tokens x this CTA's 256 V cols
constexpr uint32_t kPBytes = kRowsCta * 128;               // 64 rows x 64 tokens bf16
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kQBytes;                 // key-half ring
constexpr uint32_t kOffV = kOffK + kStages * kKBytes;       // V ring
constexpr uint32_t kOffP = kOffV + kStages * kVBytes;       // 2 P buffers
constexpr uint32_t kOffMax = kOffP + 2 * kPBytes;           // float [2][128]
constexpr uint32_t kOffBar = kOffMax + 2 * 128 * 4;
constexpr uint32_t kSmemUsed = kOffBar + 256;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // slack for aligning the base

enum Bar : uint32_t {
  kBarKFull = 0,                  // [kStages] (leader) both CTAs' key halves landed
  kBarKEmpty = 2,                 // [kStages] (both) QK done with the key stage
  kBarVFull = 4,                  // [kStages] (leader) both CTAs' V columns landed
  kBarVEmpty = 6,                 // [kStages] (both) PV done with the V stage
  kBarQFull = 8,                  // (leader) both CTAs' Q rows landed
  kBarQEmpty = 9,                 // (both) last QK of the segment done
  kBarSFull = 10,                 // [2] (both) S buffer written
  kBarPFull = 12,                 // [2] (leader) P buffer written and O rescaled: 4 local warps + relay
  kBarPLocal = 14,                // [2] (non-leader) its 4 softmax warps, forwarded by the relay
  kBarPvDone = 16,                // [2] (both) PV of that P buffer done
  kBarOEmpty = 18,                // (leader) 8 softmax warps read O out
  kBarFinal = 19,                 // (leader) MMA drain at teardown
  kBarXMax = 20,                  // (both) 4 softmax warps published their row maxima / sums
  kNumBars = 21,
};
static_assert(kStages == 2, "barrier layout assumes two stages per ring");
constexpr uint32_t kOffTmemSlot = kOffBar + 8 * kNumBars;  // u32
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;           // u32
static_assert(kOffAbort + 4 <= kSmemUsed, "barrier area");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Tensor-memory columns (per CTA; the pair allocation mirrors them).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;    // 256: lanes 0-63 / 64-127 hold the two column halves of each N=256 product
constexpr uint32_t kColS = 256;  // 2 x 32

constexpr uint32_t kIdescQK = idesc_bf16_f32(kMTile, kPage, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kMTile, 256, true);

struct Ctx {
  uint32_t base;     // shared::cta address of the aligned base
  uint8_t* gbase;    // generic pointer to the same place
  uint32_t cta;      // rank in the pair; 0 is the leader
  uint32_t peer_abort;
  uint32_t lead_bars;  // shared::cluster address of the leader's barrier block
  volatile uint32_t* abort_flag;
  int32_t* meta;
  __device__ uint32_t bar(uint32_t k) const { return base + kOffBar + 8 * k; }
  __device__ uint32_t lead_bar(uint32_t k) const { return lead_bars + 8 * k; }
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

// Arrive on one of the leader's barriers (locally in the leader, remotely from
// the other CTA).
__device__ __forceinline__ void arrive_leader(const Ctx& c, uint32_t k) {
  if (c.cta == 0) mbar_arrive(c.bar(k));
  else mbar_arrive_remote(c.lead_bar(k));
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
// Whole warp 0 of each CTA: lanes read 32 page ids at a time (one chunk
// ahead); lane 0 waits for a free stage and loads this CTA's key half (32
// tokens, 576 columns) and V columns (64 tokens, 256 columns) of each page,
// completing bytes on the leader's barriers.
__device__ __forceinline__ int load_page(const DecodeParams& p, const Ctx& c, const int32_t* table, int blk,
                                         int end) {
  if (blk >= end) return 0;
  int page = table[blk];
  if (page < 0 || page >= p.num_pages) {
    atomicOr(reinterpret_cast<unsigned int*>(c.meta + kHError), MLA_DEVERR_PAGE);
    page = 0;  // keep the copy inside the pool; the result is flagged
  }
  return page;
}

__device__ void producer(const DecodeParams& p, const Ctx& c, int s_begin, int s_end) {
  const int lane = threadIdx.x & 31;
  uint32_t k_cnt = 0, v_cnt = 0, seg_it = 0;
  bool ok = true;
  // Key halves run one page ahead of the V columns: the key stage frees after
  // QK, the V stage only after PV.
  auto load_k = [&](int page) -> bool {
    const uint32_t st = k_cnt % kStages;
    if (!wait_bar(c, c.bar(kBarKEmpty + st), ((k_cnt / kStages) & 1) ^ 1, true)) return false;
    if (c.cta == 0) mbar_arrive_expect_tx(c.bar(kBarKFull + st), 2 * kKBytes);
    const uint32_t dst = c.base + kOffK + st * kKBytes;
    const int ky = page * kPage + c.cta * (kPage / 2);
#pragma unroll
    for (int q = 0; q < 9; ++q) tma_load_2d_pair(dst + q * kKPanel, &p.tm_k, c.lead_bar(kBarKFull + st), q * 64, ky);
    ++k_cnt;
    return true;
  };
  auto load_v = [&](int page) -> bool {
    const uint32_t st = v_cnt % kStages;
    if (!wait_bar(c, c.bar(kBarVEmpty + st), ((v_cnt / kStages) & 1) ^ 1, true)) return false;
    if (c.cta == 0) mbar_arrive_expect_tx(c.bar(kBarVFull + st), 2 * kVBytes);
    const uint32_t dst = c.base + kOffV + st * kVBytes;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      tma_load_2d_pair(dst + q * kVPanel, &p.tm_v, c.lead_bar(kBarVFull + st),
                       (q >> 1) * 256 + c.cta * 128 + (q & 1) * 64, page * kPage);
    ++v_cnt;
    return true;
  };
  for (int s = s_begin; s < s_end && ok; ++s) {
    const Segment g = load_segment(p, s);
    if (g.bad) continue;
    // Q rows of this CTA (once per segment, after the previous segment's QKs).
    if (lane == 0) {
      ok = seg_it == 0 || wait_bar(c, c.bar(kBarQEmpty), (seg_it - 1) & 1, true);
      if (ok) {
        if (c.cta == 0) mbar_arrive_expect_tx(c.bar(kBarQFull), 2 * kQBytes);
        const int y = g.i * p.R + g.mt * kMTile + c.cta * kRowsCta;
#pragma unroll
        for (int q = 0; q < 9; ++q)
          tma_load_2d_pair(c.base + kOffQ + q * kQPanel, &p.tm_q, c.lead_bar(kBarQFull), q * 64, y);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok) break;
    ++seg_it;
    const int32_t* table = p.block_table + static_cast<long long>(g.i) * p.max_pages;
    int cur = load_page(p, c, table, g.b0 + lane, g.b1);
    int prev_page = 0;
    for (int c0 = g.b0; c0 < g.b1 && ok; c0 += 32) {
      const int nxt = load_page(p, c, table, c0 + 32 + lane, g.b1);
      const int n = min(32, g.b1 - c0);
      for (int k = 0; k < n; ++k) {
        const int page = __shfl_sync(0xffffffffu, cur, k);
        int good = 1;
        if (lane == 0) {
          good = load_k(page) ? 1 : 0;
          if (good && c0 + k > g.b0) good = load_v(prev_page) ? 1 : 0;  // V of the previous page
        }
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) {
          ok = false;
          break;
        }
        prev_page = page;
      }
      cur = nxt;
    }
    if (ok && lane == 0) ok = load_v(prev_page);  // V of the segment's last page
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  }
}

// ------------------------------------------------------ MMA (leader only) --
__device__ __forceinline__ void issue_qk(const Ctx& c, uint32_t tmem, uint32_t stage, uint32_t sb) {
  const uint32_t q = c.base + kOffQ;
  const uint32_t k = c.base + kOffK + stage * kKBytes;
#pragma unroll
  for (int s = 0; s < 36; ++s) {
    const uint32_t off = (s & 3) * 32;
    const uint64_t a = smem_desc(q + (s >> 2) * kQPanel + off, 16, 1024, kSwizzle128B);
    const uint64_t b = smem_desc(k + (s >> 2) * kKPanel + off, 16, 1024, kSwizzle128B);
    umma_ss_pair(tmem + kColS + 32 * sb, a, b, kIdescQK, s > 0 ? 1u : 0u);
  }
}

// Issue order per segment: QK(0), then for each page j: QK(j+1), PV(j).
// The S buffer QK(j+1) writes held S(j-1), which both CTAs had read before
// signalling P(j-1) ready, and PV(j-1) was issued after that signal.
__device__ void mma_issuer(const DecodeParams& p, const Ctx& c, uint32_t tmem, int s_begin, int s_end) {
  uint32_t kv_cnt = 0, q_cnt = 0, seg_it = 0;
  const uint16_t both = 0x3;
  for (int s = s_begin; s < s_end; ++s) {
    const Segment g = load_segment(p, s);
    if (g.bad) continue;
    const int n = g.b1 - g.b0;
    if (!wait_bar(c, c.bar(kBarQFull), seg_it & 1, true)) return;
    for (int j = -1; j < n; ++j) {
      if (j + 1 < n) {
        const uint32_t kvi = kv_cnt + j + 1, st = kvi % kStages, sb = q_cnt & 1;
        if (!wait_bar(c, c.bar(kBarKFull + st), (kvi / kStages) & 1, true)) return;
        tc_fence_after();
        issue_qk(c, tmem, st, sb);
        umma_commit_pair(c.bar(kBarSFull + sb), both);
        umma_commit_pair(c.bar(kBarKEmpty + st), both);
        ++q_cnt;
        if (j + 1 == n - 1) umma_commit_pair(c.bar(kBarQEmpty), both);  // Q free once the last QK is done
      }
      if (j < 0) continue;
      const uint32_t kvj = kv_cnt + j, st = kvj % kStages, pb = kvj & 1;
      if (!wait_bar(c, c.bar(kBarVFull + st), (kvj / kStages) & 1, true)) return;
      if (!wait_bar(c, c.bar(kBarPFull + pb), (kvj >> 1) & 1, true)) return;
      if (j == 0 && seg_it > 0 && !wait_bar(c, c.bar(kBarOEmpty), (seg_it - 1) & 1, true)) return;
      tc_fence_after();
      const uint32_t pbuf = c.base + kOffP + pb * kPBytes;
      const uint32_t vbuf = c.base + kOffV + st * kVBytes;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t a = smem_desc(pbuf + k * 32, 16, 1024, kSwizzle128B);
          // V: K = 16 tokens from token 16k; this CTA's N/2 = 128 columns of
          // the half are two panels (leading byte offset = panel stride).
          const uint64_t b = smem_desc(vbuf + h * 2 * kVPanel + k * 16 * 128, kVPanel, 1024, kSwizzle128B);
          umma_ss_pair(tmem + kColO + 128 * h, a, b, kIdescPV, (j > 0 || k > 0) ? 1u : 0u);
        }
      }
      umma_commit_pair(c.bar(kBarVEmpty + st), both);
      umma_commit_pair(c.bar(kBarPvDone + pb), both);
    }
    kv_cnt += n;
    ++seg_it;
  }
}

// Non-leader only: forwards "P buffer ready" from its 4 softmax warps to the
// leader, so that the release at cluster scope does not stall the softmax.
__device__ void relay(const DecodeParams& p, const Ctx& c, int s_begin, int s_end) {
  uint32_t k = 0;
  for (int s = s_begin; s < s_end; ++s) {
    const Segment g = load_segment(p, s);
    if (g.bad) continue;
    for (int j = g.b0; j < g.b1; ++j, ++k) {
      if (!wait_bar(c, c.bar(kBarPLocal + (k & 1)), (k >> 1) & 1)) return;
      mbar_arrive_remote(c.lead_bar(kBarPFull + (k & 1)));
    }
  }
}

// ---------------------------------------------------- softmax, epilogue --
__device__ void softmax_epilogue(const DecodeParams& p, const Ctx& c, uint32_t tmem, int s_begin, int s_end) {
  const int r = threadIdx.x - 128;  // TMEM lane
  const int lane = threadIdx.x & 31;
  const int hr = r & (kRowsCta - 1);  // query row within this CTA
  const int half = r >> 6;            // 0: tokens 0-31 / first column half; 1: the rest
  const uint32_t lane_off = static_cast<uint32_t>(r & ~31) << 16;
  const uint32_t t_s = tmem + lane_off + kColS;
  const uint32_t t_o = tmem + lane_off + kColO;
  float* smax = reinterpret_cast<float*>(c.gbase + kOffMax);
  const float sl2 = p.scale_log2;
  // blk_cnt: pages consumed (selects the V stage); x_cnt: row exchanges with
  // the partner thread (selects the exchange slot and the barrier phase).
  uint32_t s_cnt = 0, blk_cnt = 0, x_cnt = 0;
  // Wait until the PV of global page k (P buffer k & 1) has completed.
  auto pv_done = [&](uint32_t k) -> bool { return wait_bar(c, c.bar(kBarPvDone + (k & 1)), (k >> 1) & 1, true); };
  // Publish v for the partner thread (same row, other half) and return its
  // value; the 4 warps meet on an mbarrier (bounded wait).
  auto trade = [&](float v, float* out) -> bool {
    float* buf = smax + (x_cnt & 1) * 128;
    buf[r] = v;
    __syncwarp();
    if (lane == 0) mbar_arrive(c.bar(kBarXMax));
    const bool ok = wait_bar(c, c.bar(kBarXMax), x_cnt & 1);
    ++x_cnt;
    *out = buf[r ^ 64];
    return ok;
  };

  for (int s = s_begin; s < s_end; ++s) {
    const Segment g = load_segment(p, s);
    if (g.bad) {
      if (r == 0 && c.cta == 0) atomicOr(reinterpret_cast<unsigned int*>(c.meta + kHError), MLA_DEVERR_SEQLEN);
      continue;
    }
    const int n = g.b1 - g.b0;
    const int q_row = c.cta * kRowsCta + hr;  // row within the 128-row tile
    const int row_g = g.mt * kMTile + q_row;
    const bool row_valid = q_row < p.tile_rows && row_g < p.R;
    const int t = row_g / p.h_q;
    const int hh = row_g - t * p.h_q;
    int limit = 0;
    if (row_valid) {
      limit = p.causal ? g.L - p.s_q + t + 1 : g.L;
      limit = limit < 0 ? 0 : (limit > g.L ? g.L : limit);
    }
    const int last_page = ceil_div(g.L, kPage) - 1;

    float m = -INFINITY, l = 0.0f;  // l: this thread's half of the row sum
    for (int j = 0; j < n; ++j) {
      const int blk = g.b0 + j;
      const uint32_t sb = s_cnt & 1;
      if (!wait_bar(c, c.bar(kBarSFull + sb), (s_cnt >> 1) & 1, true)) return;
      tc_fence_after();
      float sv[32];
      tmem_ld32(t_s + 32 * sb, sv);
      tmem_wait_ld();
      ++s_cnt;

      // ---- mask; block max over both halves of the row ----
      int nvalid = limit - blk * kPage - 32 * half;
      nvalid = nvalid < 0 ? 0 : (nvalid > 32 ? 32 : nvalid);
      if (nvalid < 32) {
#pragma unroll
        for (int k = 0; k < 32; ++k) sv[k] = (k < nvalid) ? sv[k] : -INFINITY;
      }
      float mx;
      {
        float a[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) a[k] = fmaxf(sv[k], sv[k + 16]);
#pragma unroll
        for (int k = 0; k < 8; ++k) a[k] = fmaxf(a[k], a[k + 8]);
#pragma unroll
        for (int k = 0; k < 4; ++k) a[k] = fmaxf(a[k], a[k + 4]);
        mx = fmaxf(fmaxf(a[0], a[2]), fmaxf(a[1], a[3]));
      }
      mx = (nvalid > 0) ? mx * sl2 : -INFINITY;  // softmax_scale >= 0
      float mx_peer;
      if (!trade(mx, &mx_peer)) return;
      mx = fmaxf(mx, mx_peer);
      float m_new = m;
      if (mx > m + kTau) m_new = mx;  // also true for the first finite block
      const float alpha = (m_new == m) ? 1.0f : ex2(m - m_new);  // 0 when m was -inf
      const float neg_m = (m_new == -INFINITY) ? 0.0f : -m_new;
      uint32_t packed[16];
      float e[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float a = ex2(fmaf(sv[2 * k], sl2, neg_m));
        float b = ex2(fmaf(sv[2 * k + 1], sl2, neg_m));
        if (nvalid < 32) {
          a = (2 * k < nvalid) ? a : 0.0f;
          b = (2 * k + 1 < nvalid) ? b : 0.0f;
        }
        e[k] = a + b;
        const __nv_bfloat162 pr = __floats2bfloat162_rn(a, b);
        packed[k] = *reinterpret_cast<const uint32_t*>(&pr);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) e[k] += e[k + 8];
#pragma unroll
      for (int k = 0; k < 4; ++k) e[k] += e[k + 4];
      l = l * alpha + ((e[0] + e[2]) + (e[1] + e[3]));
      m = m_new;

      // ---- P buffer free (PV two pages back); O up to date for a rescale ----
      if (blk_cnt >= 2 && !pv_done(blk_cnt - 2)) return;
      if (j > 0) {
        const bool need = alpha < 1.0f;
        if (__any_sync(0xffffffffu, need)) {
          if (!pv_done(blk_cnt - 1)) return;
          tc_fence_after();
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
      // ---- P row hr, this thread's 32 tokens = 4 swizzled 16-byte chunks ----
      {
        uint8_t* prow = c.gbase + kOffP + (blk_cnt & 1) * kPBytes + (hr >> 3) * 1024 + (hr & 7) * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int ch = 4 * half + q;
          *reinterpret_cast<uint4*>(prow + ((ch ^ (hr & 7)) << 4)) =
              make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        }
      }
      // ---- the last page of a row may hold garbage (even NaN) past L: zero
      //      this CTA's V rows there so that 0 * garbage cannot reach O ----
      if (blk == last_page && (g.L & (kPage - 1))) {
        const int first_bad = g.L - blk * kPage;
        const int chunks = (kPage - first_bad) * 4 * 8;  // rows x panels x 16-byte chunks
        uint8_t* vst = c.gbase + kOffV + (blk_cnt % kStages) * kVBytes;
        for (int e2 = r; e2 < chunks; e2 += 128) {
          const int row = first_bad + (e2 >> 5);
          const int panel = (e2 >> 3) & 3;
          const int ch = e2 & 7;
          *reinterpret_cast<uint4*>(vst + panel * kVPanel + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(c.bar((c.cta == 0 ? kBarPFull : kBarPLocal) + (blk_cnt & 1)));
      ++blk_cnt;
    }

    // ---- epilogue ----
    if (!pv_done(blk_cnt - 1)) return;
    tc_fence_after();
    float l_peer;
    if (!trade(l, &l_peer)) return;
    const float lt = l + l_peer;
    const float inv_l = lt > 0.0f ? 1.0f / lt : 0.0f;
    const float lse_v = lt > 0.0f ? (m + __log2f(lt)) * 0.69314718055994530942f : -INFINITY;
    // This thread's O columns: for each half h of the 512, columns
    // [256h + 128*half, 256h + 128*half + 128).
    if (g.slot < 0) {
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + (static_cast<long long>(g.i) * p.R + row_g) * kDv;
#pragma unroll 1
      for (int cc = 0; cc < 256; cc += 32) {
        float o[32];
        tmem_ld32(t_o + cc, o);
        tmem_wait_ld();
        const int col = (cc >> 7) * 256 + 128 * half + (cc & 127);
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
            *reinterpret_cast<uint4*>(orow + col + k) = v;
          }
        }
      }
      if (row_valid && half == 0) p.lse[(static_cast<long long>(g.i) * p.h_q + hh) * p.s_q + t] = lse_v;
    } else {
      float* orow = p.o_part + (static_cast<long long>(g.slot) * p.tile_rows + q_row) * kDv;
#pragma unroll 1
      for (int cc = 0; cc < 256; cc += 32) {
        float o[32];
        tmem_ld32(t_o + cc, o);
        tmem_wait_ld();
        const int col = (cc >> 7) * 256 + 128 * half + (cc & 127);
        if (row_valid) {
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(orow + col + k) =
                make_float4(o[k] * inv_l, o[k + 1] * inv_l, o[k + 2] * inv_l, o[k + 3] * inv_l);
        }
      }
      if (row_valid && half == 0) p.lse_part[static_cast<long long>(g.slot) * p.tile_rows + q_row] = lse_v;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) arrive_leader(c, kBarOEmpty);
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
  c.meta = p.meta;
  c.abort_flag = reinterpret_cast<volatile uint32_t*>(c.gbase + kOffAbort);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    // Barriers of the leader's pipeline are only used in the leader, the
    // rest in both CTAs; initialise all of them everywhere.
    for (int k = 0; k < 2; ++k) {
      mbar_init(c.bar(kBarKFull + k), 1);
      mbar_init(c.bar(kBarKEmpty + k), 1);
      mbar_init(c.bar(kBarVFull + k), 1);
      mbar_init(c.bar(kBarVEmpty + k), 1);
      mbar_init(c.bar(kBarSFull + k), 1);
      mbar_init(c.bar(kBarPFull + k), 5);
      mbar_init(c.bar(kBarPLocal + k), 4);
      mbar_init(c.bar(kBarPvDone + k), 1);
    }
    mbar_init(c.bar(kBarQFull), 1);
    mbar_init(c.bar(kBarQEmpty), 1);
    mbar_init(c.bar(kBarOEmpty), 8);
    mbar_init(c.bar(kBarFinal), 1);
    mbar_init(c.bar(kBarXMax), 4);
    *c.abort_flag = 0u;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc_pair(base + kOffTmemSlot, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    tma_prefetch_desc(&p.tm_q);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // both CTAs' barriers exist before any remote arrival
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(c.gbase + kOffTmemSlot);
  c.peer_abort = map_to_rank(base + kOffAbort, c.cta ^ 1u);
  c.lead_bars = map_to_rank(base + kOffBar, 0);

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
    producer(p, c, s_begin, s_end);
  } else if (warp == 1) {
    if (lane == 0 && c.cta == 0) mma_issuer(p, c, tmem, s_begin, s_end);
    __syncwarp();
  } else if (warp == 2) {
    if (lane == 0 && c.cta == 1) relay(p, c, s_begin, s_end);
    __syncwarp();
  } else if (warp >= 4) {
    softmax_epilogue(p, c, tmem, s_begin, s_end);
  }

  // ---- teardown: drain the pair MMAs, wait for the peer, free TMEM ----
  __syncthreads();
  if (warp == 1 && c.cta == 0) {
    if (lane == 0) {
      umma_commit_pair(c.bar(kBarFinal), 0x1);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(c.bar(kBarFinal), 0) && globaltimer() - t0 < kTimeoutNs) {
      }
    }
    __syncwarp();
  }
  if (*c.abort_flag) __nanosleep(20000);  // let in-flight copies and arrivals land
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
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
