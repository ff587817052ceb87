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
//
// A tcgen05.mma costs at least ~64 cycles whatever its size, and a pair MMA
// only reaches the tensor peak at N = 256, so QK^T runs over four pages at a
// time (a group, 256 tokens); PV runs page by page at N = 256.
//   * Keys: CTA c supplies pages 2c and 2c + 1 of the group, all 64 tokens
//     and 576 columns, so a page leaves HBM once for the pair.  They stream
//     through a ring of panels (64 columns x 128 token rows, 16 KB, one TMA
//     box per page); a panel is free again as soon as its four K = 16 MMAs
//     are done.
//   * QK^T: A = Q (64 rows x 576, shared memory, loaded once per segment),
//     B = the group's panels, N = 256.  S (64 rows x 256 tokens per CTA)
//     lands in 128 TMEM columns: lane r < 64 holds pages 0 and 1 of the group
//     for row r, lane r + 64 pages 2 and 3.
//   * Values: for PV, CTA c needs all 64 tokens of a page in its value
//     columns [256h + 128c, 256h + 128c + 128) (h = 0, 1): a 32 KB tile per
//     page (one 4-D TMA box), read from L2 (the pair has just brought the
//     page in), in a ring of two.
//   * Softmax: eight warps; warps 4-7 read S columns 0-63, warps 8-11 columns
//     64-127.  A thread (TMEM lane r) handles row r mod 64 and one page of
//     the group (all 64 of its tokens), so each row of a P tile comes from a
//     single thread; the four threads of a row trade
//     their maxima (and, at the end, their sums) through shared memory.  Online softmax in the log2 domain with a lazy
//     rescale (the running max only moves when a block's max exceeds it by
//     more than kTau; O and the running sums are rescaled together, so the
//     result is exact).  The bf16-rounded weights P of each page go to a ring
//     of two shared-memory tiles (A operand of PV); the normaliser and lse use
//     the unrounded fp32 sum.
//   * PV: O (64 rows x 512 per CTA, 256 TMEM columns) += P V per page, in two
//     MMAs of N = 256 (four K = 16 steps each).
//   Two threads issue the MMAs, one the QK panels and one the PV pages, so
//   that the next group's QK overlaps this group's PV.  Pages are gathered through the
//   block table ("FlashMLA overview": paged kvcache, block size 64); the
//   producer warps read page ids 32 at a time.
// A row the plan splits writes fp32 (O / l, lse) partials to the workspace
// for the combine kernel; an unsplit row writes out (bf16, or fp32 for
// mla_decode_f32) and lse.
// Warp roles per CTA (384 threads): warp 0 = key/Q producer, warp 1 = TMEM
// owner and (leader only) QK issuer, warp 2 = value producer, warp 3 =
// (leader only) PV issuer, warps 4-11 = softmax and epilogue.  (A bulk L2 prefetch of the pages ahead of the key
// loads was measured on B200 and made the kernel slower; there is none.)
//
// Cross-CTA signals are relaxed arrivals after a CTA-scope fence (see
// mbar_arrive_remote) and every wait is at CTA scope.  Every mbarrier wait is
// bounded by %globaltimer; on expiry the kernel sets MLA_DEVERR_TIMEOUT in the
// metadata error word, tells the peer CTA to stop, drains its own MMAs, frees
// TMEM and returns.
#include <cuda_bf16.h>

#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {

// Optional clock64 timeline of the pipeline roles, for profiling builds only
// (compile with -DMLA_DECODE_TRACE; the default build records nothing).
#ifdef MLA_DECODE_TRACE
__device__ unsigned long long g_mla_trace[4][24][512];  // [traced CTA][event][index]
__device__ unsigned long long g_mla_span[160][4];  // [pair][start, end, segments, pages] (globaltimer)
// Prologue of the leader CTA of each pair: [entry, after cluster sync, after the grid dependency, exit].
__device__ unsigned long long g_mla_pro[160][4];
#define MLA_PRO(k)                                                                    \
  do {                                                                                \
    if (threadIdx.x == 0 && cluster_ctarank() == 0) g_mla_pro[blockIdx.x >> 1][k] = globaltimer(); \
  } while (0)
// First wait that ran out of time: [taken, barrier index, parity, thread, block, clock].
__device__ unsigned long long g_mla_abort[6];
// Per block and warp: the wait it left on abort (1 << 32 | barrier << 8 | parity)
// and the role's last loop position.
__device__ unsigned long long g_mla_stuck[160 * 2][16];
__device__ unsigned long long g_mla_step[160 * 2][16];
#define MLA_STEP(v) \
  do {              \
    g_mla_step[blockIdx.x][threadIdx.x >> 5] = static_cast<unsigned long long>(v); \
  } while (0)
#define MLA_TRACE(ev, k)                                                                         \
  do {                                                                                           \
    const int tr_pair_ = static_cast<int>(blockIdx.x >> 1);                                      \
    const int tr_slot_ = tr_pair_ == 0 ? 0 : (tr_pair_ == 37 ? 2 : -1);                          \
    if (tr_slot_ >= 0 && (k) < 512) g_mla_trace[tr_slot_ + (blockIdx.x & 1)][ev][k] = clock64(); \
  } while (0)
#else
#define MLA_TRACE(ev, k) \
  do {                   \
  } while (0)
#define MLA_STEP(v) \
  do {              \
  } while (0)
#define MLA_PRO(k) \
  do {             \
  } while (0)
#endif

// Error bits raised on this device since the host last took them (see
// mla_take_device_errors): the metadata's error word is rewritten by every
// plan, this one is only cleared by the host.
__device__ unsigned int g_mla_sticky_error;

namespace {

using namespace ptx;

__device__ __forceinline__ void set_error(int32_t* meta, uint32_t bits) {
  atomicOr(reinterpret_cast<unsigned int*>(meta + kHError), bits);
  atomicOr(&g_mla_sticky_error, bits);
}

constexpr int kGroup = 4;             // pages per QK group
constexpr int kVRing = 2;             // value tiles (and P tiles)
// PV completion barriers, one per page mod kPvBars.  A parity wait on page k's
// barrier is only right while the PV of page k - kPvBars is known to be done
// and that of page k + kPvBars is not; with four, every wait below has that
// window by construction (a page's writers learn of PV up to three pages
// before their group from the previous group's writers, through the row
// exchange).
constexpr int kPvBars = 4;
constexpr float kTau = 8.0f;          // lazy-rescale threshold, log2 units
constexpr uint64_t kTimeoutNs = 500ull * 1000ull * 1000ull;
constexpr uint64_t kDrainNs = 2ull * 1000ull * 1000ull;  // teardown wait for in-flight copies after an abort
constexpr int kRowsCta = kMTile / 2;  // 64 query rows per CTA

// The two cache formats the kernel is built for.
//   * bf16: the cache row is 576 bf16 values; key panels and value tiles come
//     straight from TMA.  12 warps.
//   * fp8: the 512 latent values of a row are E4M3 codes with one power-of-two
//     scale 2^e per token, the 64 rope values bf16 ("MLA 和 MHA 的 Kernel 区别",
//     section "量化友好性": the latent cache tolerates FP8 or INT8, dequantised
//     as it is loaded).  The key codes land by TMA in a staging ring and
//     four converter warps dequantise them into the key panels; each page's
//     value codes land in its value tile's slot and the two softmax warps
//     that write the page's P dequantise them in place.  The latent products
//     run as f16 MMAs: every E4M3 value times 2^e with e in [-15, 7] is exact
//     in f16, and the latent part of Q is converted to f16 once per segment;
//     the rope panel stays bf16 in both Q and the keys.  16 warps.
struct CfgBf16 {
  static constexpr bool kFp8 = false;
  static constexpr int kThreads = 384;
  static constexpr int kKRing = 4;  // key panel slots
  static constexpr int kSRing = 0;  // staging slots
};
struct CfgFp8 {
  static constexpr bool kFp8 = true;
  static constexpr int kThreads = 512;
  static constexpr int kKRing = 2;
  static constexpr int kSRing = 4;
};
// The FP8 build's 512 threads run with 128 registers each (65,536 / 512), the
// softmax warps included; no warp changes its register count at run time.

// Shared-memory layout (offsets from a 1024-byte aligned base).  All operand
// tiles are 128-byte swizzled panels of 64 16-bit columns.
constexpr uint32_t kQPanel = kRowsCta * 128;            // 64 rows x 64 cols
constexpr uint32_t kQBytes = 9 * kQPanel;               // 64 query rows x 576 cols
constexpr uint32_t kPagePanel = kPage * 128;            // 64 token rows x 64 cols
constexpr uint32_t kKSlot = 2 * kPagePanel;             // one panel of a CTA's two pages: 128 token rows
constexpr uint32_t kVPanel = kPage * 128;               // 64 tokens x 64 cols
constexpr uint32_t kVTile = 4 * kVPanel;                // 64 tokens x this CTA's 256 value cols
constexpr uint32_t kPTile = kRowsCta * 128;             // 64 rows x 64 tokens, 16-bit
constexpr uint32_t kSSlot = 8192;                       // fp8 staging: 128 token rows x 64 codes, or 64 x 64 bf16

template <class C>
struct Lay {
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQBytes;
  static constexpr uint32_t kOffS = kOffK + C::kKRing * kKSlot;
  static constexpr uint32_t kOffV = kOffS + C::kSRing * kSSlot;
  static constexpr uint32_t kOffP = kOffV + kVRing * kVTile;
  static constexpr uint32_t kOffX = kOffP + kVRing * kPTile;  // float [2][256] row exchange
  static constexpr uint32_t kOffBar = kOffX + 2 * 256 * 4;
  // Barriers.
  static constexpr uint32_t kBarKFull = 0;                          // [kKRing] (leader) both CTAs' key panel ready
  static constexpr uint32_t kBarKEmpty = kBarKFull + C::kKRing;     // [kKRing] (both) the panel's QK MMAs are done
  static constexpr uint32_t kBarVFull = kBarKEmpty + C::kKRing;     // [kVRing] (both, local) this CTA's value tile ready
  static constexpr uint32_t kBarPFull = kBarVFull + kVRing;         // [kVRing] (leader) P written by both CTAs
  static constexpr uint32_t kBarPvDone = kBarPFull + kVRing;        // [kPvBars] (both) PV of page k (mod kPvBars) done
  static constexpr uint32_t kBarSFull = kBarPvDone + kPvBars;       // [2] (both) S buffer written
  static constexpr uint32_t kBarSEmpty = kBarSFull + 2;             // [2] (leader) both CTAs' softmax warps read S
  static constexpr uint32_t kBarQFull = kBarSEmpty + 2;             // bf16: (leader) both CTAs' Q landed; fp8: (local)
  static constexpr uint32_t kBarQEmpty = kBarQFull + 1;             // (both) last QK of the segment done
  static constexpr uint32_t kBarOEmpty = kBarQEmpty + 1;            // (leader) both CTAs' softmax warps read O out
  static constexpr uint32_t kBarFinal = kBarOEmpty + 1;             // (leader) MMA drain at teardown
  static constexpr uint32_t kBarXch = kBarFinal + 1;                // (both) the 8 softmax warps published row values
  static constexpr uint32_t kBarStageFree = kBarXch + 1;            // (both, local) the epilogue read its staging
  static constexpr uint32_t kBarResc = kBarStageFree + 1;           // [2] (both, local) rows 32k.. rescaled O
  static constexpr uint32_t kBarQReady = kBarResc + 2;              // fp8: (leader) both CTAs' Q converted
  static constexpr uint32_t kBarStFull = kBarQReady + 1;            // fp8: [kSRing] (local) staging slot landed
  static constexpr uint32_t kBarStEmpty = kBarStFull + C::kSRing;   // fp8: [kSRing] (local) staging slot converted
  static constexpr uint32_t kBarVCodes = kBarStEmpty + C::kSRing;   // fp8: [kVRing] (local) a tile's value codes landed
  static constexpr uint32_t kNumBars = kBarVCodes + (C::kFp8 ? kVRing : 0);
  static constexpr uint32_t kOffTmemSlot = kOffBar + 8 * kNumBars;  // u32
  static constexpr uint32_t kOffAbort = kOffTmemSlot + 4;           // u32
  // u32 fill counts of the barriers that TMA copies complete on: [kKRing] key
  // slots (bf16) and [1] Q (the expect_tx posted: bf16 leader, fp8 each CTA),
  // [kVRing] value slots (bf16: the tiles; fp8: their codes), [kSRing]
  // staging slots (fp8); read at teardown to wait for copies still in flight
  // on abort.
  static constexpr uint32_t kOffFill = kOffAbort + 4;
  static constexpr uint32_t kFillQ = C::kKRing;
  static constexpr uint32_t kFillV = kFillQ + 1;
  static constexpr uint32_t kFillS = kFillV + kVRing;
  static constexpr uint32_t kNumFill = kFillS + C::kSRing;
  static constexpr uint32_t kSmemUsed = kOffFill + 4 * kNumFill;
  static constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // slack for aligning the base
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kOffK % 1024 == 0 && kOffS % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0,
                "1024-byte aligned tiles");
};

// Tensor-memory columns (per CTA; the pair allocation mirrors them).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;    // 256: lanes 0-63 / 64-127 hold the two column halves of each N=256 product
constexpr uint32_t kColS = 256;  // 2 x 128

constexpr uint32_t kIdescQK = idesc_bf16_f32(kMTile, kGroup * kPage, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kMTile, 256, true);
constexpr uint32_t kIdescQK16 = idesc_f16_f32(kMTile, kGroup * kPage, false);
constexpr uint32_t kIdescPV16 = idesc_f16_f32(kMTile, 256, true);

struct Segment {
  int w, b0, b1, slot;
  int i, mt, L;
  bool bad;
};

template <class C>
struct Ctx {
  using L = Lay<C>;
  uint32_t base;     // shared::cta address of the aligned base
  uint8_t* gbase;    // generic pointer to the same place
  uint32_t cta;      // rank in the pair; 0 is the leader
  uint32_t peer_abort;
  uint32_t lead_bars;  // shared::cluster address of the leader's barrier block
  volatile uint32_t* abort_flag;
  int32_t* meta;
  int s_begin;       // this pair's first segment, read with the pair's record
  Segment first;
  __device__ uint32_t bar(uint32_t k) const { return base + L::kOffBar + 8 * k; }
  __device__ uint32_t lead_bar(uint32_t k) const { return lead_bars + 8 * k; }
  __device__ uint32_t kslot(uint32_t k) const { return base + L::kOffK + k * kKSlot; }
  __device__ uint32_t stage(uint32_t k) const { return base + L::kOffS + k * kSSlot; }
  __device__ uint32_t vtile(uint32_t k) const { return base + L::kOffV + k * kVTile; }
  __device__ uint32_t ptile(uint32_t k) const { return base + L::kOffP + k * kPTile; }
  __device__ volatile uint32_t* fill() const { return reinterpret_cast<volatile uint32_t*>(gbase + L::kOffFill); }
};

template <class C>
__device__ void raise_abort(const Ctx<C>& c, uint32_t err_bits) {
  using L = Lay<C>;
  if (err_bits) set_error(c.meta, err_bits);
  *c.abort_flag = 1u;
  st_cluster_u32(c.peer_abort, 1u);
}

// Bounded wait on an mbarrier phase.  Returns false when the kernel is
// aborting (this wait timed out, or another role or the peer CTA gave up).
template <class C>
__device__ bool wait_bar(const Ctx<C>& c, uint32_t bar, uint32_t parity) {
  using L = Lay<C>;
  uint32_t spins = 0;
  uint64_t t0 = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++spins & 63u) == 0) {
      if (*c.abort_flag) {
#ifdef MLA_DECODE_TRACE
        g_mla_stuck[blockIdx.x][threadIdx.x >> 5] =
            (1ull << 32) | (static_cast<unsigned long long>((bar - c.base - L::kOffBar) / 8) << 8) | parity;
#endif
        return false;
      }
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kTimeoutNs) {
#ifdef MLA_DECODE_TRACE
        if (atomicCAS(&g_mla_abort[0], 0ull, 1ull) == 0ull) {
          g_mla_abort[1] = (bar - c.base - L::kOffBar) / 8;
          g_mla_abort[2] = parity;
          g_mla_abort[3] = threadIdx.x;
          g_mla_abort[4] = blockIdx.x;
          g_mla_abort[5] = clock64();
        }
#endif
        raise_abort(c, MLA_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Arrive on one of the leader's barriers (locally in the leader, remotely from
// the other CTA).  The caller's warp has written what the arrival publishes
// (shared memory of its own CTA, or TMEM reads that completed) and synced.
template <class C>
__device__ __forceinline__ void arrive_leader(const Ctx<C>& c, uint32_t k) {
  using L = Lay<C>;
  if (c.cta == 0) {
    mbar_arrive(c.bar(k));
  } else {
    fence_cta();
    mbar_arrive_remote(c.lead_bar(k));
  }
}

// A segment from its record (work row, first page, end page, slot; length).
// The length is the one the plan read, so every role takes the same decision
// on a bad segment whatever the lengths hold now (the softmax warps check
// them against it).
__device__ __forceinline__ Segment make_segment(const DecodeParams& p, int4 a, int L) {
  Segment g;
  g.w = a.x;
  g.b0 = a.y;
  g.b1 = a.z;
  g.slot = a.w;
  if (g.w < 0 || g.w >= p.batch * p.n_mt) {
    g.i = g.mt = g.L = 0;
    g.bad = true;
    return g;
  }
  g.i = g.w % p.batch;
  g.mt = g.w / p.batch;
  g.L = L;
  g.bad = g.L < 0 || g.L > kPage * p.max_pages || g.b1 > ceil_div(g.L, kPage) || g.b0 < 0 || g.b0 >= g.b1 ||
          g.slot >= p.max_slots;
  return g;
}

// Segment s of this pair: the first one came with the pair's record.
template <class C>
__device__ __forceinline__ Segment load_segment(const DecodeParams& p, const Ctx<C>& c, int s) {
  if (s == c.s_begin) return c.first;
  const MetaLayout lo = meta_layout(p.batch, p.h_q, p.s_q);
  const int32_t* rec = p.meta + lo.segs + kSegWords * s;
  const int4 a = *reinterpret_cast<const int4*>(rec);
  const int L = rec[4];
  return make_segment(p, a, L);
}

template <class C>
__device__ __forceinline__ int load_page(const DecodeParams& p, const Ctx<C>& c, const int32_t* table, int blk,
                                         int end) {
  using L = Lay<C>;
  if (blk >= end) return 0;
  int page = table[blk];
  if (page < 0 || page >= p.num_pages) {
    set_error(c.meta, MLA_DEVERR_PAGE);
    page = 0;  // keep the copy inside the pool; the result is flagged
  }
  return page;
}

// A group: up to kGroup consecutive pages of one segment.
struct Group {
  int blk;        // first page (logical block index within the row)
  int np;         // pages in the group, 1 to kGroup
  int page[kGroup];
  bool first;     // first group of its segment
};

// Walks this pair's segments in plan order and calls fn(segment, group) for
// every group, with the page ids read 32 at a time by the whole warp (one
// chunk ahead).  fn runs on every lane and returns false to stop the walk.
// on_segment(segment) runs on every lane before the segment's page ids are
// read, and returns false to stop the walk.
struct NoSegmentHook {
  __device__ bool operator()(const Segment&) const { return true; }
};

template <class C, typename Fn, typename SegFn = NoSegmentHook>
__device__ __forceinline__ void walk_groups(const DecodeParams& p, const Ctx<C>& c, int s_begin, int s_end, Fn&& fn,
                                            SegFn&& on_segment = SegFn()) {
  using L = Lay<C>;
  static_assert(32 % kGroup == 0, "groups never straddle a chunk of page ids");
  const int lane = threadIdx.x & 31;
  for (int s = s_begin; s < s_end; ++s) {
    const Segment sg = load_segment(p, c, s);
    if (sg.bad) continue;
    if (!on_segment(sg)) return;
    const int32_t* table = p.block_table + static_cast<long long>(sg.i) * p.max_pages;
    int cur = load_page(p, c, table, sg.b0 + lane, sg.b1);
    for (int c0 = sg.b0; c0 < sg.b1; c0 += 32) {
      const int nxt = load_page(p, c, table, c0 + 32 + lane, sg.b1);
      const int n = min(32, sg.b1 - c0);
      for (int k = 0; k < n; k += kGroup) {
        Group gr;
        gr.blk = c0 + k;
        gr.np = min(kGroup, n - k);
#pragma unroll
        for (int q = 0; q < kGroup; ++q) gr.page[q] = __shfl_sync(0xffffffffu, cur, k + q);
        gr.first = gr.blk == sg.b0;
        if (!fn(sg, gr)) return;
      }
      cur = nxt;
    }
  }
}

// ------------------------------------------------------------- producers --
// Warp 0: each segment's Q rows of this CTA, then this CTA's two pages of
// the group (pages 2c and 2c + 1, those that exist), panel by panel, into the
// key ring (bytes complete on the leader's barriers).
template <class C>
__device__ void producer_k(const DecodeParams& p, const Ctx<C>& c, int s_begin, int s_end) {
  using L = Lay<C>;
  const int lane = threadIdx.x & 31;
  uint32_t gi = 0, seg_it = 0, ks = 0;  // groups, segments started, key panels loaded
  // The segment's Q rows first, before its page ids are even read.
  auto load_q = [&](const Segment& sg) -> bool {
    int good = 1;
    if (lane == 0) {
      good = seg_it == 0 || wait_bar(c, c.bar(L::kBarQEmpty), (seg_it - 1) & 1);
      if (good) {
        MLA_TRACE(14, seg_it);
        const int y = sg.i * p.R + sg.mt * kMTile + c.cta * kRowsCta;
        if constexpr (C::kFp8) {
          // Each CTA converts its own rows: a local copy on its own barrier.
          mbar_arrive_expect_tx(c.bar(L::kBarQFull), kQBytes);
          c.fill()[L::kFillQ] += 1;
          tma_load_3d(c.base + L::kOffQ, &p.tm_q, c.bar(L::kBarQFull), 0, y, 0);
        } else {
          if (c.cta == 0) {
            mbar_arrive_expect_tx(c.bar(L::kBarQFull), 2 * kQBytes);
            c.fill()[L::kFillQ] += 1;
          }
          tma_load_3d_pair(c.base + L::kOffQ, &p.tm_q, c.lead_bar(L::kBarQFull), 0, y, 0);
        }
      }
    }
    ++seg_it;
    return __shfl_sync(0xffffffffu, good, 0) != 0;
  };
  if constexpr (C::kFp8) {
    // FP8 cache: this CTA's two pages of the group (2c and 2c + 1, those that
    // exist) go to the staging ring, ten 8 KB fills per group: the latent
    // codes of 64 columns of both pages (fills 0-7, one box per page, lanes 0
    // and 1 together), then the bf16 rope of each page (fills 8 and 9).  A
    // fill of a missing page posts no bytes but still completes, so that the
    // converters see every fill of every group.
    uint32_t sf = 0;
    walk_groups(p, c, s_begin, s_end, [&](const Segment&, const Group& gr) -> bool {
      const int my_np = min(max(gr.np - 2 * static_cast<int>(c.cta), 0), 2);
      const int page_a = gr.page[2 * c.cta], page_b = gr.page[2 * c.cta + 1];
      int good = 1;
      for (int f = 0; f < 10; ++f, ++sf) {
        const uint32_t slot = sf % C::kSRing;
        if (lane == 0 && sf >= C::kSRing)
          good = wait_bar(c, c.bar(L::kBarStEmpty + slot), ((sf / C::kSRing) - 1) & 1);
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) break;
        const uint32_t bytes = f < 8 ? my_np * (kSSlot / 2) : (f - 8 < my_np ? kSSlot : 0u);
        if (lane == 0) {
          MLA_TRACE(10, sf);
          mbar_arrive_expect_tx(c.bar(L::kBarStFull + slot), bytes);
          c.fill()[L::kFillS + slot] += 1;
        }
        __syncwarp();
        if (f < 8) {
          if (lane < my_np)
            tma_load_2d(c.stage(slot) + lane * (kSSlot / 2), &p.tm_codes, c.bar(L::kBarStFull + slot), 64 * f,
                        (lane == 0 ? page_a : page_b) * kPage);
        } else if (lane == 0 && f - 8 < my_np) {
          tma_load_2d(c.stage(slot), &p.tm_rope, c.bar(L::kBarStFull + slot), 0, (f == 8 ? page_a : page_b) * kPage);
        }
      }
      return good != 0;
    }, load_q);
    return;
  }
  walk_groups(p, c, s_begin, s_end, [&](const Segment& sg, const Group& gr) -> bool {
    if (lane == 0) MLA_TRACE(0, gi);
    // This CTA's two pages of the group; lanes 0 and 1 issue their boxes in
    // one instruction (a TMA issue holds its thread for ~300 cycles; two
    // lanes of one instruction take ~420 together instead of ~660 in turn).
    const int my_page = c.cta == 0 ? (lane == 0 ? gr.page[0] : gr.page[1]) : (lane == 0 ? gr.page[2] : gr.page[3]);
    const bool my_load = lane < 2 && 2 * static_cast<int>(c.cta) + lane < gr.np;
    int good = 1;
    for (int pn = 0; pn < 9; ++pn, ++ks) {
      const uint32_t slot = ks % C::kKRing;
      if (lane == 0 && ks >= C::kKRing) good = wait_bar(c, c.bar(L::kBarKEmpty + slot), ((ks / C::kKRing) - 1) & 1);
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) break;
      if (lane == 0) {
        MLA_TRACE(10, ks);
        MLA_STEP(ks);
        if (c.cta == 0) {
          mbar_arrive_expect_tx(c.bar(L::kBarKFull + slot), gr.np * kPagePanel);
          c.fill()[slot] += 1;
        }
      }
      __syncwarp();
      if (my_load)
        tma_load_3d_pair(c.kslot(slot) + lane * kPagePanel, &p.tm_k, c.lead_bar(L::kBarKFull + slot), 0,
                         my_page * kPage, pn);
      if (lane == 0) MLA_TRACE(15, ks);
      // The other CTA also arrives, even when it has no page in the group:
      // otherwise the slot could fill and drain without it, and its parity
      // wait on the slot's empty barrier would fall two phases behind.
      if (lane == 0 && c.cta != 0) mbar_arrive_remote(c.lead_bar(L::kBarKFull + slot));
    }
    ++gi;
    return good != 0;
  }, load_q);
}

// Warp 2: this CTA's value tile of every page (all 64 tokens, its 256 value
// columns) into the value ring once PV two pages back has released the slot;
// bytes complete on this CTA's own barrier (the softmax warps wait for it
// before releasing P, so PV never runs ahead of it).  FP8 cache: the tile's
// codes instead, into the slot's upper half, for the page's P writers to
// dequantise.
template <class C>
__device__ void producer_v(const DecodeParams& p, const Ctx<C>& c, int s_begin, int s_end) {
  using L = Lay<C>;
  const int lane = threadIdx.x & 31;
  uint32_t ps = 0, seg_it = 0;  // pages, segments
  walk_groups(p, c, s_begin, s_end, [&](const Segment&, const Group& gr) -> bool {
    int good = 1;
    if (lane == 0) {
      // The epilogue of the previous segment stages its output in the value
      // ring: a new segment's first tile waits until those stores have read it.
      if (gr.first && seg_it > 0) good = wait_bar(c, c.bar(L::kBarStageFree), (seg_it - 1) & 1);
      for (int q = 0; q < gr.np && good; ++q, ++ps) {
        const uint32_t slot = ps % kVRing;
        if (ps >= kVRing) {
          const uint32_t k = ps - kVRing;  // the tile's previous page: its PV must be done
          good = wait_bar(c, c.bar(L::kBarPvDone + k % kPvBars), (k / kPvBars) & 1);
        }
        if (good) {
          MLA_TRACE(3, ps);
          MLA_STEP(ps);
          if constexpr (C::kFp8) {
            // The page's E4M3 codes of this CTA's value columns ([h][64
            // tokens][128 codes], 16 KB) into the upper half of the tile's
            // slot; the page's P writers dequantise them over the whole slot.
            const uint32_t bar = c.bar(L::kBarVCodes + slot);
            mbar_arrive_expect_tx(bar, kVTile / 2);
            c.fill()[L::kFillV + slot] += 1;
            tma_load_4d(c.vtile(slot) + kVTile / 2, &p.tm_vcodes, bar, 0, gr.page[q] * kPage,
                        static_cast<int>(c.cta), 0);
          } else {
            const uint32_t bar = c.bar(L::kBarVFull + slot);
            mbar_arrive_expect_tx(bar, kVTile);
            c.fill()[L::kFillV + slot] += 1;
            tma_load_4d(c.vtile(slot), &p.tm_v, bar, 0, gr.page[q] * kPage, 2 * static_cast<int>(c.cta), 0);
          }
        }
      }
    }
    if (gr.first) ++seg_it;
    return __shfl_sync(0xffffffffu, good, 0) != 0;
  });
}

// ------------------------------------------------ converters (FP8 cache) --
// f16 bits of 2^e, exact for e in [-24, 15] (subnormal below -14); e is
// clamped to that range (exponents outside [-15, 7] are flagged by the key
// converter, as E4M3 values times 2^e are exact in f16 only there).
__device__ __forceinline__ uint32_t f16_pow2(int e) {
  e = max(-24, min(15, e));
  return e >= -14 ? static_cast<uint32_t>(e + 15) << 10 : 1u << (e + 24);
}

// 16 E4M3 codes (a 16-byte chunk, first code in the lowest byte) times the
// f16x2 scale, as 16 f16 values in memory order (two 16-byte chunks).
__device__ __forceinline__ void dequant16(const uint4& v, uint32_t scale2, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t r[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    r[2 * k] = mul_f16x2(e4m3x2_to_f16x2(static_cast<uint16_t>(w[k] & 0xFFFFu)), scale2);
    r[2 * k + 1] = mul_f16x2(e4m3x2_to_f16x2(static_cast<uint16_t>(w[k] >> 16)), scale2);
  }
  lo = make_uint4(r[0], r[1], r[2], r[3]);
  hi = make_uint4(r[4], r[5], r[6], r[7]);
}

// Two bf16 values (low half first) to f16, rounded to nearest.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  return f32x2_to_f16x2(__uint_as_float(w & 0xFFFF0000u), __uint_as_float(w << 16));
}

// Warps 12-15 (128 threads), FP8 cache only.
//   * At each segment start: this CTA's Q rows to f16 in place (the latent
//     panels 0-7; the rope panel stays bf16), then one arrival per warp on the
//     leader's Q barrier.  A query value past the f16 range is flagged.
//   * Per group, the nine key panels in order: a latent panel's staging slot
//     (64 codes of 128 token rows: this CTA's two pages) is dequantised with
//     each token's 2^e into a key slot (f16, 128B-swizzled, the layout of the
//     bf16 cache's key panels); the rope panel is two staging slots (one page
//     each, already bf16 and swizzled) copied into one key slot.  Each key
//     slot then gets one arrival per warp on the leader's full barrier.
template <class C>
__device__ void key_converter(const DecodeParams& p, const Ctx<C>& c, int s_begin, int s_end) {
  using L = Lay<C>;
  const int kt = static_cast<int>(threadIdx.x) - 12 * 32;  // 0-127
  const int lane = threadIdx.x & 31;
  uint32_t seg_it = 0, sf = 0, kf = 0;  // segments, staging fills, key panels
  bool out_of_range = false;
  auto conv_q = [&](const Segment&) -> bool {
    MLA_STEP((10ull << 40) | seg_it);
    if (!wait_bar(c, c.bar(L::kBarQFull), seg_it & 1)) return false;
    ++seg_it;
    uint4* q = reinterpret_cast<uint4*>(c.gbase + L::kOffQ);
    uint32_t inf_seen = 0;  // bit 15 of a half: an f16 result with the all-ones exponent
    for (int k = kt; k < static_cast<int>(8 * kQPanel / 16); k += 128) {
      uint4 v = q[k];
      v.x = bf16x2_to_f16x2(v.x);
      v.y = bf16x2_to_f16x2(v.y);
      v.z = bf16x2_to_f16x2(v.z);
      v.w = bf16x2_to_f16x2(v.w);
      inf_seen |= ((v.x & 0x7C007C00u) + 0x04000400u) | ((v.y & 0x7C007C00u) + 0x04000400u) |
                  ((v.z & 0x7C007C00u) + 0x04000400u) | ((v.w & 0x7C007C00u) + 0x04000400u);
      q[k] = v;
    }
    if (inf_seen & 0x80008000u) out_of_range = true;
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) arrive_leader(c, L::kBarQReady);
    return true;
  };
  walk_groups(p, c, s_begin, s_end, [&](const Segment& sg, const Group& gr) -> bool {
    const int my_np = min(max(gr.np - 2 * static_cast<int>(c.cta), 0), 2);
    // Exponents of this CTA's two pages: lane l holds those of rows 4l to
    // 4l + 3 (rows 0-63: page 2c, rows 64-127: page 2c + 1).
    const int half = lane >> 4;
    uint32_t ew = 0;
    if (half < my_np) {
      const int page = gr.page[2 * c.cta + half];
      ew = *reinterpret_cast<const uint32_t*>(p.exps + static_cast<long long>(page) * kPage + 4 * (lane & 15));
      const int tok0 = (gr.blk + 2 * static_cast<int>(c.cta) + half) * kPage + 4 * (lane & 15);
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int e = static_cast<int8_t>((ew >> (8 * b)) & 0xFFu);
        if (tok0 + b < sg.L && (e < -15 || e > 7)) out_of_range = true;
      }
    }
    for (int pn = 0; pn < 9; ++pn, ++kf) {
      const uint32_t ks = kf % C::kKRing;
      MLA_STEP((8ull << 40) | (static_cast<unsigned long long>(sf) << 20) | kf);
      if (kf >= C::kKRing && !wait_bar(c, c.bar(L::kBarKEmpty + ks), ((kf / C::kKRing) - 1) & 1)) return false;
      uint8_t* dst = c.gbase + L::kOffK + ks * kKSlot;
      if (pn < 8) {
        const uint32_t st = sf % C::kSRing;
        if (!wait_bar(c, c.bar(L::kBarStFull + st), (sf / C::kSRing) & 1)) return false;
        if (kt == 0) MLA_TRACE(20, kf);
        ++sf;
        // 16-byte chunk kt + 128 j of the slot: row kt / 4 + 32 j (64 bytes
        // of codes per row), codes 16 (kt % 4) to +15 -> f16 chunks 2 (kt % 4)
        // and + 1 of the row, swizzled by row % 8 = (kt / 4) % 8.
        const int row0 = kt >> 2, c4 = kt & 3;
        const uint8_t* src = c.gbase + L::kOffS + st * kSSlot + 16 * kt;
        uint8_t* drow = dst + row0 * 128;
        const uint32_t off_lo = ((2 * c4) ^ (row0 & 7)) << 4, off_hi = ((2 * c4 + 1) ^ (row0 & 7)) << 4;
        uint4 v4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v4[j] = *reinterpret_cast<const uint4*>(src + 2048 * j);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = v4[j];
          const int row = row0 + 32 * j;
          const int e = static_cast<int8_t>((__shfl_sync(0xffffffffu, ew, row >> 2) >> (8 * (row & 3))) & 0xFFu);
          const uint32_t sc = f16_pow2(e);
          uint4 lo, hi;
          dequant16(v, sc | (sc << 16), lo, hi);
          *reinterpret_cast<uint4*>(drow + 4096 * j + off_lo) = lo;
          *reinterpret_cast<uint4*>(drow + 4096 * j + off_hi) = hi;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(c.bar(L::kBarStEmpty + st));
      } else {
        for (int h = 0; h < 2; ++h, ++sf) {
          const uint32_t st = sf % C::kSRing;
          if (!wait_bar(c, c.bar(L::kBarStFull + st), (sf / C::kSRing) & 1)) return false;
          const uint4* src = reinterpret_cast<const uint4*>(c.gbase + L::kOffS + st * kSSlot);
          uint4* d = reinterpret_cast<uint4*>(dst + h * kSSlot);
#pragma unroll
          for (int k = kt; k < static_cast<int>(kSSlot / 16); k += 128) d[k] = src[k];
          __syncwarp();
          if (lane == 0) mbar_arrive(c.bar(L::kBarStEmpty + st));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (kt == 0) MLA_TRACE(21, kf);
      if (lane == 0) arrive_leader(c, L::kBarKFull + ks);
    }
    return true;
  }, conv_q);
  if (out_of_range) set_error(c.meta, MLA_DEVERR_FP8_RANGE);
}

// FP8 cache: this CTA's value tile of one page (its 256 value columns [256h +
// 128c, +128), h = 0, 1, of all 64 tokens, f16, the layout of the bf16 cache's
// value tiles), dequantised in place by the 64 softmax threads that write the
// page's P (vt = 0-63, two warps), once warp 2 has copied the page's codes of
// those columns into the upper half of the tile's slot.  Each thread reads
// its tokens' codes and writes their dequantised rows (each token's 2^e
// applied; zeros for tokens at or past `valid`, whose codes may hold
// anything) over the whole slot.  A token belongs to one warp (tokens 0 and 1
// mod 4 to the first, 2 and 3 to the second), and its f16 rows in the upper
// half lie exactly over its own codes ([h][token][128] there, panels 2 and 3
// row `token`), so a warp sync between a pass's reads and its writes is the
// only ordering needed.  ew: the page's exponent bytes of tokens 2 lane and
// 2 lane + 1.
template <class C>
__device__ __forceinline__ void convert_value_tile(const Ctx<C>& c, uint32_t slot, int vt, int valid, uint32_t ew) {
  using L = Lay<C>;
  // 16-byte chunk vt + 64 j (j = 0-15) of the tile: token tok0 + 4 j (tok0 =
  // vt / 16), half h = (vt / 8) % 2, codes 16 i8 to +15 (i8 = vt % 8) of the
  // half's 128 columns; only the token moves with j.
  const int tok0 = vt >> 4, h = (vt >> 3) & 1, i8 = vt & 7;
  const uint32_t ch = 2 * (i8 & 3);
  uint8_t* tile = c.gbase + L::kOffV + slot * kVTile;
  const uint8_t* src = tile + kVTile / 2 + (h * kPage + tok0) * 128 + 16 * i8;  // codes: [h][token][128]
  // panel [h][i8 / 4]; f16 chunks 2 (i8 % 4) and + 1 of the token's 128-byte
  // row, swizzled by tok % 8 = (tok0 % 8) ^ (4 (j % 2)).
  uint8_t* drow = tile + (2 * h + (i8 >> 2)) * kVPanel + tok0 * 128;
#pragma unroll
  for (int jb = 0; jb < 16; jb += 4) {  // four passes of four tokens
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = *reinterpret_cast<const uint4*>(src + 512 * (jb + u));
    __syncwarp();  // the pass's codes are in registers before its rows overwrite them
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = jb + u;
      const int tok = tok0 + 4 * j;
      const int e = static_cast<int8_t>((__shfl_sync(0xffffffffu, ew, tok >> 1) >> (8 * (tok & 1))) & 0xFFu);
      const uint32_t sc = f16_pow2(e);
      uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
      if (tok < valid) dequant16(v[u], sc | (sc << 16), lo, hi);
      const uint32_t sw = (tok0 & 7) ^ (4 * (j & 1));
      *reinterpret_cast<uint4*>(drow + 512 * j + ((ch ^ sw) << 4)) = lo;
      *reinterpret_cast<uint4*>(drow + 512 * j + (((ch + 1) ^ sw) << 4)) = hi;
    }
  }
}

// ------------------------------------------------------ MMA (leader only) --
// One key panel of QK^T: four K = 16 steps over its 64 columns.
template <class C>
__device__ __forceinline__ void issue_qk_panel(const Ctx<C>& c, uint32_t tmem, uint32_t slot, int pn, uint32_t sb) {
  using L = Lay<C>;
  const uint32_t q = c.base + L::kOffQ + pn * kQPanel;
  const uint32_t k = c.kslot(slot);
  // FP8 cache: the latent panels (0-7) are f16 on both sides, the rope panel bf16.
  const uint32_t idesc = (C::kFp8 && pn < 8) ? kIdescQK16 : kIdescQK;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint64_t a = smem_desc(q + s * 32, 16, 1024, kSwizzle128B);
    const uint64_t b = smem_desc(k + s * 32, 16, 1024, kSwizzle128B);
    umma_ss_pair(tmem + kColS + 128 * sb, a, b, idesc, (pn > 0 || s > 0) ? 1u : 0u);
  }
}

// O (+)= P V for one page.  For the N = 256 half h, each CTA's 128 value
// columns are two adjacent panels (leading byte offset = one panel); K step k
// takes tokens [16k, 16k + 16).
template <class C>
__device__ __forceinline__ void issue_pv_page(const Ctx<C>& c, uint32_t tmem, uint32_t slot, bool first) {
  using L = Lay<C>;
  const uint32_t pt = c.ptile(slot);
  const uint32_t vt = c.vtile(slot);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint64_t a = smem_desc(pt + k * 32, 16, 1024, kSwizzle128B);
      const uint64_t b = smem_desc(vt + h * 2 * kVPanel + k * 16 * 128, kVPanel, 1024, kSwizzle128B);
      umma_ss_pair(tmem + kColO + 128 * h, a, b, C::kFp8 ? kIdescPV16 : kIdescPV, (!first || k > 0) ? 1u : 0u);
    }
  }
}

// The MMAs go out as two independent streams, each from its own thread of the
// leader CTA, so that one waiting (or blocked on a full tensor-core queue)
// never holds the other back.  The two share no TMEM: QK writes the S
// buffers, PV accumulates O.
//   * QK (warp 1): per group, one panel at a time as the key panels land; a
//     group may start once both CTAs have read the S buffer it overwrites.
//   * PV (warp 3): per page, in order, once both CTAs have written its P
//     (which they do after reading S, so QK of its group is complete); the
//     first page of a segment also waits until O has been read out.
template <class C>
__device__ void qk_issuer(const DecodeParams& p, const Ctx<C>& c, uint32_t tmem, int s_begin, int s_end) {
  using L = Lay<C>;
  uint32_t gi = 0, ks = 0, seg_it = 0;  // groups, key panels consumed, segments
  const uint16_t both = 0x3;
  for (int s = s_begin; s < s_end; ++s) {
    const Segment sg = load_segment(p, c, s);
    if (sg.bad) continue;
    const int ng = ceil_div(sg.b1 - sg.b0, kGroup);
    // FP8 cache: both CTAs' Q rows converted; bf16: both CTAs' Q rows landed.
    if (!wait_bar(c, c.bar(C::kFp8 ? L::kBarQReady : L::kBarQFull), seg_it & 1)) return;
    for (int gq = 0; gq < ng; ++gq, ++gi) {
      const uint32_t sb = gi & 1;
      if (gi >= 2 && !wait_bar(c, c.bar(L::kBarSEmpty + sb), ((gi - 2) >> 1) & 1)) return;
      MLA_TRACE(1, gi);
      for (int pn = 0; pn < 9; ++pn, ++ks) {
        const uint32_t slot = ks % C::kKRing;
        if (!wait_bar(c, c.bar(L::kBarKFull + slot), (ks / C::kKRing) & 1)) return;
        MLA_TRACE(9, ks);
        MLA_STEP(ks);
        tc_fence_after();
        issue_qk_panel(c, tmem, slot, pn, sb);
        umma_commit_pair(c.bar(L::kBarKEmpty + slot), both);
      }
      umma_commit_pair(c.bar(L::kBarSFull + sb), both);
    }
    umma_commit_pair(c.bar(L::kBarQEmpty), both);  // Q free once the segment's last QK is done
    ++seg_it;
  }
}

template <class C>
__device__ void pv_issuer(const DecodeParams& p, const Ctx<C>& c, uint32_t tmem, int s_begin, int s_end) {
  using L = Lay<C>;
  uint32_t pg = 0, seg_it = 0;  // pages, segments
  const uint16_t both = 0x3;
  for (int s = s_begin; s < s_end; ++s) {
    const Segment sg = load_segment(p, c, s);
    if (sg.bad) continue;
    const int n = sg.b1 - sg.b0;
    for (int jp = 0; jp < n; ++jp, ++pg) {
      const uint32_t slot = pg % kVRing;
      if (!wait_bar(c, c.bar(L::kBarPFull + slot), (pg / kVRing) & 1)) return;
      if (jp == 0 && seg_it > 0 && !wait_bar(c, c.bar(L::kBarOEmpty), (seg_it - 1) & 1)) return;
      MLA_TRACE(2, pg);
      MLA_STEP(pg);
      tc_fence_after();
      issue_pv_page(c, tmem, slot, jp == 0);
      umma_commit_pair(c.bar(L::kBarPvDone + pg % kPvBars), both);
    }
    ++seg_it;
  }
}

// ---------------------------------------------------- softmax, epilogue --
// Masks the scores past `nvalid` and returns their maximum (-inf if none).
__device__ __forceinline__ float masked_max(float (&sv)[32], int nvalid) {
  if (nvalid < 32) {
#pragma unroll
    for (int k = 0; k < 32; ++k) sv[k] = (k < nvalid) ? sv[k] : -INFINITY;
  }
  float a[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) a[k] = fmaxf(sv[k], sv[k + 16]);
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = fmaxf(a[k], a[k + 8]);
#pragma unroll
  for (int k = 0; k < 4; ++k) a[k] = fmaxf(a[k], a[k + 4]);
  return fmaxf(fmaxf(a[0], a[2]), fmaxf(a[1], a[3]));
}

// p = 2^(s * sl2 - m) for the first nvalid scores, 0 past them; packs the
// weights in pairs, rounded to bf16 (or to f16 for the FP8 cache, whose PV
// product is f16), and returns their unrounded fp32 sum.
template <bool kF16>
__device__ __forceinline__ float exp_pack(const float (&sv)[32], int nvalid, float sl2, float neg_m,
                                          uint32_t (&packed)[16]) {
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
    if constexpr (kF16) {
      packed[k] = f32x2_to_f16x2(b, a);
    } else {
      const __nv_bfloat162 pr = __floats2bfloat162_rn(a, b);
      packed[k] = *reinterpret_cast<const uint32_t*>(&pr);
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) e[k] += e[k + 8];
#pragma unroll
  for (int k = 0; k < 4; ++k) e[k] += e[k + 4];
  return (e[0] + e[2]) + (e[1] + e[3]);
}

template <class C>
__device__ void softmax_epilogue(const DecodeParams& p, const Ctx<C>& c, uint32_t tmem, int s_begin, int s_end) {
  using L = Lay<C>;
  const int r = threadIdx.x - 128;  // 0-255: softmax thread
  const int sp = r >> 7;            // S columns 64 sp .. 64 sp + 63 of each lane
  const int rr = r & 127;           // TMEM lane
  const int lane = threadIdx.x & 31;
  const int hr = rr & (kRowsCta - 1);  // query row within this CTA
  const int half = rr >> 6;            // 0: pages 0-1 of each group / first O column half; 1: the rest
  const int q = 2 * half + sp;         // this thread's page of each group
  const uint32_t lane_off = static_cast<uint32_t>(rr & ~31) << 16;
  const uint32_t t_s = tmem + lane_off + kColS + 64 * sp;
  const uint32_t t_o = tmem + lane_off + kColO + 128 * sp;  // this thread's 128 O columns
  float* xbuf = reinterpret_cast<float*>(c.gbase + L::kOffX);
  // This thread's 64 weights of a page: row hr of the P tile (128 bytes,
  // 16-byte chunks swizzled by the row).
  const uint32_t prow_off = (hr >> 3) * 1024 + (hr & 7) * 128;
  const float sl2 = p.scale_log2;
  // gi: groups, ps: pages before the current group (select buffers and
  // phases); x_cnt: row exchanges among the row's four threads; n_resc: O
  // rescales of this warp's rows (the four warps holding rows 32 kr ..
  // 32 kr + 31 take the same decisions, so they count alike).
  uint32_t gi = 0, ps = 0, x_cnt = 0, n_resc = 0;
  const int kr = (rr >> 5) & 1;
  auto pv_done = [&](uint32_t k) -> bool { return wait_bar(c, c.bar(L::kBarPvDone + k % kPvBars), (k / kPvBars) & 1); };
  // Publish v for the other three threads of this row (the other half of its
  // tokens, the other page pair) and return the max or the sum of the four;
  // the eight softmax warps meet on an mbarrier (bounded wait).
  auto trade = [&](float v, bool sum, float* out) -> bool {
    float* buf = xbuf + (x_cnt & 1) * 256;
    buf[r] = v;
    __syncwarp();
    if (lane == 0) mbar_arrive(c.bar(L::kBarXch));
    const bool ok = wait_bar(c, c.bar(L::kBarXch), x_cnt & 1);
    ++x_cnt;
    const float a = buf[r ^ 64], b = buf[r ^ 128], d = buf[r ^ 192];
    *out = sum ? (v + a) + (b + d) : fmaxf(fmaxf(v, a), fmaxf(b, d));
    return ok;
  };

  for (int s = s_begin; s < s_end; ++s) {
    const Segment sg = load_segment(p, c, s);
    if (sg.bad) {
      if (r == 0 && c.cta == 0) set_error(c.meta, MLA_DEVERR_SEQLEN);
      continue;
    }
    // The plan was made for these lengths (off the critical path: these warps
    // wait for the segment's first scores anyway).
    if (r == 0 && c.cta == 0 && p.seqlens[sg.i] != sg.L) set_error(c.meta, MLA_DEVERR_PLAN);
    const int n = sg.b1 - sg.b0;
    const int q_row = c.cta * kRowsCta + hr;  // row within the 128-row tile
    const int row_g = sg.mt * kMTile + q_row;
    const bool row_valid = q_row < p.tile_rows && row_g < p.R;
    const int t = row_g / p.h_q;
    const int hh = row_g - t * p.h_q;
    int limit = 0;
    if (row_valid) {
      limit = p.causal ? sg.L - p.s_q + t + 1 : sg.L;
      limit = limit < 0 ? 0 : (limit > sg.L ? sg.L : limit);
    }
    const int last_page = ceil_div(sg.L, kPage) - 1;

    float m = -INFINITY, l = 0.0f;  // l: this thread's share of the row sum
    int np_last = 0;                // pages in the segment's last group
    for (int j = 0; j < n; j += kGroup, ++gi) {
      const int blk = sg.b0 + j;
      const int np = min(kGroup, n - j);
      np_last = np;
      const uint32_t sb = gi & 1;
      // FP8 cache: this thread's page's exponent bytes (tokens 2 lane, + 1),
      // for the value tile it dequantises; loaded before the scores are waited
      // for.  (A page id outside the pool reads page 0, as the producers do;
      // they flag it.)
      uint32_t v_ew = 0;
      if constexpr (C::kFp8) {
        if (q < np) {
          int page = p.block_table[static_cast<long long>(sg.i) * p.max_pages + blk + q];
          page = (page < 0 || page >= p.num_pages) ? 0 : page;
          v_ew = *reinterpret_cast<const uint16_t*>(p.exps + static_cast<long long>(page) * kPage + 2 * lane);
        }
      }
      if (!wait_bar(c, c.bar(L::kBarSFull + sb), (gi >> 1) & 1)) return;
      if (r == 0) MLA_TRACE(4, gi);
      MLA_STEP((1ull << 40) | (static_cast<unsigned long long>(gi) << 20) | ps);
      tc_fence_after();
      float sv[2][32];
      tmem_ld32(t_s + 128 * sb, sv[0]);
      tmem_ld32(t_s + 128 * sb + 32, sv[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(c, L::kBarSEmpty + sb);  // S buffer read

      // ---- mask; max over the group's four pages ----
      int nv[2];
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int v = limit - (blk + q) * kPage - 32 * e;
        nv[e] = (q >= np || v < 0) ? 0 : (v > 32 ? 32 : v);
        mx = fmaxf(mx, masked_max(sv[e], nv[e]));
      }
      mx = (nv[0] > 0) ? mx * sl2 : -INFINITY;  // tokens are valid from the left; softmax_scale >= 0
      if (!trade(mx, false, &mx)) return;
      if (r == 0) MLA_TRACE(5, gi);
      float m_new = m;
      if (mx > m + kTau) m_new = mx;  // also true for the first finite block
      const float alpha = (m_new == m) ? 1.0f : ex2(m - m_new);  // 0 when m was -inf
      const float neg_m = (m_new == -INFINITY) ? 0.0f : -m_new;

      // ---- rescale this thread's O columns (rare): after PV of every earlier
      //      page of the segment, and before PV of this group's first page,
      //      whose P writers wait on the row half's rescale barrier ----
      const bool resc = j > 0 && __any_sync(0xffffffffu, alpha < 1.0f);
      if (resc) {
        MLA_STEP((5ull << 40) | ps);
        if (!pv_done(ps - 1)) return;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 128; cc += 32) {
          float o[32];
          tmem_ld32(t_o + cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= alpha;
          tmem_st32(t_o + cc, o);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(c.bar(L::kBarResc + kr));
        ++n_resc;
        MLA_STEP((6ull << 40) | n_resc);
      }

      float lsum = 0.0f;
      uint32_t packed[2][16];
      if (q < np)
        lsum = exp_pack<C::kFp8>(sv[0], nv[0], sl2, neg_m, packed[0]) +
               exp_pack<C::kFp8>(sv[1], nv[1], sl2, neg_m, packed[1]);
      // ---- P tile free (PV two pages back); write this thread's row of P ----
      auto write_p = [&]() -> bool {
        const uint32_t pg = ps + q;  // global page index
        const uint32_t slot = pg % kVRing;
        if (pg >= kVRing && !pv_done(pg - kVRing)) return false;
        MLA_STEP((2ull << 40) | pg);
        if (rr == 0) MLA_TRACE(6, pg);
        uint8_t* prow = c.gbase + L::kOffP + slot * kPTile + prow_off;
#pragma unroll
        for (int ci = 0; ci < 8; ++ci)
          *reinterpret_cast<uint4*>(prow + ((ci ^ (hr & 7)) << 4)) =
              make_uint4(packed[ci >> 2][4 * (ci & 3)], packed[ci >> 2][4 * (ci & 3) + 1],
                         packed[ci >> 2][4 * (ci & 3) + 2], packed[ci >> 2][4 * (ci & 3) + 3]);
        return true;
      };
      // ---- this warp's rows of page k's P (k = q, the thread's page) and its
      //      share of the value tile are ready: release them to the PV
      //      issuer.  The group's first PV adds to O, so its P writers first
      //      wait until every warp of these rows has rescaled its O columns ----
      auto release = [&](int k) -> bool {
        if (resc && k == 0 && q == 0 && !wait_bar(c, c.bar(L::kBarResc + kr), (n_resc - 1) & 1)) return false;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_leader(c, L::kBarPFull + (ps + k) % kVRing);
        MLA_STEP((4ull << 40) | (ps + k));
        if (rr == 0) MLA_TRACE(8, ps + k);
        return true;
      };
      if constexpr (!C::kFp8) {
        if (q < np) {
          if (!write_p()) return;
          // ---- this CTA's value tile has landed; the last page of a row may
          //      hold garbage (even NaN) past L: zero the value rows there, so
          //      that 0 * garbage cannot reach O ----
          const uint32_t pg = ps + q;
          const uint32_t slot = pg % kVRing;
          if (!wait_bar(c, c.bar(L::kBarVFull + slot), (pg / kVRing) & 1)) return;
          MLA_STEP((3ull << 40) | pg);
          if (rr == 0) MLA_TRACE(7, pg);
          if (blk + q == last_page && (sg.L & (kPage - 1))) {
            const int first_bad = sg.L - last_page * kPage;
            const int chunks = (kPage - first_bad) * 4 * 8;  // tokens x panels x 16-byte chunks
            uint8_t* vt = c.gbase + L::kOffV + slot * kVTile;
            for (int e2 = hr; e2 < chunks; e2 += kRowsCta) {
              const int tok = first_bad + (e2 >> 5);
              *reinterpret_cast<uint4*>(vt + ((e2 >> 3) & 3) * kVPanel + tok * 128 + (e2 & 7) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
          }
          if (!release(q)) return;
        }
      } else {
        // ---- FP8 cache: the page's codes have landed; its P writers
        //      dequantise its value tile (zeros past L) ----
        if (q < np) {
          if (!write_p()) return;
          const uint32_t pg = ps + q;
          const uint32_t slot = pg % kVRing;
          if (!wait_bar(c, c.bar(L::kBarVCodes + slot), (pg / kVRing) & 1)) return;
          if (rr == 0) MLA_TRACE(22, pg);
          const int valid = blk + q == last_page ? sg.L - last_page * kPage : kPage;
          convert_value_tile(c, slot, hr, valid, v_ew);
          if (rr == 0) MLA_TRACE(23, pg);
          if (!release(q)) return;
        }
      }
      l = l * alpha + lsum;
      m = m_new;
      ps += np;
    }

    // ---- epilogue: the writers of the last page (whose own P-slot wait
    //      makes this parity wait exact) wait for its PV; the row exchange
    //      then orders everyone's O reads after it ----
    MLA_STEP((7ull << 40) | ps);
    if (q == np_last - 1 && !pv_done(ps - 1)) return;
    if (r == 0) MLA_TRACE(12, s - s_begin);
    float lt;
    if (!trade(l, true, &lt)) return;
    if ((threadIdx.x & 31) == 0) MLA_TRACE(16, 8 * (s - s_begin) + ((threadIdx.x >> 5) - 4));
    tc_fence_after();
    const float inv_l = lt > 0.0f ? 1.0f / lt : 0.0f;
    const float lse_v = lt > 0.0f ? (m + __log2f(lt)) * 0.69314718055994530942f : -INFINITY;
    // Output: each warp owns 32 rows x 128 columns of this CTA's tile (its
    // TMEM lanes, O columns [256 sp + 128 half, +128)).  It stages them in
    // shared memory, in the value ring (idle between segments), as 128-byte
    // rows with 16-byte chunks swizzled by row (the 128B swizzle of a TMA
    // box).  A whole row's bf16 output leaves by bulk tensor stores; fp32
    // partials and fp32 outputs are read back four rows per instruction and
    // written as whole 128-byte lines with coalesced 16-byte stores, skipping
    // rows past R (or tile_rows).  (Measured: synchronous TMA stores of 4 KB
    // boxes took ~4,500 cycles for a CTA's 128 KB of fp32 partials, ~140
    // cycles per box, about what the coalesced stores take.)
    const int ws = (threadIdx.x >> 5) - 4;  // softmax warp 0-7
    uint8_t* stage = c.gbase + L::kOffV + ws * 4096;
    const int row0 = c.cta * kRowsCta + 32 * ((rr >> 5) & 1);  // first row of this warp in the tile
    const uint32_t swz = lane & 7;
    const int col0 = 256 * sp + 128 * half;
    const int rd_row = lane >> 3;   // read-back: rows rd_row + 4 i, chunk lane % 8
    const int rd_chunk = lane & 7;
    if (sg.slot < 0 && !p.out_f32) {
      // bf16 output of a whole row: the warp's 32 rows x 128 columns are
      // staged as two 4 KB boxes (8 KB of the value ring per warp; the 128B
      // swizzle above is the one the output tensor map expects) and written
      // by two bulk tensor stores, which drain while the warp goes on; the
      // value ring is released once they have read their staging.
      uint8_t* stage8 = c.gbase + L::kOffV + ws * 8192;
#pragma unroll 1
      for (int k = 0; k < 2; ++k) {  // 64 columns (128 bytes of bf16) per box
        float o[64];
        tmem_ld32(t_o + 64 * k, *reinterpret_cast<float(*)[32]>(o));
        tmem_ld32(t_o + 64 * k + 32, *reinterpret_cast<float(*)[32]>(o + 32));
        tmem_wait_ld();
        uint8_t* srow = stage8 + 4096 * k + lane * 128;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          __nv_bfloat162 h0 = __floats2bfloat162_rn(o[8 * jj + 0] * inv_l, o[8 * jj + 1] * inv_l);
          __nv_bfloat162 h1 = __floats2bfloat162_rn(o[8 * jj + 2] * inv_l, o[8 * jj + 3] * inv_l);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(o[8 * jj + 4] * inv_l, o[8 * jj + 5] * inv_l);
          __nv_bfloat162 h3 = __floats2bfloat162_rn(o[8 * jj + 6] * inv_l, o[8 * jj + 7] * inv_l);
          uint4 v;
          v.x = *reinterpret_cast<uint32_t*>(&h0);
          v.y = *reinterpret_cast<uint32_t*>(&h1);
          v.z = *reinterpret_cast<uint32_t*>(&h2);
          v.w = *reinterpret_cast<uint32_t*>(&h3);
          *reinterpret_cast<uint4*>(srow + ((jj ^ swz) << 4)) = v;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t src = c.base + L::kOffV + ws * 8192;
        tma_store_3d(&p.tm_out, src, col0, sg.mt * kMTile + row0, sg.i);
        tma_store_3d(&p.tm_out, src + 4096, col0 + 64, sg.mt * kMTile + row0, sg.i);
        bulk_commit_group();
      }
      if (row_valid && half == 0 && sp == 0) p.lse[(static_cast<long long>(sg.i) * p.h_q + hh) * p.s_q + t] = lse_v;
    } else {
      // fp32: a piece of a split row (its partial, in the workspace), or a
      // whole row of an fp32 output.
      float* obase;
      int rows_ok;
      if (sg.slot < 0) {
        obase = static_cast<float*>(p.out) + (static_cast<long long>(sg.i) * p.R + sg.mt * kMTile + row0) * kDv + col0;
        rows_ok = p.R - (sg.mt * kMTile + row0);
      } else {
        obase = p.o_part + (static_cast<long long>(sg.slot) * p.tile_rows + row0) * kDv + col0;
        rows_ok = p.tile_rows - row0;
      }
#pragma unroll 1
      for (int k = 0; k < 4; ++k) {  // 32 columns (128 bytes of fp32) per step
        float o[32];
        tmem_ld32(t_o + 32 * k, o);
        tmem_wait_ld();
        uint8_t* srow = stage + lane * 128;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
          *reinterpret_cast<float4*>(srow + ((jj ^ swz) << 4)) =
              make_float4(o[4 * jj] * inv_l, o[4 * jj + 1] * inv_l, o[4 * jj + 2] * inv_l, o[4 * jj + 3] * inv_l);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r2 = rd_row + 4 * i;
          const float4 v = *reinterpret_cast<const float4*>(stage + r2 * 128 + ((rd_chunk ^ (r2 & 7)) << 4));
          if (r2 < rows_ok)
            *reinterpret_cast<float4*>(obase + static_cast<long long>(r2) * kDv + 32 * k + 4 * rd_chunk) = v;
        }
        __syncwarp();
      }
      if (row_valid && half == 0 && sp == 0) {
        if (sg.slot < 0)
          p.lse[(static_cast<long long>(sg.i) * p.h_q + hh) * p.s_q + t] = lse_v;
        else
          p.lse_part[static_cast<long long>(sg.slot) * p.tile_rows + q_row] = lse_v;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) MLA_TRACE(17, 8 * (s - s_begin) + ((threadIdx.x >> 5) - 4));
    if (lane == 0) arrive_leader(c, L::kBarOEmpty);  // O is read out: the next segment's PV may overwrite it
    if (lane == 0) {
      MLA_TRACE(18, 8 * (s - s_begin) + ((threadIdx.x >> 5) - 4));
      bulk_wait_read_all();                   // this warp's bulk stores (if any) have read their staging
      mbar_arrive(c.bar(L::kBarStageFree));  // staging read: the value ring may be refilled
    }
    __syncwarp();
    if (r == 0) MLA_TRACE(13, s - s_begin);
  }
  if (lane == 0) MLA_TRACE(19, (threadIdx.x >> 5) - 4);
  __syncwarp();
}

// Softmax warps on their way out (normal or abort): this warp's bulk stores
// of outputs are complete before the CTA's shared memory goes away.
template <class C>
__device__ void softmax_epilogue_then_drain(const DecodeParams& p, const Ctx<C>& c, uint32_t tmem, int s_begin,
                                            int s_end) {
  softmax_epilogue(p, c, tmem, s_begin, s_end);
  if ((threadIdx.x & 31) == 0) bulk_wait_all();
  __syncwarp();
}

// After an abort: wait, bounded, for the last phase of every barrier that a
// TMA copy of this CTA completes on, so that no copy is still writing this
// CTA's shared memory when it exits.  A barrier filled n times has at most its
// phase n - 1 outstanding (a slot is refilled only after its previous phase
// completed).  The leader waits for the key and Q barriers, which count the
// other CTA's bytes too; the other CTA then leaves only after the cluster
// barrier that follows.  Returns false if a wait ran out (a copy that was
// never issued by the other CTA, whose abort came first).
template <class C>
__device__ __noinline__ bool drain_copies(const Ctx<C>& c) {
  using L = Lay<C>;
  volatile uint32_t* fill = c.fill();
  bool ok = true;
  auto wait_last = [&](uint32_t bar, uint32_t n) {
    if (n == 0 || !ok) return;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, (n - 1) & 1u)) {
      if (globaltimer() - t0 > kDrainNs) {
        ok = false;
        return;
      }
    }
  };
  if constexpr (C::kFp8) {
    // every copy lands on this CTA's own barriers: Q and the staging slots
    wait_last(c.bar(L::kBarQFull), fill[L::kFillQ]);
    for (int k = 0; k < C::kSRing; ++k) wait_last(c.bar(L::kBarStFull + k), fill[L::kFillS + k]);
    for (int k = 0; k < kVRing; ++k) wait_last(c.bar(L::kBarVCodes + k), fill[L::kFillV + k]);
  } else {
    if (c.cta == 0) {
      for (int k = 0; k < C::kKRing; ++k) wait_last(c.bar(L::kBarKFull + k), fill[k]);
      wait_last(c.bar(L::kBarQFull), fill[L::kFillQ]);
    }
    for (int k = 0; k < kVRing; ++k) wait_last(c.bar(L::kBarVFull + k), fill[L::kFillV + k]);
  }
  return ok;
}

template <class C>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(C::kThreads, 1)
    mla_decode_kernel(const __grid_constant__ DecodeParams p) {
  using L = Lay<C>;
  extern __shared__ uint8_t smem_raw[];
  MLA_PRO(0);
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  Ctx<C> c;
  c.base = base;
  c.gbase = smem_raw + (base - raw);
  c.cta = cluster_ctarank();
  c.meta = p.meta;
  c.abort_flag = reinterpret_cast<volatile uint32_t*>(c.gbase + L::kOffAbort);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    // Barriers of the leader's pipeline are only used in the leader, the
    // rest in both CTAs; initialise all of them everywhere.
    // Key panels: bf16, the leader's expect_tx arrival plus one from the other
    // CTA; fp8, one arrival per key-converter warp of both CTAs.  Value tiles:
    // bf16, the copy's expect_tx arrival (fp8: the codes' copy completes
    // VCodes, and the page's P writers dequantise the tile before releasing
    // P).  P tiles: the page's two P-writer warps in both CTAs.
    for (int k = 0; k < C::kKRing; ++k) {
      mbar_init(c.bar(L::kBarKFull + k), C::kFp8 ? 8 : 2);
      mbar_init(c.bar(L::kBarKEmpty + k), 1);
    }
    for (int k = 0; k < kVRing; ++k) {
      mbar_init(c.bar(L::kBarVFull + k), 1);
      mbar_init(c.bar(L::kBarPFull + k), 4);
    }
    mbar_init(c.bar(L::kBarQReady), 8);
    for (int k = 0; k < C::kSRing; ++k) {
      mbar_init(c.bar(L::kBarStFull + k), 1);
      mbar_init(c.bar(L::kBarStEmpty + k), 4);
    }
    if constexpr (C::kFp8)
      for (int k = 0; k < kVRing; ++k) mbar_init(c.bar(L::kBarVCodes + k), 1);
    for (int k = 0; k < kPvBars; ++k) mbar_init(c.bar(L::kBarPvDone + k), 1);
    for (int k = 0; k < 2; ++k) {
      mbar_init(c.bar(L::kBarSFull + k), 1);
      mbar_init(c.bar(L::kBarSEmpty + k), 16);
    }
    mbar_init(c.bar(L::kBarQFull), 1);
    mbar_init(c.bar(L::kBarQEmpty), 1);
    mbar_init(c.bar(L::kBarOEmpty), 16);
    mbar_init(c.bar(L::kBarXch), 8);
    mbar_init(c.bar(L::kBarFinal), 2);
    mbar_init(c.bar(L::kBarStageFree), 8);
    mbar_init(c.bar(L::kBarResc), 4);
    mbar_init(c.bar(L::kBarResc + 1), 4);
    *c.abort_flag = 0u;
    for (uint32_t k = 0; k < L::kNumFill; ++k) c.fill()[k] = 0u;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    tmem_alloc_pair(base + L::kOffTmemSlot, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    if constexpr (C::kFp8) {
      tma_prefetch_desc(&p.tm_codes);
      tma_prefetch_desc(&p.tm_rope);
      tma_prefetch_desc(&p.tm_vcodes);
    } else {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
    }
    tma_prefetch_desc(&p.tm_q);
    if (!p.out_f32) tma_prefetch_desc(&p.tm_out);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // both CTAs' barriers exist before any remote arrival
  MLA_PRO(1);
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(c.gbase + L::kOffTmemSlot);
  c.peer_abort = map_to_rank(base + L::kOffAbort, c.cta ^ 1u);
  c.lead_bars = map_to_rank(base + L::kOffBar, 0);
  // Programmatic dependent launch: the set-up above overlapped the previous
  // kernel (the plan, or the previous call's combine); wait for its
  // completion before reading the plan or writing any output.  The combine
  // may launch from then on: it reads the plan at once and waits for this
  // kernel only before it reads the partials.
  griddep_wait();
  griddep_launch_dependents();
  MLA_PRO(2);

  // The plan must be the one built for this call's shape on this many pairs.
  // The header, this pair's record (its first segment and where its segments
  // start) and where they end are independent loads: one round trip.
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int pairs = static_cast<int>(gridDim.x >> 1);
  const MetaLayout lo = meta_layout(p.batch, p.h_q, p.s_q);
  const int4 hdr0 = *reinterpret_cast<const int4*>(p.meta);               // magic, error, pairs, work rows
  const int4 hdr2 = *reinterpret_cast<const int4*>(p.meta + 8);           // batch, kappa, splits, empties
  const int4 hdr3 = *reinterpret_cast<const int4*>(p.meta + 12);          // h_q, s_q, cap, -
  const int32_t* prec = p.meta + lo.pair_rec + kSegWords * pair;
  const int4 rec0 = *reinterpret_cast<const int4*>(prec);
  const int4 rec1 = *reinterpret_cast<const int4*>(prec + 4);
  const int s_end_raw = p.meta[lo.pair_off + pair + 1];
  static_assert(kHMagic == 0 && kHError == 1 && kHPairs == 2 && kHBatch == 8 && kHHq == 12 && kHSq == 13,
                "header words read as int4s");
  const bool plan_ok = hdr0.x == static_cast<int32_t>(kMagic) && hdr0.z == pairs && hdr2.x == p.batch &&
                       hdr3.x == p.h_q && hdr3.y == p.s_q;
  int s_begin = 0, s_end = 0;
  if (plan_ok) {
    s_begin = rec1.y;
    s_end = s_end_raw;
    // Bits the plan raised (lengths past the table, slot overflow) go to the
    // sticky word too.
    if (threadIdx.x == 0 && c.cta == 0 && pair == 0 && hdr0.y != 0)
      atomicOr(&g_mla_sticky_error, static_cast<unsigned int>(hdr0.y));
  } else if (threadIdx.x == 0 && c.cta == 0 && pair == 0) {
    set_error(c.meta, MLA_DEVERR_PLAN);
  }
  c.s_begin = s_begin;
  c.first = make_segment(p, rec0, rec1.x);

  if (threadIdx.x == 128) MLA_TRACE(11, 0);
#ifdef MLA_DECODE_TRACE
  if (threadIdx.x == 0 && c.cta == 0) g_mla_span[blockIdx.x >> 1][0] = globaltimer();
#endif
  if (warp == 0) {
    producer_k(p, c, s_begin, s_end);
  } else if (warp == 1) {
    if (lane == 0 && c.cta == 0) qk_issuer(p, c, tmem, s_begin, s_end);
    __syncwarp();
  } else if (warp == 2) {
    producer_v(p, c, s_begin, s_end);
  } else if (warp == 3) {
    if (lane == 0 && c.cta == 0) pv_issuer(p, c, tmem, s_begin, s_end);
    __syncwarp();
  } else if (warp < 12) {
    softmax_epilogue_then_drain(p, c, tmem, s_begin, s_end);
  } else {
    if constexpr (C::kFp8) key_converter(p, c, s_begin, s_end);
  }

  // ---- teardown: drain the pair MMAs, wait for the peer, free TMEM ----
  __syncthreads();
  if (warp == 3 && c.cta == 0 && lane == 0) umma_commit_pair(c.bar(L::kBarFinal), 0x1);  // PV issuer's MMAs
  if (warp == 1 && c.cta == 0) {
    if (lane == 0) {
      umma_commit_pair(c.bar(L::kBarFinal), 0x1);  // QK issuer's MMAs
      const uint64_t t0 = globaltimer();
      bool done = false;
      while (!(done = mbar_try_wait(c.bar(L::kBarFinal), 0)) && globaltimer() - t0 < kTimeoutNs) {
      }
      // MMAs that never completed are recorded; TMEM is still freed below:
      // a CTA that exits holding TMEM would leave the next kernel's
      // allocation on this SM pair waiting for good.
      if (!done) set_error(c.meta, MLA_DEVERR_TIMEOUT);
    }
    __syncwarp();
  }
#ifdef MLA_DECODE_TRACE
  if (threadIdx.x == 0 && c.cta == 0) {
    g_mla_span[blockIdx.x >> 1][1] = globaltimer();
    g_mla_span[blockIdx.x >> 1][2] = s_end - s_begin;
  }
#endif
  // On abort: wait for this CTA's copies still in flight; the fixed pause is
  // only a backstop for copies no barrier here can see (the other CTA's key
  // or Q boxes for a phase this CTA never posted).
  if (*c.abort_flag && threadIdx.x == 0) {
    drain_copies(c);
    __nanosleep(20000);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
  MLA_PRO(3);
}

}  // namespace

#ifdef MLA_DECODE_TRACE
extern "C" __attribute__((visibility("default"))) int mla_trace_read(void* host) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, g_mla_trace, sizeof(g_mla_trace)));
}
extern "C" __attribute__((visibility("default"))) int mla_trace_span(void* host) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, g_mla_span, sizeof(g_mla_span)));
}
extern "C" __attribute__((visibility("default"))) int mla_trace_pro(void* host) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, g_mla_pro, sizeof(g_mla_pro)));
}
extern "C" __attribute__((visibility("default"))) int mla_trace_abort(void* host) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, g_mla_abort, sizeof(g_mla_abort)));
}
extern "C" __attribute__((visibility("default"))) int mla_trace_stuck(void* stuck, void* step) {
  cudaError_t e = cudaMemcpyFromSymbol(stuck, g_mla_stuck, sizeof(g_mla_stuck));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(step, g_mla_step, sizeof(g_mla_step));
  return static_cast<int>(e);
}
extern "C" __attribute__((visibility("default"))) int mla_trace_clear() {
  static unsigned long long zero[4][24][512];
  return static_cast<int>(cudaMemcpyToSymbol(g_mla_trace, zero, sizeof(zero)));
}
#endif

size_t decode_kernel_smem_bytes(bool fp8) { return fp8 ? Lay<CfgFp8>::kSmemBytes : Lay<CfgBf16>::kSmemBytes; }

__device__ unsigned int g_mla_sticky_taken;

__global__ void take_sticky_kernel() { g_mla_sticky_taken = atomicExch(&g_mla_sticky_error, 0u); }

cudaError_t take_sticky_error(cudaStream_t stream, uint32_t* word) {
  take_sticky_kernel<<<1, 1, 0, stream>>>();
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess)
    e = cudaMemcpyFromSymbolAsync(word, g_mla_sticky_taken, sizeof(unsigned int), 0, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  return e;
}

namespace {

template <class C>
cudaError_t prepare_one() {
  return cudaFuncSetAttribute(mla_decode_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(Lay<C>::kSmemBytes));
}

// Co-resident 2-CTA clusters of one build of the kernel.
template <class C>
cudaError_t pairs_one(int sms, int* clusters) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1), 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Lay<C>::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaOccupancyMaxActiveClusters(clusters, mla_decode_kernel<C>, &cfg);
}

template <class C>
cudaError_t launch_one(const DecodeParams& p, int pairs, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Lay<C>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mla_decode_kernel<C>, p);
}

}  // namespace

cudaError_t decode_kernel_prepare() {
  cudaError_t e = prepare_one<CfgBf16>();
  if (e == cudaSuccess) e = prepare_one<CfgFp8>();
  return e;
}

// Both builds (bf16 and FP8 cache) run on the same pairs, as one plan serves
// both: the smaller of their co-resident cluster counts.
cudaError_t decode_kernel_pairs(int* pairs) {
  cudaError_t e = decode_kernel_prepare();
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  int c_bf16 = 0, c_fp8 = 0;
  if ((e = pairs_one<CfgBf16>(sms, &c_bf16)) != cudaSuccess) return e;
  if ((e = pairs_one<CfgFp8>(sms, &c_fp8)) != cudaSuccess) return e;
  int clusters = c_bf16 < c_fp8 ? c_bf16 : c_fp8;
  *pairs = clusters < kMaxPairs ? clusters : kMaxPairs;
  return cudaSuccess;
}

cudaError_t launch_decode(const DecodeParams& p, int pairs, cudaStream_t stream) {
  return p.fp8 ? launch_one<CfgFp8>(p, pairs, stream) : launch_one<CfgBf16>(p, pairs, stream);
}

}  // namespace mla
