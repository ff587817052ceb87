// Tile-scheduler metadata kernel: the split-KV (flash-decoding) plan.
//
// "Unlocking GPU Potential: The Impact of FlashAttention and KV Cache
// Optimization in Long-Text Inference": at decode the query length is 1, so
// parallelism over (batch x query) alone leaves most SMs idle once the batch
// is smaller than the SM count; long rows must be split across SMs and the
// pieces merged.  "FlashMLA overview" (flash_api.cpp): the plan is computed
// once per decode step (get_mla_metadata) and reused by every layer.
//
// The plan is a cost-interval partition of all work rows' 64-token pages over
// the P SM pairs (2-CTA clusters):
//   * a work row is one batch row's tile of up to 128 query rows, ordered
//     m-tile major (w = mt * batch + i), so the m-tiles of one batch row, which
//     read the same pages, land on pairs far apart and run at the same time;
//   * a row with n > 0 pages costs n + kappa (kappa: fixed cost of starting a
//     row: Q load, pipeline fill, epilogue); C_w is the cost of the rows before
//     w and T the total;
//   * page b of row w sits at cost position C_w + kappa + b; pair p owns the
//     positions [B(p), B(p + 1)) with B(p) = floor(p T / P) when T >= P (each
//     pair gets floor(T / P) or ceil(T / P) positions, so none is idle) and
//     B(p) = min(p, T) otherwise, so every pair takes one contiguous range;
//   * a row whose pages land on k > 1 pairs is cut into k pieces with k
//     consecutive partial slots (row order); its output comes from the combine.
// Everything follows from prefix sums, so one CTA computes it with block-wide
// scans over chunks of 1024 rows (one pass when the rows fit one chunk); each
// row also writes the start offset of every pair whose range begins inside it.
#include "mla_internal.h"
#include "sm100_ptx.cuh"

namespace mla {

#ifdef MLA_DECODE_TRACE
// Profiling builds only: [entry, after the grid dependency, exit] of the last launch (globaltimer).
__device__ unsigned long long g_mla_sched_times[3];
#endif

namespace {

constexpr int kSchedThreads = 1024;  // the most threads a launch uses (and rows per chunk)
constexpr int kWarps = kSchedThreads / 32;

// Block-wide exclusive scan of one value per thread; returns the exclusive
// prefix and writes the block total to *total.  All threads must call it.
template <typename T>
__device__ T block_exclusive_scan(T v, T* warp_tot, T* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  T incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const T o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nwarps = static_cast<int>(blockDim.x >> 5);
    T t = lane < nwarps ? warp_tot[lane] : T(0);
    T ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const T o = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += o;
    }
    if (lane < nwarps) warp_tot[lane] = ti - t;  // exclusive warp offsets
    if (lane == nwarps - 1) *total = ti;
  }
  __syncthreads();
  const T res = warp_tot[warp] + incl - v;
  __syncthreads();
  return res;
}

// The pairs' cost boundaries B(p) (see the header), the pair owning cost
// position x (B(p) <= x < B(p + 1)), and the first pair p with B(p) >= x.
struct Bounds {
  long long T;
  int P;
  __device__ Bounds(long long T_, int P_) : T(T_), P(P_) {}
  __device__ long long b(long long p) const { return T >= P ? (p * T) / P : (p < T ? p : T); }
  __device__ long long owner(long long x) const { return T >= P ? ((x + 1) * P - 1) / T : x; }
  __device__ long long first_at_or_past(long long x) const { return T >= P ? (x * P + T - 1) / T : x; }
};

// Length of work row w's batch row (a negative length is flagged and read as 0).
// One work row of a chunk, as the segment and pair writers need it.
struct RowPlan {
  long long C;  // cost before the row
  long long c;  // its cost (0 for an empty row)
  int L, n;     // length and pages
  int f;        // pair of its first page
  int pieces;
  int seg0;     // its first segment, counted from the chunk's first
  int slot0;    // its first partial slot (split rows)
};

__device__ __forceinline__ int row_length(const int32_t* seqlens, int batch, int w, int* err) {
  int L = seqlens[w % batch];
  if (L < 0) {
    *err = 1;
    L = 0;
  }
  return L;
}

__global__ void __launch_bounds__(kSchedThreads) mla_sched_kernel(const int32_t* __restrict__ seqlens, int batch,
                                                                  int h_q, int s_q, int pairs, int32_t* meta) {
  // Programmatic dependent launch: the decode kernel may start its set-up now;
  // this kernel itself waits until the previous kernel in the stream (which
  // may still read the metadata, or have written the lengths) has completed.
#ifdef MLA_DECODE_TRACE
  if (threadIdx.x == 0) g_mla_sched_times[0] = ptx::globaltimer();
#endif
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
#ifdef MLA_DECODE_TRACE
  if (threadIdx.x == 0) g_mla_sched_times[1] = ptx::globaltimer();
#endif
  const MetaLayout lo = meta_layout(batch, h_q, s_q);
  const int W = lo.W;
  const int R = s_q * h_q;
  const int n_mt = ceil_div(R, kMTile);
  int32_t* pair_off = meta + lo.pair_off;
  int32_t* pair_rec = meta + lo.pair_rec;
  int32_t* segs = meta + lo.segs;
  int32_t* row_info = meta + lo.row_info;
  int32_t* split_rows = meta + lo.split_rows;
  int32_t* empty_rows = meta + lo.empty_rows;
  int32_t* tasks = meta + lo.tasks;

  __shared__ long long s_wl[kWarps];
  __shared__ unsigned long long s_wp[kWarps];
  __shared__ long long s_tot_l;
  __shared__ unsigned long long s_tot_p;
  __shared__ int s_err;
  __shared__ RowPlan s_row[kSchedThreads];
  if (threadIdx.x == 0) s_err = 0;
  int err = 0;
  const int nthr = static_cast<int>(blockDim.x);  // a multiple of 32, at most kSchedThreads
  const bool one_chunk = W <= nthr;

  // Pass 1: total cost T.  With at most one row per thread, the row's pages
  // and cost prefix are kept for pass 2 instead of being read and scanned
  // again.
  int L_own = 0, n_own = 0;
  long long C_own = 0, T = 0;
  if (one_chunk) {
    L_own = threadIdx.x < W ? row_length(seqlens, batch, threadIdx.x, &err) : 0;
    n_own = ceil_div(L_own, kPage);
    C_own = block_exclusive_scan<long long>(n_own > 0 ? n_own + kKappa : 0, s_wl, &s_tot_l);
    T = s_tot_l;
  } else {
    long long local = 0;
    for (int w = threadIdx.x; w < W; w += nthr) {
      const int n = ceil_div(row_length(seqlens, batch, w, &err), kPage);
      if (n > 0) local += n + kKappa;
    }
    block_exclusive_scan<long long>(local, s_wl, &s_tot_l);
    T = s_tot_l;
  }
  const long long cap = T > 0 ? (T + pairs - 1) / pairs : 1;  // the longest range (reported only)
  const Bounds bd(T, pairs);

  // Pass 2: per-row prefix sums, chunk by chunk with carries.  The four
  // counts (segments, partial slots, split rows, empty rows) are scanned
  // together as 16-bit fields of one 64-bit word: within a chunk of 1024 rows
  // each stays below 1024 + pairs.
  long long carry_cost = 0;
  int carry_seg = 0, carry_slot = 0, carry_split = 0, carry_empty = 0;
  for (int base = 0; base < W; base += nthr) {
    const int w = base + threadIdx.x;
    const bool in = w < W;
    int L, n;
    long long C, chunk_cost;
    if (one_chunk) {
      L = L_own;
      n = n_own;
      C = C_own;
      chunk_cost = T;
    } else {
      L = in ? row_length(seqlens, batch, w, &err) : 0;
      n = ceil_div(L, kPage);
      C = carry_cost + block_exclusive_scan<long long>(n > 0 ? n + kKappa : 0, s_wl, &s_tot_l);
      chunk_cost = s_tot_l;
    }
    const long long c = n > 0 ? n + kKappa : 0;
    int f = 0, pieces = 0;
    if (n > 0) {
      f = static_cast<int>(bd.owner(C + kKappa));
      const int l = static_cast<int>(bd.owner(C + kKappa + n - 1));
      pieces = l - f + 1;
    }
    const unsigned long long v = static_cast<unsigned long long>(pieces) |
                                 (static_cast<unsigned long long>(pieces > 1 ? pieces : 0) << 16) |
                                 (static_cast<unsigned long long>(pieces > 1 ? 1 : 0) << 32) |
                                 (static_cast<unsigned long long>(in && n == 0 ? 1 : 0) << 48);
    const unsigned long long pre = block_exclusive_scan<unsigned long long>(v, s_wp, &s_tot_p);
    const unsigned long long tot = s_tot_p;
    const int seg0 = carry_seg + static_cast<int>(pre & 0xffffu);
    const int slot0 = carry_slot + static_cast<int>((pre >> 16) & 0xffffu);
    const int split_i = carry_split + static_cast<int>((pre >> 32) & 0xffffu);
    const int empty_i = carry_empty + static_cast<int>((pre >> 48) & 0xffffu);
    if (in) {
      row_info[2 * w + 0] = pieces > 1 ? slot0 : -1;
      row_info[2 * w + 1] = pieces;
      if (pieces > 1) {
        split_rows[split_i] = w;
        *reinterpret_cast<int4*>(tasks + 4 * split_i) = make_int4(w, slot0, pieces, 0);
      }
      if (n == 0) empty_rows[empty_i] = w;
    }
    // The chunk's rows to shared memory; then every segment and every pair
    // whose range starts in the chunk is written by a thread of its own (a
    // long row's pieces and pairs would otherwise be one thread's serial
    // work), which finds its row by binary search.
    s_row[threadIdx.x] = RowPlan{C, c, L, n, f, pieces, seg0 - carry_seg, slot0};
    __syncthreads();
    const int rows_here = min(nthr, W - base);
    const int segs_here = static_cast<int>(tot & 0xffffu);
    for (int j = threadIdx.x; j < segs_here; j += nthr) {
      // the last row whose first segment is at or before j (it has pieces)
      int lo_r = 0, hi_r = rows_here - 1;
      while (lo_r < hi_r) {
        const int mid = (lo_r + hi_r + 1) >> 1;
        if (s_row[mid].seg0 <= j) lo_r = mid; else hi_r = mid - 1;
      }
      const RowPlan& rp = s_row[lo_r];
      const int k = j - rp.seg0;
      const long long p = rp.f + k;
      const long long b0 = bd.b(p) - rp.C - kKappa;
      const long long b1 = bd.b(p + 1) - rp.C - kKappa;
      int32_t* rec = segs + kSegWords * (carry_seg + j);
      *reinterpret_cast<int4*>(rec) =
          make_int4(base + lo_r, b0 > 0 ? static_cast<int>(b0) : 0, b1 < rp.n ? static_cast<int>(b1) : rp.n,
                    rp.pieces > 1 ? rp.slot0 + k : -1);
      *reinterpret_cast<int4*>(rec + 4) = make_int4(rp.L, 0, 0, 0);
    }
    // Pair p's segments start with the first one on a pair >= p.  When B(p)
    // falls in a row's cost range [C, C + c), every segment of the rows
    // before sits on a pair < p, and of this row's pieces (pairs f, f + 1,
    // ...) those before pair p; later rows start at or past p.  Its first
    // segment is then this row's piece p - f (a pair p < f ends inside the
    // row's fixed-cost positions and has no segment at all).
    for (int p = threadIdx.x; p < pairs; p += nthr) {
      const long long x = bd.b(p);
      if (x < carry_cost || x >= carry_cost + chunk_cost) continue;
      int lo_r = 0, hi_r = rows_here - 1;  // the last row whose cost range starts at or before x
      while (lo_r < hi_r) {
        const int mid = (lo_r + hi_r + 1) >> 1;
        if (s_row[mid].C <= x) lo_r = mid; else hi_r = mid - 1;
      }
      const RowPlan& rp = s_row[lo_r];
      const int s0 = carry_seg + rp.seg0 + (p > rp.f ? p - rp.f : 0);
      pair_off[p] = s0;
      int32_t* rec = pair_rec + kSegWords * p;
      if (p >= rp.f) {
        const long long b0 = x - rp.C - kKappa;
        const long long b1 = bd.b(p + 1) - rp.C - kKappa;
        *reinterpret_cast<int4*>(rec) =
            make_int4(base + lo_r, b0 > 0 ? static_cast<int>(b0) : 0, b1 < rp.n ? static_cast<int>(b1) : rp.n,
                      rp.pieces > 1 ? rp.slot0 + (p - rp.f) : -1);
        *reinterpret_cast<int4*>(rec + 4) = make_int4(rp.L, s0, 0, 0);
      } else {
        *reinterpret_cast<int4*>(rec) = make_int4(-1, 0, 0, -1);
        *reinterpret_cast<int4*>(rec + 4) = make_int4(0, s0, 0, 0);
      }
    }
    __syncthreads();  // s_row is rewritten by the next chunk
    carry_cost += chunk_cost;
    carry_seg += static_cast<int>(tot & 0xffffu);
    carry_slot += static_cast<int>((tot >> 16) & 0xffffu);
    carry_split += static_cast<int>((tot >> 32) & 0xffffu);
    carry_empty += static_cast<int>((tot >> 48) & 0xffffu);
  }
  if (err) s_err = 1;
  // Pairs whose range starts at the total cost (the end marker, and when
  // T < P the pairs past T) take no segment.
  const long long p_tail = bd.first_at_or_past(T);
  for (int p = threadIdx.x; p <= pairs; p += nthr) {
    if (p >= p_tail) {
      pair_off[p] = carry_seg;
      if (p < pairs) {
        *reinterpret_cast<int4*>(pair_rec + kSegWords * p) = make_int4(-1, 0, 0, -1);
        *reinterpret_cast<int4*>(pair_rec + kSegWords * p + 4) = make_int4(0, carry_seg, 0, 0);
      }
    }
  }
  __syncthreads();  // s_err

  if (threadIdx.x == 0) {
    uint32_t e = s_err ? MLA_DEVERR_SEQLEN : 0u;
    if (carry_slot > max_slots(pairs)) e |= MLA_DEVERR_PLAN;
    meta[kHMagic] = static_cast<int32_t>(kMagic);
    meta[kHError] = static_cast<int32_t>(e);
    meta[kHPairs] = pairs;
    meta[kHWorkRows] = W;
    meta[kHSegments] = carry_seg;
    meta[kHSlots] = carry_slot;
    meta[kHRows] = R;
    meta[kHMTiles] = n_mt;
    meta[kHBatch] = batch;
    meta[kHKappa] = kKappa;
    meta[kHSplitRows] = carry_split;
    meta[kHEmptyRows] = carry_empty;
    meta[kHHq] = h_q;
    meta[kHSq] = s_q;
    meta[kHCap] = static_cast<int32_t>(cap < 0x7fffffffLL ? cap : 0x7fffffffLL);
  }
#ifdef MLA_DECODE_TRACE
  __syncthreads();
  if (threadIdx.x == 0) g_mla_sched_times[2] = ptx::globaltimer();
#endif
}

}  // namespace

#ifdef MLA_DECODE_TRACE
extern "C" __attribute__((visibility("default"))) int mla_trace_sched_times(void* host) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, g_mla_sched_times, sizeof(g_mla_sched_times)));
}
#endif

cudaError_t launch_sched(const int32_t* seqlens, int batch, int h_q, int s_q, int pairs, int32_t* meta,
                         cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  // One thread per work row (and at least one per pair), up to kSchedThreads:
  // small plans then pay for few warps at every block-wide scan.
  const int W = batch * ceil_div(s_q * h_q, kMTile);
  int threads = (W > pairs + 1 ? W : pairs + 1) + 31;
  threads = threads & ~31;
  if (threads > kSchedThreads) threads = kSchedThreads;
  cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mla_sched_kernel, seqlens, batch, h_q, s_q, pairs, meta);
}

}  // namespace mla
