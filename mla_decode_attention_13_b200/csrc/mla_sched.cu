// Tile-scheduler metadata kernel: the split-KV (flash-decoding) plan.
//
// "Unlocking GPU Potential: The Impact of FlashAttention and KV Cache
// Optimization in Long-Text Inference": at decode the query length is 1, so
// parallelism over (batch x query) alone leaves most SMs idle once the batch
// is smaller than the SM count; long rows must be split across SMs and the
// pieces merged.  "FlashMLA overview" (flash_api.cpp): the plan is computed
// once per decode step (get_mla_metadata) and reused by every layer.
//
// The plan cuts the concatenation of all work rows' 64-token pages into one
// contiguous range per SM pair (2-CTA cluster):
//   * a work row is one batch row's tile of up to 128 query rows; work rows
//     are ordered m-tile major, w = mt * batch + i, so the m-tiles of one batch
//     row (which read the same pages) land on pairs far apart in the order and
//     run at about the same time;
//   * a row with n pages costs n + kappa (kappa: fixed per-piece cost: Q load,
//     pipeline fill, epilogue), T is the total, and each pair may hold
//     cap = ceil(T / P) + 2 kappa;
//   * walking rows in order, the current pair takes as many pages of the row as
//     fit in cap - used - kappa (at least one); when nothing fits, the next pair
//     starts; the last pair takes whatever is left;
//   * a row cut into k > 1 pieces gets k consecutive partial slots (row order).
// One CTA: all threads compute the page counts and their total, then thread 0
// walks the rows (O(W + P) steps).
#include "mla_internal.h"

namespace mla {
namespace {

constexpr int kSchedThreads = 256;
constexpr int kSmemRows = 8192;

__global__ void __launch_bounds__(kSchedThreads) mla_sched_kernel(const int32_t* __restrict__ seqlens, int batch,
                                                                  int h_q, int s_q, int pairs, int32_t* meta) {
  const MetaLayout lo = meta_layout(batch, h_q, s_q);
  const int W = lo.W;
  const int R = s_q * h_q;
  const int n_mt = ceil_div(R, kMTile);
  int32_t* pair_off = meta + lo.pair_off;
  int32_t* segs = meta + lo.segs;
  int32_t* row_info = meta + lo.row_info;
  int32_t* split_rows = meta + lo.split_rows;
  int32_t* empty_rows = meta + lo.empty_rows;

  __shared__ int32_t s_pages[kSmemRows];
  __shared__ long long s_red[kSchedThreads / 32];
  __shared__ int s_err;
  // Pages per work row live in shared memory when they fit, else in the
  // empty_rows area (rewritten after the walk).
  int32_t* pages = (W <= kSmemRows) ? s_pages : empty_rows;

  if (threadIdx.x == 0) s_err = 0;
  __syncthreads();
  long long local = 0;
  for (int w = threadIdx.x; w < W; w += blockDim.x) {
    const int i = w % batch;
    int L = seqlens[i];
    if (L < 0) {
      s_err = 1;
      L = 0;
    }
    const int n = ceil_div(L, kPage);
    pages[w] = n;
    if (n > 0) local += n + kKappa;
  }
  for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(0xffffffffu, local, off);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = local;
  __syncthreads();
  if (threadIdx.x != 0) return;

  long long T = 0;
  for (int k = 0; k < kSchedThreads / 32; ++k) T += s_red[k];
  const long long cap = (T + pairs - 1) / pairs + 2 * kKappa;

  int p = 0, nseg = 0, nslots = 0;
  long long used = 0;
  for (int k = 0; k <= pairs; ++k) pair_off[k] = 0;
  for (int w = 0; w < W; ++w) {
    const int n = pages[w];
    const int first = nseg;
    int b0 = 0;
    while (b0 < n) {
      const long long room = cap - used - kKappa;
      if (room < 1 && p < pairs - 1) {
        ++p;
        pair_off[p] = nseg;
        used = 0;
        continue;
      }
      long long take = n - b0;
      if (p != pairs - 1) {
        const long long fit = room > 1 ? room : 1;
        if (fit < take) take = fit;
      }
      int32_t* s = segs + 4 * nseg;
      s[0] = w;
      s[1] = b0;
      s[2] = b0 + static_cast<int>(take);
      s[3] = -1;
      ++nseg;
      used += take + kKappa;
      b0 += static_cast<int>(take);
    }
    const int pieces = nseg - first;
    row_info[2 * w + 0] = -1;
    row_info[2 * w + 1] = pieces;
    if (pieces > 1) {
      row_info[2 * w + 0] = nslots;
      for (int k = 0; k < pieces; ++k) segs[4 * (first + k) + 3] = nslots + k;
      nslots += pieces;
    }
  }
  // Pairs after the last one that received work own empty ranges.
  for (int k = p + 1; k <= pairs; ++k) pair_off[k] = nseg;

  int n_split = 0, n_empty = 0;
  for (int w = 0; w < W; ++w) {
    const int pieces = row_info[2 * w + 1];
    if (pieces > 1) split_rows[n_split++] = w;
  }
  for (int w = 0; w < W; ++w) {
    if (row_info[2 * w + 1] == 0) empty_rows[n_empty++] = w;
  }

  uint32_t err = s_err ? MLA_DEVERR_SEQLEN : 0u;
  if (nslots > max_slots(pairs)) err |= MLA_DEVERR_PLAN;
  meta[kHMagic] = static_cast<int32_t>(kMagic);
  meta[kHError] = static_cast<int32_t>(err);
  meta[kHPairs] = pairs;
  meta[kHWorkRows] = W;
  meta[kHSegments] = nseg;
  meta[kHSlots] = nslots;
  meta[kHRows] = R;
  meta[kHMTiles] = n_mt;
  meta[kHBatch] = batch;
  meta[kHKappa] = kKappa;
  meta[kHSplitRows] = n_split;
  meta[kHEmptyRows] = n_empty;
  meta[kHHq] = h_q;
  meta[kHSq] = s_q;
  meta[kHCap] = static_cast<int32_t>(cap);
}

}  // namespace

cudaError_t launch_sched(const int32_t* seqlens, int batch, int h_q, int s_q, int pairs, int32_t* meta,
                         cudaStream_t stream) {
  mla_sched_kernel<<<1, kSchedThreads, 0, stream>>>(seqlens, batch, h_q, s_q, pairs, meta);
  return cudaGetLastError();
}

}  // namespace mla
