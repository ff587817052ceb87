// Internal layout of the kernels around the decode: the projections either
// side of it (mla_absorb_q, mla_up_project) and the merge of a row split
// across GPUs (mla_merge_splits).
#pragma once

#include "mla_internal.h"

namespace mla {

// The projections either side of the decode (mla_absorb_q, mla_up_project).
// A CTA takes one head and a tile of tokens (up to kProjAbsorbTile for the
// absorb, kProjUpTile for the up-projection).
constexpr int kProjAbsorbTile = 128;
constexpr int kProjUpTile = 64;

// Token rows of a tile's box (the MMA's N): the token count rounded up to 16,
// capped at the tile.
__host__ __device__ inline int proj_box_rows(int tokens, int tile) {
  const int r = (tokens + 15) & ~15;
  return r < tile ? r : tile;
}

struct ProjParams {
  // absorb:     q_nope as (64 cols, tokens, 2 panels, h_q);
  // up-project: latent output as (64 cols, tokens, 8 panels, h_q);
  // box (64, nb, 2, 1): 2 panels of nb tokens of one head.
  CUtensorMap tm_a;
  // The per-head weights [h_q][512][128] as (64 cols, h_q * 512 rows, 2
  // panels): box (64, 128, 2), one 128-row chunk.
  CUtensorMap tm_b;
  const void* w;      // the weights' base address (for the L2 prefetch)
  const void* extra;  // absorb: q_rope [tokens][h_q][64] bf16 (copied through)
  void* out;          // absorb: [tokens][h_q][576]; up-project: [tokens][h_q][128]
  int tokens, h_q;
  int nb;             // proj_box_rows(tokens, tile)
};

// Merge of per-split decode results (mla_merge_splits).
struct MergeParams {
  const void* outs;   // [splits][batch][s_q][h_q][512], bf16 or (in_f32) fp32
  const float* lses;  // [splits][batch][h_q][s_q]
  void* out;          // bf16 [batch][s_q][h_q][512]
  float* lse;         // [batch][h_q][s_q]
  int splits, batch, s_q, h_q;
  int in_f32;
};

cudaError_t launch_projection(const ProjParams& p, bool absorb, cudaStream_t stream);
cudaError_t launch_merge(const MergeParams& p, int sms, cudaStream_t stream);
// One bounded wait that runs out (see mla_selftest_bounded_wait).
cudaError_t launch_wait_selftest(cudaStream_t stream);
// Reads and clears the projection kernels' sticky error bits.
cudaError_t take_project_sticky_error(cudaStream_t stream, uint32_t* word);

}  // namespace mla
