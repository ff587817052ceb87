"""One long row split across GPUs: each rank decodes the pages it holds, the
(out, lse) pairs are exchanged, and mla_merge_splits merges them.

"Unlocking GPU Potential: The Impact of FlashAttention and KV Cache
Optimization in Long-Text Inference" splits the keys of a decode step into
chunks that are attended to separately and merged by their log-sum-exp, so
that a small batch still fills the processors.  Across GPUs a chunk is one
rank's share of every row's cache: a long context whose cache exceeds one GPU's
memory, or a latency-bound step spread over several GPUs.

The shard rule (page-aligned, contiguous):
  * row i has n = ceil(L_i / 64) pages; rank r holds pages [b_r, b_{r+1}) with
    b_r = min(floor(r n / W), cap) for 0 < r < W, b_0 = 0, b_W = n;
  * cap = floor(max(L_i - s_q + 1, 0) / 64) keeps every token of ranks
    0..W-2 visible to every query token of a causal step (query token t sees
    cache positions j <= L_i - s_q + t), so those ranks decode with causal = 0
    and only rank W - 1, which holds the row's last tokens, applies the mask,
    with its local length L_i - 64 b_{W-1}: its mask then equals the global one
    shifted by 64 b_{W-1} positions.
Ranks with no pages of a row get lse = -inf for it, which the merge ignores.

The partial results cross between ranks unrounded: each rank decodes with
mla_decode_f32 (fp32 out, 2052 bytes per query row with its lse) and
mla_merge_splits_f32 merges them in fp32 and rounds once to bf16, so the split
result keeps the error bars of an unsplit decode.

Only host logic lives here: the compute is the library's kernels
(mla_get_metadata, mla_decode_f32, mla_merge_splits_f32) and the exchange is
torch.distributed (NCCL between GPUs).
"""

from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import binding

PAGE = 64


def shard_bounds(length: int, world: int, s_q: int = 1) -> List[int]:
    """Page boundaries b_0..b_W of one row of ``length`` tokens over ``world`` ranks."""
    if world < 1:
        raise ValueError("world must be >= 1")
    length = max(int(length), 0)
    n = (length + PAGE - 1) // PAGE
    cap = max(length - int(s_q) + 1, 0) // PAGE
    b = [0] * (world + 1)
    for r in range(1, world):
        b[r] = min(r * n // world, cap)
    b[world] = n
    return b


def shard_lengths(seqlens: Sequence[int], world: int, s_q: int = 1) -> List[List[int]]:
    """Tokens of each row held by each rank: [world][batch]."""
    out = [[0] * len(seqlens) for _ in range(world)]
    for i, L in enumerate(seqlens):
        L = max(int(L), 0)
        b = shard_bounds(L, world, s_q)
        for r in range(world):
            out[r][i] = max(0, min(b[r + 1] * PAGE, L) - b[r] * PAGE)
    return out


def shard_block_table(block_table: torch.Tensor, seqlens: Sequence[int], world: int, rank: int,
                      s_q: int = 1) -> Tuple[torch.Tensor, torch.Tensor]:
    """Rank ``rank``'s block table and lengths, cut from a whole-row table.

    Row i keeps the page ids block_table[i][b_r : b_{r+1}] (in order; the rest
    of the row repeats its last entry, or the row's first entry if it has none,
    and is never read).  The page ids stay those of the whole table: a rank
    that owns a pool of its own renumbers them into it.
    """
    table = block_table.cpu()
    lens = [max(int(x), 0) for x in seqlens]
    local_lens = shard_lengths(lens, world, s_q)[rank]
    cuts = [shard_bounds(L, world, s_q) for L in lens]
    width = max([c[rank + 1] - c[rank] for c in cuts] + [1])
    local = torch.empty(len(lens), width, dtype=table.dtype)
    for i, c in enumerate(cuts):
        pages = table[i, c[rank]:c[rank + 1]]
        fill = pages[-1] if pages.numel() else table[i, 0]
        local[i] = fill
        local[i, :pages.numel()] = pages
    return local.to(block_table.device), torch.tensor(local_lens, dtype=torch.int32, device=block_table.device)


def gather_partials(out_r: torch.Tensor, lse_r: torch.Tensor,
                    group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Every rank's (out, lse), stacked in rank order on every rank."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    if world == 1:
        return out_r.unsqueeze(0).contiguous(), lse_r.unsqueeze(0).contiguous()
    outs = torch.empty((world,) + tuple(out_r.shape), dtype=out_r.dtype, device=out_r.device)
    lses = torch.empty((world,) + tuple(lse_r.shape), dtype=lse_r.dtype, device=lse_r.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(outs, out_r.contiguous(), group=group)
        dist.all_gather_into_tensor(lses, lse_r.contiguous(), group=group)
    else:
        dist.all_gather(list(outs.unbind(0)), out_r.contiguous(), group=group)
        dist.all_gather(list(lses.unbind(0)), lse_r.contiguous(), group=group)
    return outs, lses


def decode_sharded(q: torch.Tensor, kv_cache: torch.Tensor, local_table: torch.Tensor, local_seqlens: torch.Tensor,
                   softmax_scale: float, causal: bool, group=None,
                   metadata: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's share of a split decode step, exchanged and merged.

    ``local_table`` and ``local_seqlens`` come from shard_block_table (or the
    same rule applied when the pages were placed).  Returns the merged
    (out, lse) on every rank.  Everything runs on torch's current stream, the
    one the collectives are ordered with.
    """
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    _, s_q, h_q, _ = q.shape
    meta = binding.mla_get_metadata(local_seqlens, h_q, s_q, metadata=metadata)
    out_r, lse_r = binding.mla_decode_f32(q, kv_cache, local_table, local_seqlens, softmax_scale,
                                          bool(causal) and rank == world - 1, meta)
    outs, lses = gather_partials(out_r, lse_r, group)
    return binding.mla_merge_splits_f32(outs, lses)
