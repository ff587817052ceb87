"""The long-row split on the GPU: mla_merge_splits against the oracle's
log-sum-exp combine, and the whole split (each rank's plan and decode on its
share of the pages, then the merge) emulated rank by rank on one GPU against
the oracle's unsplit decode.  The exchange between GPUs is torch.distributed
and is covered on CPU ranks in tests/test_longrow.py.

Tolerances.  The merge reads bf16 (mla_merge_splits) or fp32
(mla_merge_splits_f32) partial outputs and fp32 lse values, merges in fp32 and
rounds once to bf16: |out - oracle| <= 2^-8 |oracle| + 1e-5 and
|lse - oracle| <= 1e-5 (1 + |lse|).  The emulated split runs each rank's
decode with fp32 output (mla_decode_f32) and merges the fp32 partials, so
nothing is rounded before the merge: the merge weights sum to one and the
merged error stays within an unsplit decode's.  The result is held to the
unsplit decode's bars: mean-abs 1e-3 and lse 1e-3, and per element the larger
of 8e-3 and the bf16-weight bound of parity_bounds, which exceeds 8e-3 only on
rows where a few tokens carry the weight (the cases below include rows of 1
to 3 tokens, causal); the long-context workload's split is held to 8e-3.
"""

import numpy as np
import pytest
import torch

from mla_decode_attention_13_b200 import binding, inputs, longrow
from oracle import mla_oracle
from parity_bounds import bf16_weight_bound

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("f32", [False, True])
@pytest.mark.parametrize("splits,batch,s_q,h_q", [(1, 2, 1, 16), (2, 3, 2, 16), (5, 2, 1, 128), (8, 1, 4, 4)])
def test_merge_matches_oracle_combine(splits, batch, s_q, h_q, f32):
    gen = torch.Generator()
    gen.manual_seed(splits * 100 + batch * 10 + s_q)
    outs = torch.randn(splits, batch, s_q, h_q, 512, generator=gen) * 0.25
    if not f32:
        outs = outs.to(torch.bfloat16)
    lses = torch.randn(splits, batch, h_q, s_q, generator=gen) * 3.0
    # a split with no visible token for some rows, and one row empty everywhere
    if splits > 1:
        lses[1, 0, : h_q // 2, 0] = -float("inf")
        outs[1, 0, 0, : h_q // 2] = 0
    lses[:, -1, -1, -1] = -float("inf")
    outs[:, -1, -1, -1] = 0
    merge = binding.mla_merge_splits_f32 if f32 else binding.mla_merge_splits
    out, lse = merge(outs.cuda(), lses.cuda())
    torch.cuda.synchronize()
    rows = batch * s_q * h_q
    parts = [(mla_oracle.as_f64(outs[k]).reshape(rows, 512),
              mla_oracle.as_f64(lses[k]).transpose(0, 2, 1).reshape(rows)) for k in range(splits)]
    want_out, want_lse = mla_oracle.combine_partials(parts)
    got = mla_oracle.as_f64(out.cpu()).reshape(rows, 512)
    got_lse = mla_oracle.as_f64(lse.cpu()).transpose(0, 2, 1).reshape(rows)
    assert np.all(np.abs(got - want_out) <= 2.0 ** -8 * np.abs(want_out) + 1e-5)
    assert np.array_equal(np.isneginf(got_lse), np.isneginf(want_lse))
    fin = np.isfinite(want_lse)
    assert np.all(np.abs(got_lse[fin] - want_lse[fin]) <= 1e-5 * (1 + np.abs(want_lse[fin])))
    assert np.all(got[~fin] == 0)


CASES = [
    # (lengths, h_q, s_q, causal)
    ([5000, 70, 1, 0, 3000], 16, 1, False),
    ([2000, 130, 65, 3], 32, 2, True),
    ([700, 64, 129], 128, 1, False),
]


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_split_decode_emulated_on_one_gpu_matches_unsplit_oracle(world, case):
    lens, h_q, s_q, causal = CASES[case]
    x = inputs.make_inputs(lens, h_q, s_q, seed=40 + case, causal=causal)
    g = x.to("cuda")
    outs, lses = [], []
    for rank in range(world):
        table, local = longrow.shard_block_table(g.block_table, lens, world, rank, s_q)
        meta = binding.mla_get_metadata(local, h_q, s_q)
        o, l = binding.mla_decode_f32(g.q, g.kv_cache, table, local, x.softmax_scale, causal and rank == world - 1,
                                      meta)
        assert binding.mla_check_device_error(meta) == 0
        outs.append(o)
        lses.append(l)
    out, lse = binding.mla_merge_splits_f32(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    want_out, want_lse = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, causal)
    got = mla_oracle.as_f64(out.cpu())
    err = np.abs(got - want_out)
    tol = np.maximum(8e-3, bf16_weight_bound(x, want_out, list(range(x.batch))))
    assert (err <= tol).all() and err.mean() <= 1e-3, (err.max(), err.mean())
    got_lse = mla_oracle.as_f64(lse.cpu())
    assert np.array_equal(np.isneginf(got_lse), np.isneginf(want_lse))
    fin = np.isfinite(want_lse)
    assert np.max(np.abs(got_lse[fin] - want_lse[fin])) <= 1e-3


def test_split_of_the_long_context_workload_at_full_size():
    # b4_h16_L128k-1k (rows of 131072, 1024, 32768 and 8192 tokens, 16 heads)
    # over 4 emulated ranks, every output against the oracle's unsplit decode.
    x = inputs.workload_inputs("b4_h16_L128k-1k")
    lens = [int(v) for v in x.seqlens]
    g = x.to("cuda")
    world = 4
    outs, lses = [], []
    for rank in range(world):
        table, local = longrow.shard_block_table(g.block_table, lens, world, rank, x.s_q)
        meta = binding.mla_get_metadata(local, x.h_q, x.s_q)
        o, l = binding.mla_decode_f32(g.q, g.kv_cache, table, local, x.softmax_scale,
                                      x.causal and rank == world - 1, meta)
        assert binding.mla_check_device_error(meta) == 0
        outs.append(o)
        lses.append(l)
    out, lse = binding.mla_merge_splits_f32(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    want_out, want_lse = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal)
    err = np.abs(mla_oracle.as_f64(out.cpu()) - want_out)
    assert err.max() <= 8e-3 and err.mean() <= 1e-3, (err.max(), err.mean())
    assert np.max(np.abs(mla_oracle.as_f64(lse.cpu()) - want_lse)) <= 1e-3


def test_decode_f32_rounds_to_the_bf16_decode():
    # mla_decode_f32 is the same attention as mla_decode with the output left
    # unrounded: rounding it to bf16 gives mla_decode's output bit for bit (the
    # split rows' fp32 merge and the unsplit rows' epilogue compute the same
    # values in both), and the lse values are identical.
    lens = [5000, 70, 1, 0, 3000, 129]
    for h_q, s_q, causal in ((16, 1, False), (128, 2, True)):
        x = inputs.make_inputs(lens, h_q, s_q, seed=91 + h_q, causal=causal)
        g = x.to("cuda")
        meta = binding.mla_get_metadata(g.seqlens, h_q, s_q)
        o16, l16 = binding.mla_decode(g.q, g.kv_cache, g.block_table, g.seqlens, x.softmax_scale, causal, meta)
        o32, l32 = binding.mla_decode_f32(g.q, g.kv_cache, g.block_table, g.seqlens, x.softmax_scale, causal, meta)
        torch.cuda.synchronize()
        assert binding.mla_check_device_error(meta) == 0
        assert torch.equal(o32.to(torch.bfloat16).view(torch.int16), o16.view(torch.int16))
        assert torch.equal(l32, l16)


def test_decode_sharded_on_one_rank_equals_the_unsplit_call():
    # Without a process group (one rank) the exchange is the identity and the
    # merge of a single fp32 split rounds it once: mla_decode's result exactly
    # (out, the same bf16 rounding of the same fp32 values) and its lse.
    lens = [900, 64, 1]
    x = inputs.make_inputs(lens, 32, 2, seed=77, causal=True)
    g = x.to("cuda")
    table, local = longrow.shard_block_table(g.block_table, lens, 1, 0, x.s_q)
    out, lse = longrow.decode_sharded(g.q, g.kv_cache, table, local, x.softmax_scale, True)
    meta = binding.mla_get_metadata(g.seqlens, x.h_q, x.s_q)
    ref_out, ref_lse = binding.mla_decode(g.q, g.kv_cache, g.block_table, g.seqlens, x.softmax_scale, True, meta)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)
    assert torch.allclose(lse, ref_lse, rtol=0, atol=1e-6) or torch.equal(lse, ref_lse)
