"""The long-row split on the GPU: mla_merge_splits against the oracle's
log-sum-exp combine, and the whole split (each rank's plan and decode on its
share of the pages, then the merge) emulated rank by rank on one GPU against
the oracle's unsplit decode.  The exchange between GPUs is torch.distributed
and is covered on CPU ranks in tests/test_longrow.py.

Tolerances.  The merge reads bf16 partial outputs and fp32 lse values, merges
in fp32 and rounds once to bf16: |out - oracle| <= 2^-8 |oracle| + 1e-5 and
|lse - oracle| <= 1e-5 (1 + |lse|).  For the emulated split each rank's decode
is held to the decode bars (max-abs 8e-3, mean-abs 1e-3, lse 1e-3); the merge
weights sum to one, so the merged error is within the same bars plus the bf16
rounding of the partial outputs and of the result, 2^-9 (max_k |out_k| +
|out|), which the max-abs bar adds.
"""

import numpy as np
import pytest
import torch

from mla_decode_attention_13_b200 import binding, inputs, longrow
from oracle import mla_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("splits,batch,s_q,h_q", [(1, 2, 1, 16), (2, 3, 2, 16), (5, 2, 1, 128), (8, 1, 4, 4)])
def test_merge_matches_oracle_combine(splits, batch, s_q, h_q):
    gen = torch.Generator()
    gen.manual_seed(splits * 100 + batch * 10 + s_q)
    outs = (torch.randn(splits, batch, s_q, h_q, 512, generator=gen) * 0.25).to(torch.bfloat16)
    lses = torch.randn(splits, batch, h_q, s_q, generator=gen) * 3.0
    # a split with no visible token for some rows, and one row empty everywhere
    if splits > 1:
        lses[1, 0, : h_q // 2, 0] = -float("inf")
        outs[1, 0, 0, : h_q // 2] = 0
    lses[:, -1, -1, -1] = -float("inf")
    outs[:, -1, -1, -1] = 0
    out, lse = binding.mla_merge_splits(outs.cuda(), lses.cuda())
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
        o, l = binding.mla_decode(g.q, g.kv_cache, table, local, x.softmax_scale, causal and rank == world - 1, meta)
        assert binding.mla_check_device_error(meta) == 0
        outs.append(o)
        lses.append(l)
    out, lse = binding.mla_merge_splits(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    want_out, want_lse = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, causal)
    got = mla_oracle.as_f64(out.cpu())
    err = np.abs(got - want_out)
    parts_max = max(float(o.abs().max()) for o in outs)
    bar = 8e-3 + 2.0 ** -9 * (parts_max + float(np.abs(want_out).max()))
    assert err.max() <= bar and err.mean() <= 1e-3, (err.max(), bar, err.mean())
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
        o, l = binding.mla_decode(g.q, g.kv_cache, table, local, x.softmax_scale, x.causal and rank == world - 1, meta)
        assert binding.mla_check_device_error(meta) == 0
        outs.append(o)
        lses.append(l)
    out, lse = binding.mla_merge_splits(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    want_out, want_lse = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal)
    err = np.abs(mla_oracle.as_f64(out.cpu()) - want_out)
    parts_max = max(float(o.abs().max()) for o in outs)
    bar = 8e-3 + 2.0 ** -9 * (parts_max + float(np.abs(want_out).max()))
    assert err.max() <= bar and err.mean() <= 1e-3, (err.max(), bar, err.mean())
    assert np.max(np.abs(mla_oracle.as_f64(lse.cpu()) - want_lse)) <= 1e-3


def test_decode_sharded_on_one_rank_equals_the_unsplit_call():
    # Without a process group (one rank) the exchange is the identity and the
    # merge of a single split must reproduce mla_decode's result exactly
    # (lse) and to the bf16 rounding of a value that is already bf16 (out).
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
