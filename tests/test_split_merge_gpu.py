"""Split rows of one, two, three and many pieces in one call, against the fp64
oracle, with one plan serving several calls.

A row the plan cuts into pieces is merged with exact log-sum-exp weights
("Unlocking GPU Potential: The Impact of FlashAttention and KV Cache
Optimization in Long-Text Inference", split and merge): each piece writes its
fp32 partial (O / l, lse) to the workspace and the combine kernel merges
them.  The lengths are chosen, from the oracle's plan for this GPU's SM pairs and
the plan's fixed per-piece cost, to give rows of one, two, three and many
pieces, plus an empty row; one plan serves three bf16 calls and one fp32
call.

Bars: those of the other parity tests (mean-abs 1e-3, |lse difference|
1e-3, per element the larger of 8e-3 and parity_bounds.bf16_weight_bound);
the fp32 output (mla_decode_f32) skips the final bf16 rounding, so it is held
to the same bound, and its bf16 rounding must equal the bf16 call's output.
Calls that reuse one plan must give the same bits.
"""

import numpy as np
import pytest
import torch

from mla_decode_attention_13_b200 import binding, inputs
from oracle import mla_oracle
from parity_bounds import bf16_weight_bound

pytestmark = pytest.mark.gpu

BASE_LENS = [30000, 15000, 10000, 5000, 0, 64, 500, 1000, 1250, 1500]


def plan_pieces(lens, h_q, s_q, kappa):
    plan = mla_oracle.split_plan(lens, h_q, s_q, binding.mla_num_sm_pairs(), kappa)
    return plan["pieces"]


def lengths_with_every_piece_count(h_q, s_q, kappa):
    """BASE_LENS with its ninth row's length moved until the plan (this GPU's
    pairs, the plan's fixed per-piece cost) has rows of 0, 1, 2, 3 and more
    than 3 pieces."""
    for L in range(1250, 8000, 50):
        lens = BASE_LENS[:8] + [L] + BASE_LENS[9:]
        pc = plan_pieces(lens, h_q, s_q, kappa)
        if {0, 1, 2, 3} <= set(pc) and max(pc) > 3:
            return lens
    raise AssertionError("no length set gives every piece count")


def check(x, out, lse, want_o, want_l, tol):
    got_o = out.double().numpy()
    d = np.abs(got_o - want_o)
    assert np.isfinite(got_o).all()
    assert (d <= tol).all(), f"max-abs {d.max():.3e}"
    assert d.mean() <= 1e-3, f"mean-abs {d.mean():.3e}"
    got_l = lse.double().numpy()
    inf = np.isneginf(want_l)
    assert np.array_equal(np.isneginf(got_l), inf)
    assert np.abs(got_l[~inf] - want_l[~inf]).max() <= 1e-3


@pytest.mark.parametrize("h_q,s_q,causal", [(128, 1, False), (64, 1, False), (16, 2, True)])
def test_rows_of_few_and_many_pieces(h_q, s_q, causal):
    probe = torch.tensor(BASE_LENS, dtype=torch.int32, device="cuda")
    kappa = int(binding.mla_get_metadata(probe, h_q, s_q).cpu()[9])  # the plan's fixed per-piece cost
    lens = lengths_with_every_piece_count(h_q, s_q, kappa)
    x = inputs.make_inputs(lens, h_q, s_q, seed=80 + h_q + s_q, causal=causal)
    g = x.to("cuda")
    meta = binding.mla_get_metadata(g.seqlens, h_q, s_q)
    pieces = plan_pieces(lens, h_q, s_q, kappa)
    assert {0, 1, 2, 3} <= set(pieces) and max(pieces) > 3, pieces
    results = []
    for _ in range(3):  # one plan, three calls
        out, lse = binding.mla_decode(g.q, g.kv_cache, g.block_table, g.seqlens, x.softmax_scale, causal, meta)
        results.append((out.cpu(), lse.cpu()))
    assert binding.mla_check_device_error(meta) == 0
    out, lse = results[0]
    for o, l in results[1:]:
        assert torch.equal(o, out) and torch.equal(l, lse)
    want_o, want_l = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal)
    tol = np.maximum(8e-3, bf16_weight_bound(x, want_o, list(range(x.batch))))
    check(x, out, lse, want_o, want_l, tol)
    o32, l32 = binding.mla_decode_f32(g.q, g.kv_cache, g.block_table, g.seqlens, x.softmax_scale, causal, meta)
    assert binding.mla_check_device_error(meta) == 0
    check(x, o32.cpu(), l32.cpu(), want_o, want_l, tol)
    # the bf16 output is the fp32 one rounded once
    assert torch.equal(o32.cpu().to(torch.bfloat16), out)
    assert torch.equal(l32.cpu(), lse)
