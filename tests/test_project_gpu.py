"""Parity of the projections either side of the absorbed decode (through the
C ABI) with the fp64 oracle.

Tolerances.  Each output element is one dot product of bf16 operands (128
products for the absorbed query, 512 for the up-projection), accumulated in
fp32 on the tensor cores and rounded to bf16 once.  The products of two bf16
numbers are exact in fp32; accumulating n of them costs at most about
n * 2^-24 * sum |terms| (under 5e-4 for these draws, whose sum |terms| stays
below 20), and the final rounding at most half a bf16 unit, 2^-8 |x|.  So
    |gpu - oracle| <= 2^-8 |oracle| + 5e-4
element by element, and the rope columns of the absorbed query are copied, so
they match bit for bit.  Nearly every element must also equal the oracle's
value rounded to bf16 (the two differ only where the fp32 sum and the exact one
straddle a rounding boundary).

The layer test chains absorb -> decode -> up-project on the GPU and compares
with the unabsorbed definition (keys and values up-projected per head) in fp64.
W_UV's columns have unit norm in expectation, so the up-projection carries the
decode's own error through at about its size, and the absorbed query's bf16
rounding adds an error of the same order: the bars are twice the decode's
(max-abs 1.6e-2, mean-abs 2e-3).
"""

import numpy as np
import pytest
import torch

from mla_decode_attention_13_b200 import binding, inputs
from oracle import mla_oracle

pytestmark = pytest.mark.gpu

ATOL = 5e-4
RTOL = 2.0 ** -8
MIN_EXACT = 0.98

# (tokens, h_q): one token; every decode workload's tokens (batch * s_q) and
# heads (1 x 16, 16 x 128, 64 x 128, 256 x 128, 4 x 16); a ragged second tile
# (200 = 128 + 72); an odd head count; one head.
CASES = [(1, 128), (1, 16), (16, 128), (64, 128), (256, 128), (4, 16), (200, 16), (300, 3), (129, 1)]


def bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.bfloat16).double().numpy()


def check(gpu: np.ndarray, ref: np.ndarray):
    err = np.abs(gpu - ref)
    bound = RTOL * np.abs(ref) + ATOL
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (worst, gpu[worst], ref[worst])
    exact = np.mean(gpu == bf16_round(ref))
    assert exact >= MIN_EXACT, exact


@pytest.mark.parametrize("tokens,h_q", CASES)
def test_absorb_matches_oracle(tokens, h_q):
    binding.mla_take_device_errors()  # start from a clear sticky word
    x = inputs.make_projection_inputs(tokens, h_q, seed=tokens * 131 + h_q)
    g = x.to("cuda")
    out = binding.mla_absorb_q(g.q_nope, g.q_rope, g.w_uk)
    assert binding.mla_take_device_errors() == 0
    out = mla_oracle.as_f64(out.cpu())
    ref = np.stack([mla_oracle.absorb_query(x.q_nope[t], x.q_rope[t], x.w_uk) for t in range(tokens)])
    assert out.shape == ref.shape == (tokens, h_q, 576)
    check(out[..., :512], ref[..., :512])
    assert np.array_equal(out[..., 512:], ref[..., 512:])


@pytest.mark.parametrize("tokens,h_q", CASES)
def test_up_project_matches_oracle(tokens, h_q):
    binding.mla_take_device_errors()
    x = inputs.make_projection_inputs(tokens, h_q, seed=7 + tokens * 131 + h_q)
    g = x.to("cuda")
    out = binding.mla_up_project(g.o_latent, g.w_uv)
    assert binding.mla_take_device_errors() == 0
    out = mla_oracle.as_f64(out.cpu())
    ref = np.stack([mla_oracle.expand_output(x.o_latent[t], x.w_uv) for t in range(tokens)])
    assert out.shape == ref.shape == (tokens, h_q, 128)
    check(out, ref)


def test_outputs_past_the_tokens_are_untouched():
    # Rows past `tokens` in the last 128-token tile are read as zeros and never
    # stored: a guard row after the output keeps its fill.
    tokens, h_q = 130, 4
    x = inputs.make_projection_inputs(tokens, h_q, seed=3).to("cuda")
    buf = torch.full((tokens + 1, h_q, 576), 7.0, dtype=torch.bfloat16, device="cuda")
    binding.mla_absorb_q(x.q_nope, x.q_rope, x.w_uk, out=buf[:tokens])
    ubuf = torch.full((tokens + 1, h_q, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    binding.mla_up_project(x.o_latent, x.w_uv, out=ubuf[:tokens])
    torch.cuda.synchronize()
    assert bool((buf[tokens] == 7.0).all()) and bool((ubuf[tokens] == 7.0).all())
    assert not bool((buf[:tokens] == 7.0).all(dim=-1).any())


def test_zero_tokens_is_a_no_op():
    x = inputs.make_projection_inputs(1, 2, seed=1).to("cuda")
    out = binding.mla_absorb_q(x.q_nope[:0], x.q_rope[:0], x.w_uk)
    assert out.shape == (0, 2, 576)


def test_layer_absorb_decode_up_project_matches_unabsorbed_definition():
    binding.mla_take_device_errors()
    lens = [300, 64, 1000, 129]
    h_q = 16
    d = inputs.make_inputs(lens, h_q, 1, seed=11, pool_factor=1.5)
    x = inputs.make_projection_inputs(len(lens), h_q, seed=12)
    g, gx = d.to("cuda"), x.to("cuda")
    q = binding.mla_absorb_q(gx.q_nope, gx.q_rope, gx.w_uk).view(len(lens), 1, h_q, 576)
    meta = binding.mla_get_metadata(g.seqlens, h_q, 1)
    o_lat, _ = binding.mla_decode(q, g.kv_cache, g.block_table, g.seqlens, d.softmax_scale, False, meta)
    out = binding.mla_up_project(o_lat.view(len(lens), h_q, 512), gx.w_uv)
    assert binding.mla_check_device_error(meta) == 0
    assert binding.mla_take_device_errors() == 0
    out = mla_oracle.as_f64(out.cpu())
    table = mla_oracle.as_int(d.block_table)
    for i, L in enumerate(lens):
        rows = mla_oracle.depage(d.kv_cache, table[i], L)
        ref, _ = mla_oracle.decode_unabsorbed(rows[:, :512], rows[:, 512:], x.q_nope[i], x.q_rope[i], x.w_uk,
                                              x.w_uv, d.softmax_scale)
        err = np.abs(out[i] - ref)
        assert err.max() <= 1.6e-2 and err.mean() <= 2e-3, (i, err.max(), err.mean())
