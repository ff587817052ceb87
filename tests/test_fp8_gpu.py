"""Parity of the FP8-latent-cache decode (mla_decode_fp8, through the C ABI)
with the fp64 oracle's decode_fp8 on the same seeded inputs.

The cache format ("MLA 和 MHA 的 Kernel 区别", section "量化友好性"): E4M3 codes
for the 512 latent dims of each token with one power-of-two scale 2^e per
token, bf16 rope.  decode_fp8 dequantises exactly and runs the fp64 decode.

Tolerances.  The kernel's arithmetic differs from the bf16 cache's only in
formats that lose nothing or less: the dequantised values are exact in f16
(e in [-15, 7]), q's latent part is exact in f16 for these N(0, 1) draws
except below 2^-14 (absolute error <= 2^-25), and the softmax weights go to
the PV product as f16 (relative error <= 2^-11 instead of bf16's 2^-8).  The
five workload shapes are held to the parity bars: max-abs 8e-3 and
mean-abs 1e-3 on the bf16 output, |lse difference| <= 1e-3, -inf where the
oracle has no visible token.  The other cases keep the mean-abs and lse bars;
per element they take the larger of 8e-3 and parity_bounds.fp8_weight_bound,
1.01 (2^-8 |out| + 2^-11 sum_j w_j |v_j|) + 1e-4, which passes 8e-3 only on
rows where a few tokens carry the weight and |out| reaches a few units (the
bf16 rounding of the exact output alone can reach 2^-8 |out|).
"""

import numpy as np
import pytest
import torch

from mla_decode_attention_13_b200 import binding, inputs
from oracle import mla_oracle
from parity_bounds import fp8_weight_bound

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN, TOL_LSE = 8e-3, 1e-3, 1e-3


def run_fp8(x, meta=None):
    g = x.to("cuda")
    if meta is None:
        meta = binding.mla_get_metadata(g.seqlens, g.h_q, g.s_q)
    out, lse = binding.mla_decode_fp8(g.q, g.latent_codes, g.rope, g.exps, g.block_table, g.seqlens,
                                      g.softmax_scale, g.causal, meta)
    err = binding.mla_check_device_error(meta)
    return out.cpu(), lse.cpu(), err


def assert_parity(x, out, lse, rows=None, strict=False):
    want_o, want_l = mla_oracle.decode_fp8(x.q, x.latent_codes, x.rope, x.exps, x.block_table, x.seqlens,
                                           x.softmax_scale, x.causal, rows=rows)
    sel = list(range(x.batch)) if rows is None else list(rows)
    got_o = out.double().numpy()[sel]
    got_l = lse.double().numpy()[sel]
    want_o, want_l = want_o[sel], want_l[sel]
    assert np.isfinite(got_o).all(), "non-finite output"
    d = np.abs(got_o - want_o)
    if strict:
        assert d.max() <= TOL_MAX, f"max-abs {d.max():.3e}"
    else:
        tol = np.maximum(TOL_MAX, fp8_weight_bound(x, want_o, sel))
        worst = np.unravel_index(np.argmax(d - tol), d.shape)
        assert (d <= tol).all(), f"max-abs {d.max():.3e}; worst excess at {worst}: {d[worst]:.3e} > {tol[worst]:.3e}"
    assert d.mean() <= TOL_MEAN, f"mean-abs {d.mean():.3e}"
    inf = np.isneginf(want_l)
    assert np.array_equal(np.isneginf(got_l), inf), "lse -inf pattern differs"
    if (~inf).any():
        dl = np.abs(got_l[~inf] - want_l[~inf])
        assert dl.max() <= TOL_LSE, f"lse max-abs {dl.max():.3e}"
    return d.max(), d.mean()


def test_tiny_shape():
    x = inputs.make_fp8_inputs([256], 16, seed=1, pool_factor=None)
    out, lse, err = run_fp8(x)
    assert err == 0
    assert_parity(x, out, lse)


@pytest.mark.parametrize("h_q", [16, 32, 64, 128])
def test_ragged_lengths(h_q):
    lens = [1, 2, 3, 63, 64, 65, 127, 128, 129, 500, 1000, 0]
    x = inputs.make_fp8_inputs(lens, h_q, seed=10 + h_q)
    out, lse, err = run_fp8(x)
    assert err == 0
    assert_parity(x, out, lse)
    assert (out[-1] == 0).all() and torch.isneginf(lse[-1]).all()


@pytest.mark.parametrize("s_q,h_q", [(2, 128), (4, 32), (16, 128), (3, 16)])
def test_causal_multi_token(s_q, h_q):
    x = inputs.make_fp8_inputs([1, 2, 3, 64, 65, 200, 777], h_q, s_q, seed=20 + s_q, causal=True)
    out, lse, err = run_fp8(x)
    assert err == 0
    assert_parity(x, out, lse)


def test_long_row_split_over_every_pair():
    x = inputs.make_fp8_inputs([40000, 900], 16, seed=30)
    out, lse, err = run_fp8(x)
    assert err == 0
    assert_parity(x, out, lse)


@pytest.mark.parametrize("exp_range,q_scale", [((-15, -13), 2.0 ** 13), ((5, 7), 2.0 ** -10)])
def test_exponents_at_the_ends_of_the_supported_range(exp_range, q_scale):
    # Token exponents at the low end (dequantised values down to 2^-24, f16's
    # smallest subnormal) and the high end (up to 448 * 2^7) of [-15, 7].  The
    # latent part of q is scaled so that the scores stay O(1); the outputs
    # then scale with 2^e, so the bar is relative to their size: 2^-7 of the
    # largest |out| (bf16 rounding of the output is at most 2^-8 of it).
    x = inputs.make_fp8_inputs([3000, 77, 640], 64, seed=40 + exp_range[0], exp_range=exp_range)
    x.q[..., :512] = (x.q[..., :512].float() * q_scale).to(torch.bfloat16)
    out, lse, err = run_fp8(x)
    assert err == 0
    want_o, want_l = mla_oracle.decode_fp8(x.q, x.latent_codes, x.rope, x.exps, x.block_table, x.seqlens,
                                           x.softmax_scale, x.causal)
    got_o = out.double().numpy()
    scale = np.abs(want_o).max()
    assert np.isfinite(got_o).all()
    assert np.abs(got_o - want_o).max() <= 2.0 ** -7 * scale, (np.abs(got_o - want_o).max(), scale)
    assert np.abs(lse.double().numpy() - want_l).max() <= TOL_LSE


def _sample_rows(lens, k, seed):
    order = sorted(range(len(lens)), key=lambda i: (lens[i], i))
    rows = {order[0], order[-1]}
    rng = np.random.default_rng(seed)
    for i in rng.permutation(len(lens)):
        if len(rows) >= k:
            break
        rows.add(int(i))
    return sorted(rows)


@pytest.mark.parametrize("index", [0, 1, 2, 3, 4])
def test_workload_shapes_full_size(index):
    # The five workloads' shapes (lengths, heads, query tokens, causality,
    # pool) with an FP8 cache: every row of the small ones, at least 8 seeded
    # rows with the shortest and longest of the 64- and 128-row ones.
    wl = inputs.WORKLOADS[index]
    gen = torch.Generator()
    gen.manual_seed(1000 + index)
    lens = inputs.draw_lengths(wl.lengths, wl.batch, gen)
    x = inputs.make_fp8_inputs(lens, wl.h_q, wl.s_q, seed=2000 + index, causal=wl.causal,
                               softmax_scale=wl.softmax_scale, pool_factor=wl.pool_factor)
    out, lse, err = run_fp8(x)
    assert err == 0
    rows = None if wl.batch <= 16 else _sample_rows(lens, 8, seed=index)
    assert_parity(x, out, lse, rows=rows, strict=True)


def test_one_plan_serves_fp8_and_bf16_calls():
    # one plan per step, whatever the cache format of the layer
    lens = [3000, 70, 1500]
    x8 = inputs.make_fp8_inputs(lens, 128, seed=50)
    x16 = inputs.make_inputs(lens, 128, seed=51)
    g16 = x16.to("cuda")
    meta = binding.mla_get_metadata(g16.seqlens, 128, 1)
    for _ in range(2):
        out, lse, err = run_fp8(x8, meta=meta)
        assert err == 0
        assert_parity(x8, out, lse)
        o16, l16 = binding.mla_decode(g16.q, g16.kv_cache, g16.block_table, g16.seqlens, x16.softmax_scale, False,
                                      meta)
        torch.cuda.synchronize()
        want_o, want_l = mla_oracle.decode(x16.q, x16.kv_cache, x16.block_table, x16.seqlens, x16.softmax_scale,
                                           False)
        assert np.abs(o16.cpu().double().numpy() - want_o).max() <= TOL_MAX


def test_matches_the_bf16_kernel_on_the_dequantised_cache():
    # The same attention through the bf16 path, on the cache dequantised and
    # assembled as bf16 rows (every value is exact in bf16): the two kernels
    # differ only in the weights' rounding (f16 vs bf16) and fp32 order.
    lens = [2000, 64, 333]
    x = inputs.make_fp8_inputs(lens, 32, 2, seed=60, causal=True)
    lat = mla_oracle.dequantize_latent(x.latent_codes, x.exps)
    pool = np.concatenate([lat, mla_oracle.as_f64(x.rope)], axis=-1)[:, :, None, :]
    kv = torch.from_numpy(pool).to(torch.bfloat16)
    exact = torch.from_numpy(pool)
    same = (kv.double() == exact) | (kv.double().isnan() & exact.isnan())
    assert bool(same.all()), "dequantised rows must be exact in bf16"
    g = x.to("cuda")
    meta = binding.mla_get_metadata(g.seqlens, 32, 2)
    o16, l16 = binding.mla_decode(g.q, kv.cuda(), g.block_table, g.seqlens, x.softmax_scale, True, meta)
    o8, l8, err = run_fp8(x, meta=meta)
    assert err == 0
    d = (o16.cpu().float() - o8.float()).abs()
    assert d.max().item() <= TOL_MAX and d.mean().item() <= TOL_MEAN
    fin = torch.isfinite(l16.cpu())
    assert torch.equal(fin, torch.isfinite(l8))
    assert (l16.cpu()[fin] - l8[fin]).abs().max().item() <= TOL_LSE


def test_out_of_range_exponent_and_query_are_flagged():
    binding.mla_take_device_errors()  # start from a clear sticky word
    lens = [300, 200]
    # a visible token with exponent 9 (E4M3 values times 2^9 overflow f16)
    x = inputs.make_fp8_inputs(lens, 16, seed=70)
    x.exps[int(x.block_table[0, 2]), 5] = 9
    _, _, err = run_fp8(x)
    assert err & binding.MLA_DEVERR_FP8_RANGE
    # one below the range
    x = inputs.make_fp8_inputs(lens, 16, seed=71)
    x.exps[int(x.block_table[1, 0]), 0] = -16
    _, _, err = run_fp8(x)
    assert err & binding.MLA_DEVERR_FP8_RANGE
    # a query value past the f16 range
    x = inputs.make_fp8_inputs(lens, 16, seed=72)
    x.q[1, 0, 3, 17] = 1.0e5
    _, _, err = run_fp8(x)
    assert err & binding.MLA_DEVERR_FP8_RANGE
    # exponents out of range past a row's length are never read: no flag
    x = inputs.make_fp8_inputs([300], 16, seed=73)
    x.exps[int(x.block_table[0, 4]), 300 % 64 + 3] = 12
    out, lse, err = run_fp8(x)
    assert err == 0
    assert_parity(x, out, lse)
    # and the context stays usable
    x = inputs.make_fp8_inputs(lens, 16, seed=74)
    out, lse, err = run_fp8(x)
    assert err == 0
    assert_parity(x, out, lse)
    assert binding.mla_take_device_errors() & binding.MLA_DEVERR_FP8_RANGE
    assert binding.mla_take_device_errors() == 0


def test_graph_replays_on_one_plan():
    # A CUDA graph of the FP8 call, replayed with a new query each time on
    # one plan, gives what the oracle gives for that query.
    lens = [2000, 333, 5000]
    x = inputs.make_fp8_inputs(lens, 64, seed=80)
    x_alt = inputs.make_fp8_inputs(lens, 64, seed=80)
    x_alt.q = inputs.make_fp8_inputs(lens, 64, seed=81).q
    g = x.to("cuda")
    meta = binding.mla_get_metadata(g.seqlens, 64, 1)
    ws = torch.empty(binding.mla_workspace_bytes(3, 64, 1), dtype=torch.uint8, device="cuda")
    out = torch.empty(3, 1, 64, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(3, 64, 1, dtype=torch.float32, device="cuda")
    q_buf = g.q.clone()
    st = torch.cuda.Stream()

    def call():
        binding.mla_decode_fp8(q_buf, g.latent_codes, g.rope, g.exps, g.block_table, g.seqlens, g.softmax_scale,
                               False, meta, workspace=ws, out=out, lse=lse, stream=st)

    with torch.cuda.stream(st):
        call()
    st.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=st):
        call()
    for k in range(4):
        src = x_alt if k % 2 else x
        with torch.cuda.stream(st):
            q_buf.copy_(src.q.to("cuda"))
            graph.replay()
        st.synchronize()
        assert binding.mla_check_device_error(meta) == 0
        assert_parity(src, out.cpu(), lse.cpu())
    del graph


def test_page_outside_pool_is_flagged_and_other_rows_hold():
    binding.mla_take_device_errors()  # start from a clear sticky word
    x = inputs.make_fp8_inputs([700, 1500, 300], 64, seed=82)
    x.block_table[1, 3] = x.latent_codes.shape[0] + 7  # outside [0, num_pages)
    out, lse, err = run_fp8(x)
    assert err & binding.MLA_DEVERR_PAGE
    assert torch.isfinite(out.float()).all()
    x_ok = inputs.make_fp8_inputs([700, 1500, 300], 64, seed=82)
    assert_parity(x_ok, out, lse, rows=[0, 2])
    assert binding.mla_take_device_errors() & binding.MLA_DEVERR_PAGE
