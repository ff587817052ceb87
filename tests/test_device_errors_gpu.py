"""Errors only the GPU can see: bits in the device error word, no fault.

The host checks arguments before it enqueues anything; what it cannot check
without reading device memory (block-table entries, lengths) the kernels check
as they go.  A page id outside the pool is flagged (MLA_DEVERR_PAGE) and the
copy reads page 0 instead, so it stays inside the pool; a length past the
row's block table or below zero is flagged (MLA_DEVERR_SEQLEN) and the row's
work is skipped (a negative length counts as an empty row).  Besides the word
in the metadata, which the next plan on that buffer rewrites, every bit also
lands in a per-device sticky word that only mla_take_device_errors clears.

Rows without a bad entry still match the oracle under the usual bar (the
checked rows are a few hundred tokens long, where 8e-3 max-abs holds).
"""

import numpy as np
import pytest
import torch

from mla_decode_attention_13_b200 import binding, inputs
from oracle import mla_oracle

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN, TOL_LSE = 8e-3, 1e-3, 1e-3


def _decode(x, seqlens_dev=None):
    g = x.to("cuda")
    lens = g.seqlens if seqlens_dev is None else seqlens_dev
    meta = binding.mla_get_metadata(lens, g.h_q, g.s_q)
    out, lse = binding.mla_decode(g.q, g.kv_cache, g.block_table, lens, g.softmax_scale, g.causal, meta)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu(), meta, g


def _rows_match(x, out, lse, rows):
    want_o, want_l = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal,
                                       rows=rows)
    want_o, want_l = want_o[rows], want_l[rows]
    got_o = out[rows].double().numpy()
    d = np.abs(got_o - want_o)
    assert np.isfinite(got_o).all()
    assert d.max() <= TOL_MAX and d.mean() <= TOL_MEAN
    gl = lse[rows].double().numpy()
    inf = np.isneginf(want_l)
    assert np.array_equal(inf, np.isneginf(gl))
    if (~inf).any():
        assert np.abs(gl[~inf] - want_l[~inf]).max() <= TOL_LSE


def test_page_outside_pool_is_flagged_and_sticky():
    binding.mla_take_device_errors()  # start from a clear sticky word
    x = inputs.make_inputs([700, 1500, 300], 64, seed=1200)
    bad = x.block_table.clone()
    bad[1, 3] = x.kv_cache.shape[0] + 7  # outside [0, num_pages)
    xb = inputs.DecodeInputs(**{**x.__dict__, "block_table": bad})
    out, lse, meta, g = _decode(xb)
    assert binding.mla_check_device_error(meta) & binding.MLA_DEVERR_PAGE
    _rows_match(x, out, lse, [0, 2])
    # A new plan on the same metadata clears its word; the sticky bit stays
    # until taken, and is gone after.
    binding.mla_get_metadata(g.seqlens, g.h_q, g.s_q, metadata=meta)
    assert binding.mla_check_device_error(meta) == 0
    assert binding.mla_take_device_errors() & binding.MLA_DEVERR_PAGE
    assert binding.mla_take_device_errors() == 0


def test_length_past_block_table_is_flagged():
    binding.mla_take_device_errors()
    x = inputs.make_inputs([640, 200, 260], 16, seed=1300)
    max_pages = x.block_table.shape[1]
    lens = x.seqlens.clone()
    lens[0] = 64 * max_pages + 10  # needs one page more than the table holds
    out, lse, meta, _ = _decode(x, lens.to("cuda"))
    assert binding.mla_check_device_error(meta) & binding.MLA_DEVERR_SEQLEN
    _rows_match(x, out, lse, [1, 2])
    assert binding.mla_take_device_errors() & binding.MLA_DEVERR_SEQLEN


def test_negative_length_is_flagged_as_an_empty_row():
    binding.mla_take_device_errors()
    x = inputs.make_inputs([300, 128, 333], 32, seed=1400)
    lens = x.seqlens.clone()
    lens[1] = -5
    out, lse, meta, _ = _decode(x, lens.to("cuda"))
    assert binding.mla_check_device_error(meta) & binding.MLA_DEVERR_SEQLEN
    assert (out[1] == 0).all() and torch.isneginf(lse[1]).all()
    _rows_match(x, out, lse, [0, 2])
    assert binding.mla_take_device_errors() & binding.MLA_DEVERR_SEQLEN


def test_clean_calls_leave_the_sticky_word_clear():
    binding.mla_take_device_errors()
    x = inputs.make_inputs([5000, 64, 1], 128, 2, seed=1500, causal=True)
    for _ in range(3):
        _decode(x)
    assert binding.mla_take_device_errors() == 0


def test_lengths_changed_since_the_plan_are_flagged():
    binding.mla_take_device_errors()
    x = inputs.make_inputs([900, 300, 1200], 64, seed=1600)
    g = x.to("cuda")
    meta = binding.mla_get_metadata(g.seqlens, g.h_q, g.s_q)
    changed = g.seqlens.clone()
    changed[2] -= 100  # same pages table, shorter row: the plan no longer matches
    binding.mla_decode(g.q, g.kv_cache, g.block_table, changed, g.softmax_scale, g.causal, meta)
    torch.cuda.synchronize()
    assert binding.mla_check_device_error(meta) & binding.MLA_DEVERR_PLAN
    assert binding.mla_take_device_errors() & binding.MLA_DEVERR_PLAN


def test_a_bounded_wait_that_runs_out_reports_a_timeout_and_the_context_stays_usable():
    # A barrier nothing arrives at: the wait gives up after its limit (1 s),
    # raises the timeout bit and the kernel returns; later calls still work.
    import time

    binding.mla_take_device_errors()
    t0 = time.perf_counter()
    binding.mla_selftest_bounded_wait()
    assert binding.mla_take_device_errors() == binding.MLA_DEVERR_TIMEOUT
    assert 0.9 < time.perf_counter() - t0 < 30
    x = inputs.workload_inputs(0)
    g = x.to("cuda")
    meta = binding.mla_get_metadata(g.seqlens, g.h_q, g.s_q)
    out, lse = binding.mla_decode(g.q, g.kv_cache, g.block_table, g.seqlens, g.softmax_scale, g.causal, meta)
    assert binding.mla_check_device_error(meta) == 0
    assert binding.mla_take_device_errors() == 0
    want_out, _ = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal)
    assert np.abs(out.cpu().double().numpy() - want_out).max() <= 8e-3
