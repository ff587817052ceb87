"""mla_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc (or ask torch for a new
tensor) inside their decode loop: a serving engine that sized all of its
device memory before it started, a framework that owns the allocator, or a
frozen memory plan around a captured graph.  They own every input and output
buffer already; what they cannot provide is the scratch workspace that
mla_decode takes for the partial results of rows split across SM pairs.
mla_decode_noalloc keeps that scratch in a fixed array inside the library.

These tests call it through the C ABI on two calls in a row (the second with
different inputs, so that scratch left over from the first call must not
matter), on shapes whose plans do split rows, and check its results two ways:

  * against the fp64 oracle, with the bar the other GPU tests use (max-abs
    8e-3, mean-abs 1e-3 on the bf16 output, |lse difference| <= 1e-3, -inf in
    the same places);
  * against mla_decode with a caller-allocated workspace, bit for bit: both
    run the same plan through the same deterministic kernels and differ only
    in where the partials live, so any difference at all (stale or partly
    overwritten scratch) is a fault.

One call runs on a non-default stream and is synchronised through that stream
alone.  The file is named so that pytest collects it last.
"""

import numpy as np
import pytest
import torch

from mla_decode_attention_13_b200 import binding, inputs
from oracle import mla_oracle

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN, TOL_LSE = 8e-3, 1e-3, 1e-3

# Few long rows: the plan cuts them across SM pairs, so the scratch is used.
CASES = [
    ([9000, 1024, 4100, 77], 16, 1, False),
    ([6000, 300, 2000], 128, 2, True),
]


def _against_oracle(x, out, lse):
    want_o, want_l = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal)
    got_o = out.cpu().double().numpy()
    got_l = lse.cpu().double().numpy()
    assert np.isfinite(got_o).all(), "non-finite output"
    d = np.abs(got_o - want_o)
    assert d.max() <= TOL_MAX, f"max-abs {d.max():.3e}"
    assert d.mean() <= TOL_MEAN, f"mean-abs {d.mean():.3e}"
    inf = np.isneginf(want_l)
    assert np.array_equal(inf, np.isneginf(got_l)), "lse -inf pattern differs"
    if (~inf).any():
        assert np.abs(got_l[~inf] - want_l[~inf]).max() <= TOL_LSE


def _bitwise_equal(ref, got):
    (ro, rl), (go, gl) = ref, got
    assert torch.equal(ro.view(torch.int16), go.view(torch.int16)), "out differs from mla_decode"
    assert torch.equal(rl.view(torch.int32), gl.view(torch.int32)), "lse differs from mla_decode"


@pytest.mark.parametrize("lens,h_q,s_q,causal", CASES)
def test_noalloc_matches_oracle_and_decode_on_two_calls(lens, h_q, s_q, causal):
    side = torch.cuda.Stream()
    for call in range(2):
        xc = inputs.make_inputs(lens, h_q, s_q, seed=70 + call, causal=causal)
        x = xc.to("cuda")
        meta = binding.mla_get_metadata(x.seqlens, x.h_q, x.s_q)
        torch.cuda.synchronize()
        assert int(meta[5].item()) > 0, "the plan should split at least one row"
        ref = binding.mla_decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, meta)
        torch.cuda.synchronize()
        out = torch.full((x.batch, x.s_q, x.h_q, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((x.batch, x.h_q, x.s_q), float("nan"), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        # the second call goes through an explicit non-default stream, synchronised on that stream only
        stream = side if call == 1 else None
        got = binding.mla_decode_noalloc(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, meta,
                                         out, lse, stream=stream)
        assert binding.mla_check_device_error(meta, stream=stream) == 0
        _against_oracle(xc, got[0], got[1])
        _bitwise_equal(ref, got)


def test_noalloc_rejects_bad_arguments_before_launch():
    lib = binding.lib()
    # NULL q: argument error from the host checks, nothing enqueued.
    st = lib.mla_decode_noalloc(None, None, 1, None, 1, None, 1, 1, 16, 0.1, 0, None, None, None, None)
    assert st == binding.MLA_ERR_ARG
    # Unsupported head count.
    st = lib.mla_decode_noalloc(None, None, 1, None, 1, None, 1, 1, 129, 0.1, 0, None, None, None, None)
    assert st == binding.MLA_ERR_UNSUPPORTED
