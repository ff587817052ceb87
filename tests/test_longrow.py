"""The long-row split across ranks on the CPU: the shard rule against the
global causal mask (brute force), the per-rank block tables, and the exchange
over gloo ranks, whose merged result must equal the unsplit decode.

Each rank's partial here comes from the oracle (the GPU kernels need a GPU);
the merge is the oracle's log-sum-exp combine.  So these tests cover the host
logic of the split (which pages a rank holds, which rank masks, what is
exchanged); tests/test_longrow_gpu.py runs the library's kernels on it.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from mla_decode_attention_13_b200 import inputs, longrow
from oracle import mla_oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def visible_tokens(L, s_q, t, causal):
    """Cache positions query token t of a step sees, straight from the rule:
    every position below L, and with causal only those j <= L - s_q + t."""
    return {j for j in range(L) if not causal or j <= L - s_q + t}


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("s_q", [1, 2, 5, 16])
def test_shards_cover_each_row_and_keep_every_query_tokens_view(world, s_q):
    rng = np.random.default_rng(world * 31 + s_q)
    lengths = [0, 1, 15, 16, 17, 63, 64, 65, 66, 127, 128, 129, 130, 1000] + list(rng.integers(1, 3000, 12))
    for L in lengths:
        b = longrow.shard_bounds(L, world, s_q)
        n = (L + 63) // 64
        assert b[0] == 0 and b[-1] == n and all(b[r] <= b[r + 1] for r in range(world))
        lens = [longrow.shard_lengths([L], world, s_q)[r][0] for r in range(world)]
        assert sum(lens) == L
        for causal in (False, True):
            for t in range(s_q):
                seen = set()
                for r in range(world):
                    start = 64 * b[r]
                    local_causal = causal and r == world - 1
                    # what rank r's decode sees: its first `lens[r]` tokens, masked by
                    # its own length when it is the masking rank
                    local = visible_tokens(lens[r], s_q, t, local_causal)
                    seen |= {start + j for j in local}
                assert seen == visible_tokens(L, s_q, t, causal), (L, world, s_q, causal, t)


def test_shard_block_table_slices_each_row():
    x = inputs.make_inputs([300, 64, 1, 0, 700], 4, 1, seed=3)
    lens = [int(v) for v in x.seqlens]
    for world in (1, 2, 3):
        for rank in range(world):
            table, local = longrow.shard_block_table(x.block_table, lens, world, rank)
            for i, L in enumerate(lens):
                b = longrow.shard_bounds(L, world)
                k = b[rank + 1] - b[rank]
                assert torch.equal(table[i, :k], x.block_table[i, b[rank]:b[rank + 1]])
                assert int(local[i]) == longrow.shard_lengths(lens, world)[rank][i]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, case, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist

    from mla_decode_attention_13_b200 import inputs, longrow
    from oracle import mla_oracle

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lens, h_q, s_q, causal = case
        x = inputs.make_inputs(lens, h_q, s_q, seed=17, causal=causal)
        table, local = longrow.shard_block_table(x.block_table, lens, world, rank, s_q)
        out_r, lse_r = mla_oracle.decode(x.q, x.kv_cache, table, local, x.softmax_scale, causal and rank == world - 1)
        outs, lses = longrow.gather_partials(torch.from_numpy(out_r), torch.from_numpy(lse_r))
        outs, lses = outs.numpy(), lses.numpy()
        # merge per query row: out [b, s_q, h, 512], lse [b, h, s_q]
        b = len(lens)
        parts = [(outs[k].reshape(b * s_q * h_q, 512), lses[k].transpose(0, 2, 1).reshape(-1)) for k in range(world)]
        out, lse = mla_oracle.combine_partials(parts)
        want_out, want_lse = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, causal)
        err = float(np.max(np.abs(out - want_out.reshape(out.shape))))
        want_l = want_lse.transpose(0, 2, 1).reshape(-1)
        same_inf = bool(np.array_equal(np.isinf(lse), np.isinf(want_l)))
        fin = np.isfinite(want_l)
        lerr = float(np.max(np.abs(lse[fin] - want_l[fin]))) if fin.any() else 0.0
        q.put((rank, err, lerr, same_inf))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world,case", [
    (2, ([300, 64, 1, 0, 700], 4, 1, False)),
    (2, ([300, 65, 3, 130, 700], 4, 3, True)),
    (3, ([1000, 129, 64, 2], 2, 2, True)),
])
def test_gloo_ranks_exchange_partials_that_merge_to_the_unsplit_decode(world, case):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(170)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, err, lerr, same_inf in res:
        assert err < 1e-12 and lerr < 1e-12 and same_inf, (rank, err, lerr, same_inf)


def _sharded_worker(rank, world, port, case, q):
    # longrow.decode_sharded itself across gloo ranks, with the library calls
    # replaced by oracle-backed stand-ins: this checks the orchestration (which
    # rank masks, the gather order, what reaches the merge).
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import types

    import torch.distributed as dist

    from mla_decode_attention_13_b200 import inputs, longrow
    from oracle import mla_oracle

    calls = []

    def get_metadata(seqlens, h_q, s_q, metadata=None, stream=None):
        return ("plan", tuple(int(v) for v in seqlens))

    def decode_f32(q, kv, table, seqlens, scale, causal, meta, **kw):
        # the split exchanges unrounded partials: fp32 out, as mla_decode_f32 writes
        assert meta == ("plan", tuple(int(v) for v in seqlens))
        calls.append(bool(causal))
        o, l = mla_oracle.decode(q, kv, table, seqlens, scale, causal)
        return torch.from_numpy(o).float(), torch.from_numpy(l).float()

    def merge_f32(outs, lses, **kw):
        assert outs.dtype == torch.float32 and lses.dtype == torch.float32
        w, b, s, h, _ = outs.shape
        parts = [(outs[k].numpy().reshape(b * s * h, 512), lses[k].numpy().transpose(0, 2, 1).reshape(-1))
                 for k in range(w)]
        o, l = mla_oracle.combine_partials(parts)
        return torch.from_numpy(o.reshape(b, s, h, 512)), torch.from_numpy(l.reshape(b, s, h).transpose(0, 2, 1))

    longrow.binding = types.SimpleNamespace(mla_get_metadata=get_metadata, mla_decode_f32=decode_f32,
                                            mla_merge_splits_f32=merge_f32)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lens, h_q, s_q, causal = case
        x = inputs.make_inputs(lens, h_q, s_q, seed=23, causal=causal)
        table, local = longrow.shard_block_table(x.block_table, lens, world, rank, s_q)
        out, lse = longrow.decode_sharded(x.q, x.kv_cache, table, local, x.softmax_scale, causal)
        want_out, want_lse = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, causal)
        err = float(np.max(np.abs(out.numpy() - want_out)))
        fin = np.isfinite(want_lse)
        lerr = float(np.max(np.abs(lse.numpy()[fin] - want_lse[fin]))) if fin.any() else 0.0
        same_inf = bool(np.array_equal(np.isneginf(lse.numpy()), np.isneginf(want_lse)))
        q.put((rank, err, lerr, same_inf, calls))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world,case", [
    (2, ([300, 65, 3, 130, 700], 4, 3, True)),
    (3, ([1000, 129, 64, 2, 0], 2, 1, False)),
])
def test_decode_sharded_over_gloo_ranks_equals_the_unsplit_decode(world, case):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(170)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    causal = case[3]
    for rank, err, lerr, same_inf, calls in res:
        # the stand-ins pass fp32 partials, as the library's do: fp32 rounding only
        assert err < 1e-5 and lerr < 1e-5 and same_inf, (rank, err, lerr)
        assert calls == [causal and rank == world - 1]  # one decode per rank; only the last one masks
