"""The seeded workload generator: determinism, layout and poisoning."""

import math

import torch

from mla_decode_attention_13_b200 import inputs as I


def test_seeded_and_deterministic():
    a = I.workload_inputs(0)
    b = I.workload_inputs(0)
    assert torch.equal(a.q, b.q) and torch.equal(a.block_table, b.block_table)
    assert torch.equal(a.kv_cache.view(torch.int16), b.kv_cache.view(torch.int16))


def test_tiny_workload_shape():
    x = I.workload_inputs(0)
    assert x.q.shape == (1, 1, 16, 576) and x.q.dtype == torch.bfloat16
    assert x.kv_cache.shape == (4, 64, 1, 576)
    assert sorted(x.block_table[0].tolist()) == [0, 1, 2, 3]
    assert x.seqlens.tolist() == [256]
    assert not x.causal and abs(x.softmax_scale - 192 ** -0.5) < 1e-15


def test_table_pages_distinct_and_poison_elsewhere():
    lens = [1, 64, 65, 200, 0]
    x = I.make_inputs(lens, 16, seed=3, extra_table_cols=2)
    used = []
    for i, L in enumerate(lens):
        n = -(-L // 64)
        used += x.block_table[i, :n].tolist()
        for j in range(n, x.block_table.shape[1]):
            spare = int(x.block_table[i, j])
            assert torch.isnan(x.kv_cache[spare].float()).all()
        if n and L % 64:
            last = int(x.block_table[i, n - 1])
            assert (x.kv_cache[last, L % 64:] == torch.tensor(1e4, dtype=torch.bfloat16)).all()
            assert torch.isfinite(x.kv_cache[last, : L % 64].float()).all()
    assert len(used) == len(set(used))
    assert x.num_pages == max(math.ceil(1.25 * len(used)), len(used) + 1)


def test_length_recipes():
    g = torch.Generator().manual_seed(0)
    u = I.draw_lengths(("uniform", 1024, 4096), 500, g)
    assert min(u) >= 1024 and max(u) <= 4096
    n = I.draw_lengths(("normal", 8192.0, 2048.0, 256, 16384), 500, g)
    assert min(n) >= 256 and max(n) <= 16384 and 7500 < sum(n) / len(n) < 8900


def test_fp8_inputs_layout():
    x = I.make_fp8_inputs([300, 64, 1, 0, 130], 8, 2, seed=5)
    pool = x.latent_codes.shape[0]
    assert x.latent_codes.dtype == torch.uint8 and x.latent_codes.shape[1:] == (64, 512)
    assert x.rope.shape == (pool, 64, 64) and x.exps.shape == (pool, 64)
    lens = [int(v) for v in x.seqlens]
    used = set()
    for i, L in enumerate(lens):
        n = (L + 63) // 64
        pages = [int(p) for p in x.block_table[i, :n]]
        used |= set(pages)
        for j in range(L):  # every visible token: finite codes, exponent in range
            p, sl = pages[j // 64], j % 64
            assert not bool(((x.latent_codes[p, sl] & 0x7F) == 0x7F).any())
            assert -8 <= int(x.exps[p, sl]) <= -5
        if n and L % 64:  # slots past L in the last page: largest code, exponent 5
            assert bool((x.latent_codes[pages[-1], L % 64:] == 0x7E).all())
            assert bool((x.exps[pages[-1], L % 64:] == 5).all())
    assert len(used) == sum((L + 63) // 64 for L in lens)
    for p in set(range(pool)) - used:  # pages no row holds: NaN codes
        assert bool((x.latent_codes[p] == 0x7F).all())
