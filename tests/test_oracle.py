"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: each pin is a closed form, a
brute-force sum written with ``math`` on tiny inputs, a library routine
(torch's scaled_dot_product_attention in float64), a hand-derived worked
example (tests/golden), or an invariant the definition implies.  The mutation
tests at the bottom plant plausible mistakes in the oracle (on the CPU) and
check that at least one pin fails for each.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import mla_oracle as O
from mla_decode_attention_13_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SCALE = 192.0 ** -0.5


def _rand_inputs(lens, h_q=4, s_q=1, seed=0, causal=False, scale=SCALE, pool_factor=1.5):
    return I.make_inputs(lens, h_q, s_q, seed=seed, causal=causal, softmax_scale=scale,
                         pool_factor=pool_factor)


def _run(O, x, rows=None):
    return O.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, rows=rows)


def _own_depage(x, i):
    """Contiguous cache rows of batch row i, by reshaping whole pages (test-side route)."""
    L = int(x.seqlens[i])
    n = (L + 63) // 64
    pages = x.kv_cache[x.block_table[i, :n].long()]          # [n, 64, 1, 576]
    return pages.reshape(n * 64, 576)[:L].to(torch.float64)


# ---------------------------------------------------------------- pins ----

def pin_golden_three_tokens(O):
    g = json.load(open(os.path.join(GOLDEN, "closed_form_three_tokens.json")))
    q = np.zeros((1, 1, 1, 576))
    for k, v in g["q_nonzero"].items():
        q[0, 0, 0, int(k)] = v
    pool = np.zeros((1, 64, 1, 576))
    for j, row in enumerate(g["k_rows_nonzero"]):
        for k, v in row.items():
            pool[0, j, 0, int(k)] = v
    pool[0, 3:] = np.nan  # slots past L must not matter
    out, lse = O.decode(q, pool, np.zeros((1, 1), np.int64), np.array([g["L"]]), g["softmax_scale"], False)
    want = np.zeros(512)
    for k, v in g["expected_out_nonzero"].items():
        want[int(k)] = v
    np.testing.assert_allclose(out[0, 0, 0], want, rtol=0, atol=1e-14)
    assert abs(lse[0, 0, 0] - g["expected_lse"]) < 1e-14


def pin_single_token(O):
    x = _rand_inputs([1, 1, 1], h_q=3, seed=1)
    out, lse = _run(O, x)
    for i in range(3):
        k0 = x.kv_cache[int(x.block_table[i, 0]), 0, 0].to(torch.float64).numpy()
        for h in range(3):
            qv = x.q[i, 0, h].to(torch.float64).numpy()
            np.testing.assert_array_equal(out[i, 0, h], k0[:512])
            z0 = SCALE * math.fsum(float(a) * float(b) for a, b in zip(qv, k0))
            assert abs(lse[i, h, 0] - z0) < 1e-12


def pin_two_tokens(O):
    x = _rand_inputs([2], h_q=5, seed=2)
    out, lse = _run(O, x)
    rows = _own_depage(x, 0).numpy()
    for h in range(5):
        qv = x.q[0, 0, h].to(torch.float64).numpy()
        z = [SCALE * math.fsum(float(a) * float(b) for a, b in zip(qv, rows[j])) for j in range(2)]
        sig = lambda t: 1.0 / (1.0 + math.exp(-t))
        want = sig(z[0] - z[1]) * rows[0, :512] + sig(z[1] - z[0]) * rows[1, :512]
        np.testing.assert_allclose(out[0, 0, h], want, rtol=0, atol=1e-12)
        want_lse = max(z) + math.log1p(math.exp(-abs(z[0] - z[1])))
        assert abs(lse[0, h, 0] - want_lse) < 1e-12


def pin_brute_force_small(O):
    lens = [1, 2, 3, 4]
    x = _rand_inputs(lens, h_q=2, seed=3)
    out, lse = _run(O, x)
    for i, L in enumerate(lens):
        rows = _own_depage(x, i).numpy()
        for h in range(2):
            qv = [float(a) for a in x.q[i, 0, h].to(torch.float64)]
            z = [SCALE * math.fsum(qv[d] * float(rows[j, d]) for d in range(576)) for j in range(L)]
            m = max(z)
            e = [math.exp(zj - m) for zj in z]
            s = math.fsum(e)
            want = [math.fsum(e[j] * float(rows[j, d]) for j in range(L)) / s for d in range(512)]
            np.testing.assert_allclose(out[i, 0, h], want, rtol=0, atol=1e-12)
            assert abs(lse[i, h, 0] - (m + math.log(s))) < 1e-12


def pin_constant_cache(O):
    L, h = 200, 3
    q = np.random.default_rng(4).standard_normal((1, 1, h, 576))
    row = np.random.default_rng(5).standard_normal(576)
    pool = np.broadcast_to(row, (4, 64, 1, 576)).copy()
    table = np.array([[2, 0, 3, 1]])
    out, lse = O.decode(q, pool, table, np.array([L]), SCALE, False)
    for k in range(h):
        np.testing.assert_allclose(out[0, 0, k], row[:512], rtol=0, atol=1e-12)
        z = SCALE * math.fsum(a * b for a, b in zip(q[0, 0, k], row))
        assert abs(lse[0, k, 0] - (math.log(L) + z)) < 1e-11


def pin_weights_sum_to_one(O):
    rng = np.random.default_rng(6)
    for n in (1, 7, 300):
        z = rng.standard_normal(n) * 10
        w, _ = O.attention_weights(z)
        assert abs(math.fsum(w) - 1.0) < 1e-12
    # Through the whole call: a cache whose latent dims are all ones returns ones.
    x = _rand_inputs([130, 64], h_q=2, seed=7)
    x.kv_cache[..., :512] = 1.0
    out, _ = _run(O, x)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)


def pin_absorbed_equals_unabsorbed(O):
    rng = np.random.default_rng(8)
    H, L, d_c, d_r, d_n, d_vh = 4, 70, 512, 64, 128, 128
    c = rng.standard_normal((L, d_c))
    kr = rng.standard_normal((L, d_r))
    q_nope = rng.standard_normal((H, d_n))
    q_rope = rng.standard_normal((H, d_r))
    w_uk = rng.standard_normal((H, d_c, d_n)) / math.sqrt(d_c)
    w_uv = rng.standard_normal((H, d_c, d_vh)) / math.sqrt(d_c)
    ref_out, ref_lse = O.decode_unabsorbed(c, kr, q_nope, q_rope, w_uk, w_uv, SCALE)
    q_t = O.absorb_query(q_nope, q_rope, w_uk)                   # [H, 576]
    pool = np.zeros((2, 64, 1, 576))
    flat = np.concatenate([c, kr], axis=1)
    pool.reshape(128, 576)[:L] = flat
    o_lat, lse = O.decode(q_t[None, None], pool, np.array([[0, 1]]), np.array([L]), SCALE, False)
    out = O.expand_output(o_lat[0, 0], w_uv)
    np.testing.assert_allclose(out, ref_out, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse[0, :, 0], ref_lse, rtol=1e-10, atol=0)


def pin_paged_equals_contiguous(O):
    rng = np.random.default_rng(9)
    L, h = 300, 3
    cache = rng.standard_normal((L, 576))
    q = rng.standard_normal((1, 1, h, 576))
    n = (L + 63) // 64
    ident = np.full((n, 64, 1, 576), np.nan)
    ident.reshape(n * 64, 576)[:L] = cache
    out_c, lse_c = O.decode(q, ident, np.arange(n)[None], np.array([L]), SCALE, False)
    perm = rng.permutation(n + 3)
    pool = np.full((n + 3, 64, 1, 576), np.nan)
    for p in range(n):
        pool[perm[p]] = ident[p]
    out_p, lse_p = O.decode(q, pool, perm[:n][None], np.array([L]), SCALE, False)
    np.testing.assert_array_equal(out_p, out_c)
    np.testing.assert_array_equal(lse_p, lse_c)


def pin_split_combine_equals_single(O):
    rng = np.random.default_rng(10)
    L, R = 500, 6
    keys = rng.standard_normal((L, 576))
    q = rng.standard_normal((R, 576))
    limits = [L, L, 1, 250, 499, 64]
    want_o, want_l = O.attend(q, keys, keys[:, :512], SCALE, limits)
    cuts = [0, 63, 64, 200, 201, 450, L]
    parts = [O.partial_attention(q, keys, keys[:, :512], SCALE, limits, a, b) for a, b in zip(cuts, cuts[1:])]
    o, l = O.combine_partials(parts)
    np.testing.assert_allclose(o, want_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, want_l, rtol=0, atol=1e-12)


def pin_head_permutation(O):
    x = _rand_inputs([100, 33], h_q=6, seed=11)
    out, lse = _run(O, x)
    perm = torch.tensor([3, 0, 5, 1, 4, 2])
    x.q = x.q[:, :, perm].contiguous()
    out2, lse2 = _run(O, x)
    np.testing.assert_array_equal(out2, out[:, :, perm.numpy()])
    np.testing.assert_array_equal(lse2, lse[:, perm.numpy()])


def pin_constant_shift(O):
    rng = np.random.default_rng(12)
    L, h = 150, 3
    cache = rng.standard_normal((3, 64, 1, 576))
    r = rng.standard_normal(64)
    cache[..., 512:] = r  # every token has the same rope half
    q = rng.standard_normal((1, 1, h, 576))
    table = np.array([[1, 2, 0]])
    out, lse = O.decode(q, cache, table, np.array([L]), SCALE, False)
    dq = rng.standard_normal((h, 64))
    q2 = q.copy()
    q2[0, 0, :, 512:] += dq
    out2, lse2 = O.decode(q2, cache, table, np.array([L]), SCALE, False)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-12)
    delta = SCALE * (dq @ r)  # every score of head k moves by the same amount
    np.testing.assert_allclose(lse2[0, :, 0] - lse[0, :, 0], delta, rtol=0, atol=1e-11)


def pin_causal_single_token_is_noncausal(O):
    x = _rand_inputs([77, 1, 128], h_q=2, seed=15)
    out_nc, lse_nc = _run(O, x)
    x.causal = True
    out_c, lse_c = _run(O, x)
    np.testing.assert_array_equal(out_c, out_nc)
    np.testing.assert_array_equal(lse_c, lse_nc)


def pin_causal_two_tokens(O):
    x = _rand_inputs([90, 2, 64], h_q=2, s_q=2, seed=16, causal=True)
    out, lse = _run(O, x)
    # token t = 1 sees everything: equals the non-causal result
    x2 = _rand_inputs([90, 2, 64], h_q=2, s_q=2, seed=16, causal=False)
    out_nc, lse_nc = _run(O, x2)
    np.testing.assert_array_equal(out[:, 1], out_nc[:, 1])
    # token t = 0 equals a non-causal decode over the first L - 1 tokens
    x2.seqlens = x2.seqlens - 1
    out_s, lse_s = _run(O, x2)
    np.testing.assert_array_equal(out[:, 0], out_s[:, 0])
    np.testing.assert_array_equal(lse[:, :, 0], lse_s[:, :, 0])


def pin_library_sdpa(O):
    x = _rand_inputs([1, 64, 65, 333], h_q=4, s_q=2, seed=17, causal=True)
    out, lse = _run(O, x)
    for i in range(4):
        kv = _own_depage(x, i)
        L = kv.shape[0]
        q = x.q[i].to(torch.float64).reshape(2 * 4, 576)
        mask = torch.zeros(8, L, dtype=torch.bool)
        for t in range(2):
            mask[t * 4:(t + 1) * 4, : max(0, L - 2 + t + 1)] = True
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[None], kv[None], kv[None, :, :512], attn_mask=mask[None], scale=SCALE)[0]
        z = SCALE * q @ kv.T
        ref_lse = torch.logsumexp(z.masked_fill(~mask, -math.inf), dim=1)
        got = torch.from_numpy(out[i]).reshape(8, 512)
        ok = mask.any(dim=1)
        torch.testing.assert_close(got[ok], ref[ok], rtol=0, atol=1e-12)
        got_lse = torch.from_numpy(lse[i]).transpose(0, 1).reshape(8)
        torch.testing.assert_close(got_lse[ok], ref_lse[ok], rtol=0, atol=1e-12)


def pin_empty_rows(O):
    x = _rand_inputs([0, 5, 1], h_q=2, s_q=2, seed=18, causal=True)
    out, lse = _run(O, x)
    assert np.all(out[0] == 0) and np.all(lse[0] == -np.inf)
    # L = 1 with s_q = 2 causal: token 0 sees nothing, token 1 sees token 0
    assert np.all(out[2, 0] == 0) and np.all(lse[2, :, 0] == -np.inf)
    v0 = _own_depage(x, 2)[0, :512].numpy()
    np.testing.assert_array_equal(out[2, 1, 0], v0)


def pin_monotone_scores(O):
    L, h = 200, 2
    x = _rand_inputs([L], h_q=h, seed=19, scale=1.0)
    x.q[..., 512:] = 0
    x.q[..., 512] = 1.0
    rows_before = _own_depage(x, 0)
    n = (L + 63) // 64
    for j in range(L):
        x.kv_cache[int(x.block_table[0, j // 64]), j % 64, 0, 512] = 0.25 * j
    out, lse = _run(O, x)
    rows = _own_depage(x, 0).numpy()
    del rows_before, n
    for k in range(h):
        qv = [float(a) for a in x.q[0, 0, k].to(torch.float64)]
        z = [math.fsum(qv[d] * float(rows[j, d]) for d in range(576)) for j in range(L)]
        m = max(z)
        e = [math.exp(zj - m) for zj in z]
        s = math.fsum(e)
        want = np.array([math.fsum(e[j] * rows[j, d] for j in range(L)) / s for d in range(512)])
        np.testing.assert_allclose(out[0, 0, k], want, rtol=0, atol=1e-12)
        assert abs(lse[0, k, 0] - (m + math.log(s))) < 1e-12


def pin_e4m3_codes(O):
    # Every E4M3 bit pattern against torch's float8_e4m3fn conversion (a
    # library routine), and closed forms of the format: 0x7E = 448 (largest),
    # 0x01 = 2^-9 (smallest subnormal), 0x08 = 2^-6 (smallest normal),
    # 0x38 = 1, 0xB8 = -1, 0x00 = 0, S.1111.111 = NaN.
    import torch

    codes = np.arange(256, dtype=np.uint8)
    mine = O.e4m3_value(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(lib))
    assert np.array_equal(mine[~np.isnan(mine)], lib[~np.isnan(lib)])
    want = {0x7E: 448.0, 0x01: 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0xB8: -1.0, 0x00: 0.0}
    for c, v in want.items():
        assert O.e4m3_value([c])[0] == v, hex(c)
    assert np.isnan(O.e4m3_value([0x7F, 0xFF])).all()


def pin_fp8_dequantized_values_are_bf16_exact(O):
    import torch

    rng = np.random.default_rng(31)
    codes = rng.integers(0, 256, size=(64, 512)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x7E
    exps = rng.integers(-20, 21, size=64)
    lat = O.dequantize_latent(codes, exps)
    back = torch.from_numpy(lat).to(torch.bfloat16).double().numpy()
    assert np.array_equal(back, lat)


def pin_fp8_decode_equals_bf16_decode(O):
    # The FP8 path against the pinned bf16 decode over a cache assembled
    # independently: torch's float8 conversion times 2^exp, rope appended.
    import torch

    from mla_decode_attention_13_b200 import inputs as I

    x = I.make_fp8_inputs([300, 64, 1, 0, 130], 8, 2, seed=21, causal=True)
    lat = x.latent_codes.view(torch.float8_e4m3fn).to(torch.float64) * torch.pow(2.0, x.exps.to(torch.float64))[..., None]
    pool = torch.cat([lat, x.rope.to(torch.float64)], dim=-1)[:, :, None, :].numpy()
    want_o, want_l = O.decode(x.q, pool, x.block_table, x.seqlens, x.softmax_scale, True)
    got_o, got_l = O.decode_fp8(x.q, x.latent_codes, x.rope, x.exps, x.block_table, x.seqlens, x.softmax_scale,
                                True)
    np.testing.assert_allclose(got_o, want_o, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(got_l), np.isneginf(want_l))
    fin = np.isfinite(want_l)
    np.testing.assert_allclose(got_l[fin], want_l[fin], rtol=0, atol=1e-12)


def pin_fp8_quantizer(O):
    # The writer's exponent puts each row's largest magnitude in (224, 448];
    # codes equal torch's float8_e4m3fn rounding (nearest, ties to even) of
    # x / 2^e; the round trip errs by at most half an E4M3 step, 2^-4 |x| in
    # the normal range and 2^-10 2^e below it; dequantised rows quantise back
    # to the same values; an all-zero row gets e = 0 and zero codes.
    import torch

    rng = np.random.default_rng(41)
    x = rng.standard_normal((300, 512)) * rng.uniform(1e-3, 1e3, size=(300, 1))
    x[7] = 0.0
    codes, e = O.quantize_latent(x)
    amax = np.abs(x).max(axis=1)
    r = amax[amax > 0] / np.power(2.0, e[amax > 0])
    assert np.all((r > 224.0) & (r <= 448.0))
    assert e[7] == 0 and not codes[7].any()
    y = x / np.power(2.0, e)[:, None]
    lib = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(lib, codes)
    deq = O.dequantize_latent(codes, e)
    step = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * np.power(2.0, e)[:, None])
    assert np.all(np.abs(deq - x) <= step)
    codes2, e2 = O.quantize_latent(deq)
    assert np.array_equal(O.dequantize_latent(codes2, e2), deq)


NUMERIC_PINS = [
    pin_golden_three_tokens, pin_single_token, pin_two_tokens, pin_brute_force_small,
    pin_constant_cache, pin_weights_sum_to_one, pin_absorbed_equals_unabsorbed,
    pin_paged_equals_contiguous, pin_split_combine_equals_single, pin_head_permutation,
    pin_constant_shift, pin_causal_single_token_is_noncausal, pin_causal_two_tokens,
    pin_library_sdpa, pin_empty_rows, pin_monotone_scores,
    pin_e4m3_codes, pin_fp8_dequantized_values_are_bf16_exact, pin_fp8_decode_equals_bf16_decode,
    pin_fp8_quantizer,
]


@pytest.mark.parametrize("pin", NUMERIC_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(O)


def test_golden_fixture_matches_its_closed_form():
    g = json.load(open(os.path.join(GOLDEN, "closed_form_three_tokens.json")))
    assert abs(g["expected_lse"] - (math.log(6) + 0.5)) < 1e-15
    assert abs(g["expected_out_nonzero"]["0"] - (2 * math.log(2) + 3 * math.log(3)) / 6) < 1e-15


# ------------------------------------------------------- plan pins ----

def _plan_cases():
    rng = np.random.default_rng(20)
    cases = [([256], 16, 1, 74), ([4096] * 8, 128, 2, 74), ([131072, 1024, 32768, 8192], 16, 1, 74),
             ([0, 0, 5], 128, 1, 74), ([0], 16, 1, 3), ([1], 16, 1, 1), ([64 * 7] * 3, 128, 1, 2)]
    for _ in range(20):
        b = int(rng.integers(1, 40))
        lens = [int(v) for v in rng.integers(0, 20000, size=b)]
        cases.append((lens, int(rng.choice([16, 32, 64, 128])), int(rng.integers(1, 4)), int(rng.integers(1, 80))))
    return cases


@pytest.mark.parametrize("case", _plan_cases())
@pytest.mark.parametrize("kappa", [0, 2, 5])
def test_plan_covers_every_page_once_and_balances(case, kappa):
    lens, h_q, s_q, P = case
    plan = O.split_plan(lens, h_q, s_q, P, kappa)
    n_mt = -(-s_q * h_q // 128)
    b = len(lens)
    covered = {}
    for (w, b0, b1, slot), p in zip(plan["segments"], plan["segment_pair"]):
        assert 0 <= p < P and 0 <= b0 < b1
        for blk in range(b0, b1):
            assert (w, blk) not in covered
            covered[(w, blk)] = p
    want = {(mt * b + i, blk) for mt in range(n_mt) for i in range(b) for blk in range(-(-lens[i] // 64))}
    assert set(covered) == want
    # pairs take contiguous ranges in (row, page) order
    order = sorted(covered)
    owners = [covered[k] for k in order]
    assert owners == sorted(owners)
    # per-pair load stays within cap
    load = [0] * P
    pages = [0] * P
    for (w, b0, b1, _), p in zip(plan["segments"], plan["segment_pair"]):
        load[p] += b1 - b0 + kappa
        pages[p] += b1 - b0
    assert max(load, default=0) <= plan["cap"] + 2 * kappa
    assert max(pages, default=0) <= plan["cap"]
    # proportional ranges: when every range is longer than kappa, no pair is idle
    T = sum(-(-max(L, 0) // 64) + kappa for L in lens if L > 0) * n_mt
    assert plan["cap"] == max(1, -(-T // P))
    if T >= (kappa + 1) * P:
        assert min(pages) >= 1
    # pair offsets index the segment list
    offs = plan["pair_offsets"]
    assert offs[0] == 0 and offs[-1] == len(plan["segments"])
    for p in range(P):
        assert all(plan["segment_pair"][k] == p for k in range(offs[p], offs[p + 1]))


@pytest.mark.parametrize("case", _plan_cases())
def test_plan_slots_are_consecutive_per_split_row(case):
    lens, h_q, s_q, P = case
    plan = O.split_plan(lens, h_q, s_q, P, 2)
    by_row = {}
    for (w, b0, b1, slot) in plan["segments"]:
        by_row.setdefault(w, []).append((b0, slot))
    next_slot = 0
    for w in sorted(by_row):
        segs = sorted(by_row[w])
        if len(segs) == 1:
            assert segs[0][1] == -1 and plan["pieces"][w] == 1
        else:
            assert [s for _, s in segs] == list(range(next_slot, next_slot + len(segs)))
            assert plan["slot_base"][w] == next_slot
            next_slot += len(segs)
    assert plan["num_slots"] == next_slot
    assert plan["split_rows"] == [w for w in sorted(by_row) if len(by_row[w]) > 1]
    assert set(plan["empty_rows"]).isdisjoint(by_row)


# --------------------------------------------------- planted mistakes ----

def _mut_drop_rope(mp):
    mp.setattr(O, "scaled_scores", lambda q, k, s: s * (q[:, :512] @ k[:, :512].T))


def _mut_rope_sign(mp):
    mp.setattr(O, "scaled_scores", lambda q, k, s: s * (q[:, :512] @ k[:, :512].T - q[:, 512:] @ k[:, 512:].T))


def _mut_value_window(mp):
    mp.setattr(O, "value_of", lambda rows: rows[:, 64:576])


def _mut_no_scale(mp):
    mp.setattr(O, "scaled_scores", lambda q, k, s: q @ k.T)


def _mut_causal_off_by_one(mp):
    mp.setattr(O, "visible_limit", lambda L, s, t, c: max(0, min((L - s + t) if c else L, L)))


def _mut_ignore_table(mp):
    def depage(pool, row, L):
        j = np.arange(L)
        return pool[j // 64, j % 64, 0, :]
    mp.setattr(O, "depage", depage)


def _mut_slot_major(mp):
    mp.setattr(O, "token_location", lambda j: (j % 64 % max(1, (j.max() // 64 + 1) if j.size else 1), j // 64))


def _mut_log2_lse(mp):
    orig = O.log_sum_exp

    def lse2(z):
        v = orig(z)
        return v / math.log(2) if math.isfinite(v) else v
    mp.setattr(O, "log_sum_exp", lse2)


def _mut_unnormalised(mp):
    def w(z):
        m = np.max(z) if z.size else -np.inf
        if not np.isfinite(m):
            return np.zeros_like(z), -math.inf
        e = np.exp(z - m)
        return e, float(m + np.log(np.sum(e)))
    mp.setattr(O, "attention_weights", w)


def _mut_combine_mean(mp):
    orig = O.combine_partials

    def comb(parts):
        o, l = orig(parts)
        return np.mean(np.stack([p[0] for p in parts]), axis=0), l
    mp.setattr(O, "combine_partials", comb)


def _mut_absorb_one_head(mp):
    # every head absorbed with head 0's W_UK
    orig = O.absorb_query
    mp.setattr(O, "absorb_query", lambda qn, qr, w: orig(qn, qr, np.broadcast_to(O.as_f64(w)[:1], np.shape(w))))


def _mut_absorb_drops_rope(mp):
    orig = O.absorb_query

    def absorb(qn, qr, w):
        q = orig(qn, qr, w)
        q[:, 512:] = 0.0
        return q
    mp.setattr(O, "absorb_query", absorb)


def _mut_expand_heads_reversed(mp):
    orig = O.expand_output
    mp.setattr(O, "expand_output", lambda o, w: orig(o, O.as_f64(w)[::-1]))


def _mut_e4m3_bias_8(mp):
    orig = O.e4m3_value
    mp.setattr(O, "e4m3_value", lambda c: orig(c) / 2.0)


def _mut_e4m3_subnormal_scale(mp):
    orig = O.e4m3_value

    def v(c):
        out = orig(c)
        sub = ((np.asarray(c, dtype=np.int64) >> 3) & 0xF) == 0
        return np.where(sub, out / 2.0, out)
    mp.setattr(O, "e4m3_value", v)


def _mut_fp8_scale_inverted(mp):
    mp.setattr(O, "dequantize_latent",
               lambda codes, exps: O.e4m3_value(O.as_int(codes)) * np.power(2.0, -O.as_int(exps).astype(float))[..., None])


def _mut_fp8_rope_scaled(mp):
    orig = O.decode

    def decode_fp8(q, codes, rope, exps, table, lens, scale, causal, rows=None):
        lat = O.dequantize_latent(codes, exps)
        r = O.as_f64(rope) * np.power(2.0, O.as_int(exps).astype(float))[..., None]
        pool = np.concatenate([lat, r], axis=-1)[:, :, None, :]
        return orig(q, pool, table, lens, scale, causal, rows=rows)
    mp.setattr(O, "decode_fp8", decode_fp8)


def _mut_quantize_exponent_high(mp):
    orig = O.quantize_latent

    def q(rows):
        codes, e = orig(rows)
        return orig(O.as_f64(rows) / 2.0)[0], e + 1
    mp.setattr(O, "quantize_latent", q)


MUTATIONS = [_mut_drop_rope, _mut_rope_sign, _mut_value_window, _mut_no_scale, _mut_causal_off_by_one,
             _mut_ignore_table, _mut_slot_major, _mut_log2_lse, _mut_unnormalised, _mut_combine_mean,
             _mut_absorb_one_head, _mut_absorb_drops_rope, _mut_expand_heads_reversed,
             _mut_e4m3_bias_8, _mut_e4m3_subnormal_scale, _mut_fp8_scale_inverted, _mut_fp8_rope_scaled,
             _mut_quantize_exponent_high]


@pytest.mark.parametrize("mutation", MUTATIONS, ids=lambda f: f.__name__)
def test_planted_mistake_is_caught(mutation, monkeypatch):
    mutation(monkeypatch)
    failed = []
    for pin in NUMERIC_PINS:
        try:
            pin(O)
        except Exception:  # an assertion, or a shape error the mistake causes
            failed.append(pin.__name__)
    assert failed, f"no pin caught {mutation.__name__}"
