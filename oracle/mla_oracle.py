"""fp64 CPU oracle for MLA decode over a paged, compressed latent KV cache.

TEST INFRASTRUCTURE.  Only the tests, the package's ``__graft_entry__.smoke()``
check and ``bench.py``'s CPU-baseline leg may import this module.  It shares no
code with the CUDA path: nothing here is used by the library, and nothing from
the library is used here.

What it computes, and where each step comes from
------------------------------------------------
"MLA 和 MHA 的 Kernel 区别" (sealessland.top), section "内存布局和 KV Cache 大小 /
MLA": the cache holds only the compressed vector ``c_KV`` per token; keys and
values are its up-projections ``K = c_KV W_UK`` and ``V = c_KV W_UV``.  Section
"Decode 阶段的 HBM 访问模式 / MLA Decode": a decode step scores one query against
every cached token, takes a softmax, and sums the values weighted by it.

The absorbed form (weights folded into the query and the output) stores one
576-wide row per token: 512 latent dims followed by 64 rope dims.  The query
row is 576 wide too; the score is ``softmax_scale * <q, k_j>`` over all 576
dims, and the value is the first 512 dims of the same row.  ``decode`` is that
definition written out; ``decode_unabsorbed`` is the page's explicit
up-projection form (plus the rope half of the key), and the tests check that
the two agree.

"FlashMLA overview" (nullthought.net FlashMLA walkthrough): BF16 cache, paged
with 64-token blocks, variable-length rows.  ``token_location`` is the paging.

"Unlocking GPU Potential: The Impact of FlashAttention and KV Cache
Optimization in Long-Text Inference": decode has query length 1, so long rows
are split across processors and merged.  ``partial_attention`` and
``combine_partials`` are the split and the log-sum-exp merge; ``split_plan`` is
the integer tile-scheduler plan of the CUDA path's metadata kernel, restated
here from its definition so that the plan can be compared bit for bit.

"MLA 和 MHA 的 Kernel 区别", section "量化友好性": the latent ``c_KV`` may be
cached quantised (FP8 or INT8), the dequantisation fused with the load.  The
pages fix no format; ``e4m3_value``, ``dequantize_latent`` and ``decode_fp8``
take the plainest reading: the 512 latent dims of a cached token are OCP FP8
E4M3 codes with one power-of-two scale 2^e per token, and the 64 rope dims
(not part of ``c_KV``) stay bf16.  Every E4M3 value times a power of two is
exact in bf16, so the attention over the dequantised cache is again the
definition above.

Readings where the pages are silent (parity unpinned by the pages themselves;
the tests pin them only to these stated conventions):
  * causal decode with ``s_q > 1``: the ``s_q`` new tokens are the last
    ``s_q`` cache positions, so query token ``t`` sees cache tokens
    ``j <= L - s_q + t`` (bottom-right alignment);
  * a query with no visible token returns ``out = 0`` and ``lse = -inf``.
Everything else is pinned in ``tests/test_oracle.py`` against closed forms,
brute force, a library routine and invariants.

All arithmetic is float64.  Inputs may be bf16 tensors or arrays; they are
converted exactly to float64 first.
"""

from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

D_LATENT = 512
D_ROPE = 64
D_QK = D_LATENT + D_ROPE
D_V = D_LATENT
PAGE = 64
M_TILE = 128  # query rows per work row of the split plan


def as_f64(x) -> np.ndarray:
    """Exact conversion of a numpy array or torch tensor (any float type) to float64."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: the oracle itself does not need torch

        if x.dtype in (torch.bfloat16, torch.float16):
            x = x.to(torch.float32)
        return x.numpy().astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def as_int(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.asarray(x, dtype=np.int64)


# --------------------------------------------------------------------------
# Paging ("FlashMLA overview": paged kvcache, block size 64)
# --------------------------------------------------------------------------

def token_location(j: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Logical token index -> (logical page, slot within the page)."""
    return j // PAGE, j % PAGE


def depage(kv_pool, table_row: np.ndarray, length: int) -> np.ndarray:
    """Gather the first ``length`` cache rows of one sequence: [length, 576] float64.

    ``kv_pool`` may be a float array or a (bf16) torch tensor; only the rows
    gathered are converted.
    """
    j = np.arange(length, dtype=np.int64)
    page, slot = token_location(j)
    phys = table_row[page]
    if hasattr(kv_pool, "detach"):
        import torch  # local: the oracle itself does not need torch

        return as_f64(kv_pool[torch.from_numpy(phys), torch.from_numpy(slot), 0, :])
    return np.asarray(kv_pool[phys, slot, 0, :], dtype=np.float64)


def key_of(rows: np.ndarray) -> np.ndarray:
    """Absorbed key: the whole 576-wide row (latent then rope)."""
    return rows[:, :D_QK]


def value_of(rows: np.ndarray) -> np.ndarray:
    """Absorbed value: the first 512 (latent) dims of the same row."""
    return rows[:, :D_V]


# --------------------------------------------------------------------------
# Masking convention (pages silent; see module docstring)
# --------------------------------------------------------------------------

def visible_limit(length: int, s_q: int, t: int, causal: bool) -> int:
    """Number of leading cache tokens query token ``t`` may attend to."""
    n = (length - s_q + t + 1) if causal else length
    return max(0, min(n, length))


# --------------------------------------------------------------------------
# Attention of a set of query rows over a contiguous token list
# --------------------------------------------------------------------------

def scaled_scores(q_rows: np.ndarray, keys: np.ndarray, scale: float) -> np.ndarray:
    """z[r, j] = scale * <q_r, k_j>."""
    return scale * (q_rows @ keys.T)


def log_sum_exp(z: np.ndarray) -> float:
    """ln sum_j exp(z_j) of one masked score row (-inf entries are masked)."""
    m = np.max(z) if z.size else -np.inf
    if not np.isfinite(m):
        return -math.inf
    return float(m + np.log(np.sum(np.exp(z - m))))


def attention_weights(z: np.ndarray) -> Tuple[np.ndarray, float]:
    """Softmax of one masked score row and its log-sum-exp."""
    lse = log_sum_exp(z)
    if lse == -math.inf:
        return np.zeros_like(z), lse
    return np.exp(z - lse), lse


def attend(q_rows: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float,
           limits: Sequence[int]) -> Tuple[np.ndarray, np.ndarray]:
    """Row r attends to tokens [0, limits[r]).  Returns (out [R, dv], lse [R])."""
    z = scaled_scores(q_rows, keys, scale)
    out = np.zeros((q_rows.shape[0], values.shape[1]), dtype=np.float64)
    lse = np.full(q_rows.shape[0], -np.inf, dtype=np.float64)
    for r in range(q_rows.shape[0]):
        n = int(limits[r])
        w, lse[r] = attention_weights(z[r, :n])
        out[r] = w @ values[:n]
    return out, lse


# --------------------------------------------------------------------------
# The decode call: absorbed form over the paged cache
# --------------------------------------------------------------------------

def decode(q, kv_cache, block_table, seqlens, softmax_scale: float, causal: bool,
           rows: Sequence[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """MLA decode in absorbed form.

    q           [batch, s_q, h_q, 576]
    kv_cache    [num_pages, 64, 1, 576]
    block_table [batch, max_pages]
    seqlens     [batch]
    Returns ``out`` [batch, s_q, h_q, 512] and ``lse`` [batch, h_q, s_q] (natural
    log of sum_j exp(softmax_scale * <q, k_j>)), both float64.  ``rows`` limits
    the work to those batch rows (the others stay zero / -inf).
    """
    q = as_f64(q)
    pool = kv_cache if hasattr(kv_cache, "detach") else as_f64(kv_cache)
    table = as_int(block_table)
    lens = as_int(seqlens)
    batch, s_q, h_q, _ = q.shape
    out = np.zeros((batch, s_q, h_q, D_V), dtype=np.float64)
    lse = np.full((batch, h_q, s_q), -np.inf, dtype=np.float64)
    for i in (range(batch) if rows is None else rows):
        L = int(lens[i])
        cache = depage(pool, table[i], L)
        keys, values = key_of(cache), value_of(cache)
        for t in range(s_q):
            n = visible_limit(L, s_q, t, causal)
            o, l = attend(q[i, t], keys, values, softmax_scale, [n] * h_q)
            out[i, t] = o
            lse[i, :, t] = l
    return out, lse


# --------------------------------------------------------------------------
# The unabsorbed definition (explicit up-projection, per head)
# --------------------------------------------------------------------------

def decode_unabsorbed(c_kv, k_rope, q_nope, q_rope, w_uk, w_uv, scale: float,
                      limit: int = None) -> Tuple[np.ndarray, np.ndarray]:
    """Per head h: K^h_j = [c_j W_UK^h, k_rope_j], V^h_j = c_j W_UV^h, explicitly.

    c_kv [L, d_c], k_rope [L, d_r], q_nope [H, d_n], q_rope [H, d_r],
    w_uk [H, d_c, d_n], w_uv [H, d_c, d_vh].  Returns (out [H, d_vh], lse [H]).
    """
    c_kv, k_rope, q_nope, q_rope = map(as_f64, (c_kv, k_rope, q_nope, q_rope))
    w_uk, w_uv = as_f64(w_uk), as_f64(w_uv)
    L = c_kv.shape[0] if limit is None else limit
    H = q_nope.shape[0]
    out = np.zeros((H, w_uv.shape[2]))
    lse = np.zeros(H)
    for h in range(H):
        k_h = np.concatenate([c_kv @ w_uk[h], k_rope], axis=1)   # [L, d_n + d_r]
        v_h = c_kv @ w_uv[h]                                      # [L, d_vh]
        q_h = np.concatenate([q_nope[h], q_rope[h]])[None, :]
        o, l = attend(q_h, k_h, v_h, scale, [L])
        out[h], lse[h] = o[0], l[0]
    return out, lse


# --------------------------------------------------------------------------
# FP8 (E4M3) latent cache
# --------------------------------------------------------------------------

def e4m3_value(codes) -> np.ndarray:
    """float64 value of OCP FP8 E4M3 codes (uint8): 1 sign bit, 4 exponent
    bits with bias 7, 3 mantissa bits; exponent field 0 is subnormal
    (m / 8 * 2^-6); no infinities; S.1111.111 is NaN; the largest finite
    value is 448."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = (1.0 + m / 8.0) * np.power(2.0, e - 7)
    subnormal = (m / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, subnormal, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


def dequantize_latent(codes, exps) -> np.ndarray:
    """Latent rows from FP8 codes [..., 512] and per-token exponents [...]:
    e4m3_value(code) * 2^exp, in float64."""
    e = np.asarray(as_int(exps), dtype=np.float64)
    return e4m3_value(as_int(codes)) * np.power(2.0, e)[..., None]


def _e4m3_table() -> Tuple[np.ndarray, np.ndarray]:
    """The finite E4M3 values in increasing order, with their codes."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.int64)
    vals = e4m3_value(codes)
    order = np.lexsort((codes, vals))
    return vals[order], codes[order]


def quantize_latent(rows) -> Tuple[np.ndarray, np.ndarray]:
    """The cache writer's side of the FP8 format: per token (last axis = 512
    latent dims) the exponent e is the smallest integer with
    max|x| / 2^e <= 448 (e = 0 for an all-zero row), and each code is x / 2^e
    rounded to the nearest E4M3 value, ties to the even mantissa.  Returns
    (codes uint8 [..., 512], exps int64 [...])."""
    x = as_f64(rows)
    amax = np.max(np.abs(x), axis=-1)
    e = np.zeros(amax.shape, dtype=np.int64)
    nz = amax > 0
    e[nz] = np.ceil(np.log2(amax[nz] / 448.0)).astype(np.int64)
    # log2 rounding can leave e one too small or too large: settle it exactly
    e[nz] += (amax[nz] / np.power(2.0, e[nz]) > 448.0)
    e[nz] -= (amax[nz] / np.power(2.0, e[nz] - 1) <= 448.0)
    y = x / np.power(2.0, e.astype(np.float64))[..., None]
    vals, codes = _e4m3_table()
    # the codes with the sign bit clear (+0 .. 448), for rounding |y|
    pos = (codes & 0x80) == 0
    pv, pc = vals[pos], codes[pos]
    a = np.abs(y)
    hi = np.clip(np.searchsorted(pv, a, side="left"), 1, len(pv) - 1)
    lo = hi - 1
    d_lo, d_hi = a - pv[lo], pv[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((pc[hi] & 1) == 0))
    mag = np.where(take_hi, pc[hi], pc[lo])
    mag = np.where(a >= pv[-1], pc[-1], mag)
    code = np.where(np.signbit(y), mag | 0x80, mag)  # the sign is kept, on zero too
    return code.astype(np.uint8), e


def decode_fp8(q, latent_codes, rope, exps, block_table, seqlens, softmax_scale: float, causal: bool,
               rows: Sequence[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """``decode`` over an FP8 latent cache.

    latent_codes [num_pages, 64, 512] uint8 (E4M3), rope [num_pages, 64, 64]
    (bf16 or float), exps [num_pages, 64] integer (token scale 2^exp).  Each
    cached row is [dequantised latent, rope]; the rest is ``decode``.  Only
    the pages the computed rows read are dequantised (a pool of those pages,
    with the block table renumbered into it), so that a large pool costs no
    more than the rows asked for.
    """
    table = as_int(block_table)
    lens = as_int(seqlens)
    batch = table.shape[0]
    sel = range(batch) if rows is None else rows
    used = sorted({int(table[i, j]) for i in sel for j in range((max(int(lens[i]), 0) + PAGE - 1) // PAGE)})
    index = {page: k for k, page in enumerate(used)}
    local = np.zeros_like(table)
    for i in sel:
        for j in range((max(int(lens[i]), 0) + PAGE - 1) // PAGE):
            local[i, j] = index[int(table[i, j])]
    if not used:
        pool = np.zeros((0, PAGE, D_QK))
    else:
        # index first (a plain list works for arrays and tensors), then convert
        lat = dequantize_latent(as_int(latent_codes[used]), as_int(exps[used]))
        pool = np.concatenate([lat, as_f64(rope[used])], axis=-1)
    return decode(q, pool[:, :, None, :], local, seqlens, softmax_scale, causal, rows=rows)


def absorb_query(q_nope, q_rope, w_uk) -> np.ndarray:
    """q~^h = [W_UK^h q_nope^h, q_rope^h]: the query seen by the latent cache."""
    q_nope, q_rope, w_uk = as_f64(q_nope), as_f64(q_rope), as_f64(w_uk)
    lat = np.einsum("hcn,hn->hc", w_uk, q_nope)
    return np.concatenate([lat, q_rope], axis=1)


def expand_output(o_latent, w_uv) -> np.ndarray:
    """o^h = o~^h W_UV^h: the head's output from its latent-space output."""
    return np.einsum("hc,hcv->hv", as_f64(o_latent), as_f64(w_uv))


# --------------------------------------------------------------------------
# Split-KV (flash-decoding) and the log-sum-exp merge
# --------------------------------------------------------------------------

def partial_attention(q_rows, keys, values, scale: float, limits: Sequence[int],
                      j0: int, j1: int) -> Tuple[np.ndarray, np.ndarray]:
    """Attention of each row over tokens [j0, min(j1, limit)) only (normalised)."""
    R = q_rows.shape[0]
    out = np.zeros((R, values.shape[1]))
    lse = np.full(R, -np.inf)
    z = scaled_scores(q_rows, keys[j0:j1], scale)
    for r in range(R):
        n = max(0, min(int(limits[r]), j1) - j0)
        w, lse[r] = attention_weights(z[r, :n])
        out[r] = w @ values[j0:j0 + n]
    return out, lse


def combine_partials(parts: List[Tuple[np.ndarray, np.ndarray]]) -> Tuple[np.ndarray, np.ndarray]:
    """Merge normalised partial results (o_k, lse_k) of disjoint token ranges.

    lse = ln sum_k exp(lse_k);  out = sum_k exp(lse_k - lse) * o_k.
    """
    lses = np.stack([p[1] for p in parts])            # [K, R]
    outs = np.stack([p[0] for p in parts])            # [K, R, dv]
    m = np.max(lses, axis=0)
    lse = np.full(m.shape, -np.inf)
    out = np.zeros(outs.shape[1:])
    for r in range(m.shape[0]):
        if not np.isfinite(m[r]):
            continue
        w = np.exp(lses[:, r] - m[r])
        lse[r] = m[r] + np.log(np.sum(w))
        out[r] = np.sum(np.exp(lses[:, r] - lse[r])[:, None] * outs[:, r], axis=0)
    return out, lse


# --------------------------------------------------------------------------
# The split-KV plan (integer; compared bit for bit with the metadata kernel)
# --------------------------------------------------------------------------

def split_plan(seqlens, h_q, s_q, num_pairs: int, kappa: int) -> dict:
    """Cost-interval partition of all (work row, page) units over ``num_pairs``.

    A work row is one batch row's block of up to 128 query rows; work rows are
    ordered m-tile major (w = mt * batch + i).  A work row with n > 0 pages
    costs c = n + kappa (kappa: the fixed cost of starting a row, in page
    units), else 0.  With C_w the cost of the rows before w and T the total,
    page b of row w sits at cost position C_w + kappa + b.  Pair p owns the
    positions [B(p), B(p + 1)), with B(p) = floor(p * T / P) when T >= P (every
    pair gets floor(T / P) or ceil(T / P) positions) and B(p) = min(p, T)
    otherwise (one position each; the pairs past T get none).  Each pair thus
    takes one contiguous range of pages; a row whose pages land on k > 1 pairs
    is cut into k pieces and gets k consecutive partial slots, numbered in row
    order.  ``cap`` reports the longest range, max(1, ceil(T / P)).
    """
    lens = [int(x) for x in as_int(seqlens)]
    batch = len(lens)
    R = s_q * h_q
    n_mt = (R + M_TILE - 1) // M_TILE
    W = batch * n_mt
    n_blk = [0] * W
    for mt in range(n_mt):
        for i in range(batch):
            n_blk[mt * batch + i] = (max(lens[i], 0) + PAGE - 1) // PAGE
    cost = [(n + kappa) if n > 0 else 0 for n in n_blk]
    T = sum(cost)
    P = num_pairs
    cap = max(1, (T + P - 1) // P)
    bound = [(p * T) // P if T >= P else min(p, T) for p in range(P + 1)]
    segs = []  # (pair, w, b0, b1)
    C = 0
    for w in range(W):
        n = n_blk[w]
        if n > 0:
            lo, hi = C + kappa, C + kappa + n  # this row's page positions
            for p in range(P):
                b0 = max(lo, bound[p]) - lo
                b1 = min(hi, bound[p + 1]) - lo
                if b0 < b1:
                    segs.append([p, w, b0, b1])
        C += cost[w]
    pieces = [0] * W
    for sg in segs:
        pieces[sg[1]] += 1
    slot_base = [-1] * W
    nslots = 0
    for w in range(W):
        if pieces[w] > 1:
            slot_base[w] = nslots
            nslots += pieces[w]
    seen = [0] * W
    seg_slots = []
    for sg in segs:
        w = sg[1]
        if pieces[w] > 1:
            seg_slots.append(slot_base[w] + seen[w])
            seen[w] += 1
        else:
            seg_slots.append(-1)
    pair_off = [0] * (num_pairs + 1)
    for sg in segs:
        pair_off[sg[0] + 1] += 1
    for k in range(num_pairs):
        pair_off[k + 1] += pair_off[k]
    return {
        "num_pairs": num_pairs, "work_rows": W, "n_mt": n_mt, "cap": cap,
        "segments": [(sg[1], sg[2], sg[3], sl) for sg, sl in zip(segs, seg_slots)],
        "segment_pair": [sg[0] for sg in segs],
        "pair_offsets": pair_off,
        "pieces": pieces, "slot_base": slot_base, "num_slots": nslots,
        "split_rows": [w for w in range(W) if pieces[w] > 1],
        "empty_rows": [w for w in range(W) if pieces[w] == 0],
    }
