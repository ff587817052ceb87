"""The per-element error bound of the bf16 decode kernels for rows where a few
tokens carry most of the softmax weight (shared by the GPU parity tests).

The kernel feeds bf16 weights p~ = p (1 + e), |e| <= 2^-8, to the PV product,
normalises by the unrounded fp32 sum of the weights and rounds the output to
bf16, so
    |out_gpu - out| <= 1.01 * 2^-8 (|out| + sum_j w_j |v_j|) + 1e-4
(1e-4 covers fp32 accumulation and the ex2 approximation).  Pieces of a row
split across SM pairs, or across GPUs with fp32 partials, are merged with
exact weights and add no rounding of their own.  For rows of one to a few
tokens with N(0, 1) values this bound reaches 1-2e-2, above 8e-3; over
hundreds to thousands of tokens it stays below 8e-3.
"""

import numpy as np


def bf16_weight_bound(x, want_o, rows):
    """Per-element bound 1.01 * 2^-8 (|out| + sum_j w_j |v_j|) + 1e-4 (module docstring)."""
    B = np.zeros_like(want_o)
    for n, i in enumerate(rows):
        L = int(x.seqlens[i])
        pages = (L + 63) // 64
        kv = x.kv_cache[x.block_table[i, :pages].long()].reshape(pages * 64, 576)[:L].double().numpy()
        for t in range(x.s_q):
            lim = min(max((L - x.s_q + t + 1) if x.causal else L, 0), L)
            q = x.q[i, t].double().numpy()
            for h in range(x.h_q):
                o = want_o[n, t, h]
                if lim == 0:
                    continue
                z = x.softmax_scale * (kv[:lim] @ q[h])
                w = np.exp(z - z.max())
                w /= w.sum()
                mag = w @ np.abs(kv[:lim, :512])
                B[n, t, h] = 1.01 * 2.0 ** -8 * (np.abs(o) + mag) + 1e-4
    return B


def fp8_weight_bound(x, want_o, rows):
    """The same bound for the FP8-cache kernel (mla_decode_fp8), whose weights
    go to the PV product as f16 (|e| <= 2^-11) and whose output is rounded to
    bf16 once (bf16's unit roundoff: 2^-8 |out|):
        |out_gpu - out| <= 1.01 * (2^-8 |out| + 2^-11 sum_j w_j |v_j|) + 1e-4.
    x is an Fp8DecodeInputs; the values are the dequantised latent dims."""
    from oracle import mla_oracle

    B = np.zeros_like(want_o)
    table = x.block_table.numpy()
    for n, i in enumerate(rows):
        L = int(x.seqlens[i])
        if L <= 0:
            continue
        pages = (L + 63) // 64
        ids = [int(v) for v in table[i, :pages]]
        lat = mla_oracle.dequantize_latent(x.latent_codes[ids], x.exps[ids]).reshape(pages * 64, 512)[:L]
        rope = x.rope[ids].double().numpy().reshape(pages * 64, 64)[:L]
        keys = np.concatenate([lat, rope], axis=1)
        for t in range(x.s_q):
            lim = min(max((L - x.s_q + t + 1) if x.causal else L, 0), L)
            if lim == 0:
                continue
            q = x.q[i, t].double().numpy()
            for h in range(x.h_q):
                z = x.softmax_scale * (keys[:lim] @ q[h])
                w = np.exp(z - z.max())
                w /= w.sum()
                mag = w @ np.abs(lat[:lim])
                B[n, t, h] = 1.01 * (2.0 ** -8 * np.abs(want_o[n, t, h]) + 2.0 ** -11 * mag) + 1e-4
    return B
