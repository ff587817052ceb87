"""Seeded synthetic workloads for MLA decode over a paged latent KV cache.

This module only draws random numbers and lays them out (per-row sequence
lengths, a shuffled physical block pool, the block table, Q, and the latent
cache).  It performs none of the attention arithmetic, so both the CUDA path's
tests and the CPU oracle's tests can take their inputs from here.

The five workloads mirror the decode shapes of the method: one shared
576-wide latent-plus-rope row per cached token (512 latent + 64 rope, bf16),
64-token pages looked up through a block table ("FlashMLA overview": BF16,
paged kvcache with block size 64, variable-length sequences).

Recipe (all draws from ``torch.Generator`` seeded with ``1000 + index``):
  1. per-row sequence lengths from the workload's length recipe;
  2. ``n_blk_i = ceil(L_i / 64)`` pages per row; the pool holds
     ``ceil(pool_factor * sum n_blk)`` pages (exactly ``sum n_blk`` for the tiny
     case), in a random permutation handed out to rows in order;
  3. block-table entries past a row's pages point at a poisoned spare page
     (NaN-filled) so that any stray read shows up as NaN in the result;
  4. Q and the cache are N(0, 1) rounded to bf16 (round-to-nearest-even);
  5. cache slots past ``L_i`` in a row's last page hold ``tail_fill``
     (1e4 by default: finite, but large enough to be noticed if read).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

D_LATENT = 512
D_ROPE = 64
D_QK = D_LATENT + D_ROPE
D_V = D_LATENT
PAGE = 64
DEFAULT_SCALE = 192.0 ** -0.5


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and length recipe of one synthetic decode workload."""

    name: str
    batch: int
    s_q: int
    h_q: int
    lengths: tuple  # ("fixed", [...]) | ("uniform", lo, hi) | ("normal", mu, sigma, lo, hi)
    pool_factor: Optional[float]  # None: pool holds exactly the pages needed
    causal: bool = False
    softmax_scale: float = DEFAULT_SCALE


# Index i of this tuple uses seed 1000 + i.
WORKLOADS = (
    Workload("tiny_b1_h16_L256", 1, 1, 16, ("fixed", [256]), None),
    Workload("b16_h128_L1k-4k", 16, 1, 128, ("uniform", 1024, 4096), 1.25),
    Workload("b64_h128_L8k+-2k", 64, 1, 128, ("normal", 8192.0, 2048.0, 256, 16384), 1.25),
    Workload("b128_s2_h128_L4k_causal", 128, 2, 128, ("fixed", [4096] * 128), 1.25, causal=True),
    Workload("b4_h16_L128k-1k", 4, 1, 16, ("fixed", [131072, 1024, 32768, 8192]), 1.1),
)

BY_NAME = {w.name: (i, w) for i, w in enumerate(WORKLOADS)}


@dataclasses.dataclass
class DecodeInputs:
    """One decode step's tensors, in the layouts the C ABI takes."""

    q: torch.Tensor            # [batch, s_q, h_q, 576] bf16
    kv_cache: torch.Tensor     # [num_pages, 64, 1, 576] bf16
    block_table: torch.Tensor  # [batch, max_pages_per_row] int32
    seqlens: torch.Tensor      # [batch] int32
    s_q: int
    h_q: int
    causal: bool
    softmax_scale: float
    name: str = ""

    @property
    def batch(self) -> int:
        return int(self.q.shape[0])

    @property
    def num_pages(self) -> int:
        return int(self.kv_cache.shape[0])

    def to(self, device) -> "DecodeInputs":
        return dataclasses.replace(
            self,
            q=self.q.to(device),
            kv_cache=self.kv_cache.to(device),
            block_table=self.block_table.to(device),
            seqlens=self.seqlens.to(device),
        )


def draw_lengths(recipe: tuple, batch: int, gen: torch.Generator) -> list:
    kind = recipe[0]
    if kind == "fixed":
        lens = list(recipe[1])
        if len(lens) != batch:
            raise ValueError("fixed length list must have one entry per row")
        return [int(x) for x in lens]
    if kind == "uniform":
        lo, hi = int(recipe[1]), int(recipe[2])
        return [int(x) for x in torch.randint(lo, hi + 1, (batch,), generator=gen)]
    if kind == "normal":
        mu, sigma, lo, hi = recipe[1:]
        x = torch.randn(batch, generator=gen, dtype=torch.float64) * sigma + mu
        return [int(min(max(round(float(v)), lo), hi)) for v in x]
    raise ValueError(f"unknown length recipe {kind!r}")


def make_inputs(
    seqlens: Sequence[int],
    h_q: int,
    s_q: int = 1,
    *,
    seed: int = 0,
    causal: bool = False,
    softmax_scale: float = DEFAULT_SCALE,
    pool_factor: Optional[float] = 1.25,
    tail_fill: float = 1e4,
    poison: float = float("nan"),
    extra_table_cols: int = 0,
    device: str = "cpu",
    name: str = "",
) -> DecodeInputs:
    """Build one paged decode step with the given per-row lengths.

    ``extra_table_cols`` widens the block table past the longest row (the extra
    entries point at the poisoned page).  ``device`` only chooses where the
    random numbers are drawn: the CPU and CUDA generators give different
    streams for the same seed, so parity tests draw on the CPU.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    batch = len(seqlens)
    pages_per_row = [(int(L) + PAGE - 1) // PAGE for L in seqlens]
    needed = sum(pages_per_row)
    if pool_factor is None:
        pool = max(needed, 1)
    else:
        pool = max(int(math.ceil(pool_factor * needed)), needed + 1)
    perm = torch.randperm(pool, generator=gen, device=device).to("cpu")
    spare = int(perm[needed]) if pool > needed else 0
    width = max(max(pages_per_row, default=0), 1) + int(extra_table_cols)
    table = torch.full((batch, width), spare, dtype=torch.int32)
    cursor = 0
    for i, n in enumerate(pages_per_row):
        table[i, :n] = perm[cursor:cursor + n].to(torch.int32)
        cursor += n

    q = torch.randn(batch, s_q, h_q, D_QK, generator=gen, device=device).to(torch.bfloat16)
    kv = torch.empty(pool, PAGE, 1, D_QK, dtype=torch.bfloat16, device=device)
    chunk = 4096
    for p0 in range(0, pool, chunk):
        p1 = min(pool, p0 + chunk)
        kv[p0:p1] = torch.randn(p1 - p0, PAGE, 1, D_QK, generator=gen, device=device).to(torch.bfloat16)
    used = torch.zeros(pool, dtype=torch.bool)
    used[perm[:needed]] = True
    unused_ids = (~used).nonzero().flatten()
    if unused_ids.numel():
        kv[unused_ids.to(device)] = poison
    for i, (L, n) in enumerate(zip(seqlens, pages_per_row)):
        if n and L % PAGE:
            last = int(table[i, n - 1])
            kv[last, L % PAGE:] = tail_fill
    return DecodeInputs(
        q=q,
        kv_cache=kv,
        block_table=table.to(device),
        seqlens=torch.tensor([int(L) for L in seqlens], dtype=torch.int32, device=device),
        s_q=s_q,
        h_q=h_q,
        causal=causal,
        softmax_scale=softmax_scale,
        name=name,
    )


def workload_inputs(index_or_name, *, device: str = "cpu", seed_offset: int = 0, **overrides) -> DecodeInputs:
    """Inputs of one of the five standard workloads (seed ``1000 + index``)."""
    if isinstance(index_or_name, str):
        index, wl = BY_NAME[index_or_name]
    else:
        index, wl = int(index_or_name), WORKLOADS[int(index_or_name)]
    seed = 1000 + index + seed_offset
    gen = torch.Generator()
    gen.manual_seed(seed)
    lens = draw_lengths(wl.lengths, wl.batch, gen)
    kwargs = dict(
        seed=seed,
        causal=wl.causal,
        softmax_scale=wl.softmax_scale,
        pool_factor=wl.pool_factor,
        device=device,
        name=wl.name,
    )
    kwargs.update(overrides)
    return make_inputs(lens, wl.h_q, wl.s_q, **kwargs)



D_NOPE = 128  # per-head query dims without position (W_UK^h: [512][128])
D_VH = 128    # per-head value dims (W_UV^h: [512][128])


@dataclasses.dataclass
class ProjectionInputs:
    """Tensors of the projections either side of the absorbed decode."""

    q_nope: torch.Tensor    # [tokens, h_q, 128] bf16
    q_rope: torch.Tensor    # [tokens, h_q, 64] bf16
    w_uk: torch.Tensor      # [h_q, 512, 128] bf16, latent index first
    w_uv: torch.Tensor      # [h_q, 512, 128] bf16, latent index first
    o_latent: torch.Tensor  # [tokens, h_q, 512] bf16

    def to(self, device) -> "ProjectionInputs":
        return ProjectionInputs(*(getattr(self, f.name).to(device) for f in dataclasses.fields(self)))


def make_projection_inputs(tokens: int, h_q: int, *, seed: int = 0) -> ProjectionInputs:
    """Seeded N(0, 1) activations and N(0, 1 / fan-in) weights, rounded to bf16.

    The weights are scaled by the inverse square root of the summed dimension
    (128 for W_UK, 512 for W_UV) so that both products come out O(1), as a
    trained layer's would.  Drawn on the CPU generator.
    """
    gen = torch.Generator()
    gen.manual_seed(seed)

    def draw(*shape, scale=1.0):
        return (torch.randn(*shape, generator=gen) * scale).to(torch.bfloat16)

    return ProjectionInputs(
        q_nope=draw(tokens, h_q, D_NOPE),
        q_rope=draw(tokens, h_q, D_ROPE),
        w_uk=draw(h_q, D_LATENT, D_NOPE, scale=D_NOPE ** -0.5),
        w_uv=draw(h_q, D_LATENT, D_VH, scale=D_LATENT ** -0.5),
        o_latent=draw(tokens, h_q, D_LATENT),
    )


@dataclasses.dataclass
class Fp8DecodeInputs:
    """One decode step over an FP8 latent cache: E4M3 codes for the 512 latent
    dims with one power-of-two scale 2^exp per cached token, bf16 rope."""

    q: torch.Tensor             # [batch, s_q, h_q, 576] bf16
    latent_codes: torch.Tensor  # [num_pages, 64, 512] uint8 (E4M3 bit patterns)
    rope: torch.Tensor          # [num_pages, 64, 64] bf16
    exps: torch.Tensor          # [num_pages, 64] int8 (token scale 2^exp)
    block_table: torch.Tensor   # [batch, max_pages_per_row] int32
    seqlens: torch.Tensor       # [batch] int32
    s_q: int
    h_q: int
    causal: bool
    softmax_scale: float

    @property
    def batch(self) -> int:
        return int(self.seqlens.shape[0])

    def to(self, device) -> "Fp8DecodeInputs":
        return dataclasses.replace(self, q=self.q.to(device), latent_codes=self.latent_codes.to(device),
                                   rope=self.rope.to(device), exps=self.exps.to(device),
                                   block_table=self.block_table.to(device), seqlens=self.seqlens.to(device))


E4M3_NAN = 0x7F   # S.1111.111
E4M3_MAX = 0x7E   # 448


def make_fp8_inputs(seqlens: Sequence[int], h_q: int, s_q: int = 1, *, seed: int = 0, causal: bool = False,
                    softmax_scale: float = DEFAULT_SCALE, pool_factor: Optional[float] = 1.25,
                    exp_range: tuple = (-8, -6), device: str = "cpu") -> Fp8DecodeInputs:
    """Paged FP8 decode step drawn on the CPU generator.

    The latent codes are N(0, 64^2) values rounded to E4M3 (so that the
    codes span the format's range, |v| < 448), each token's exponent is
    uniform in ``exp_range`` (dequantised values ~ N(0, 1/16 .. 1)), rope and
    Q are N(0, 1) rounded to bf16.  Pages as in ``make_inputs``: a shuffled
    pool, table entries past a row's pages on a spare page whose codes are
    NaN, and slots past L in a row's last page holding the largest code with
    exponent 5 (14336: finite, large enough to be noticed if read).
    ``device`` only chooses where the random numbers are drawn (as in
    ``make_inputs``: parity tests draw on the CPU).
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    batch = len(seqlens)
    pages_per_row = [(int(L) + PAGE - 1) // PAGE for L in seqlens]
    needed = sum(pages_per_row)
    pool = max(needed, 1) if pool_factor is None else max(int(math.ceil(pool_factor * needed)), needed + 1)
    perm = torch.randperm(pool, generator=gen, device=device).to("cpu")
    spare = int(perm[needed]) if pool > needed else 0
    width = max(max(pages_per_row, default=0), 1)
    table = torch.full((batch, width), spare, dtype=torch.int32)
    cursor = 0
    for i, n in enumerate(pages_per_row):
        table[i, :n] = perm[cursor:cursor + n].to(torch.int32)
        cursor += n
    q = torch.randn(batch, s_q, h_q, D_QK, generator=gen, device=device).to(torch.bfloat16)
    codes = torch.empty(pool, PAGE, D_LATENT, dtype=torch.uint8, device=device)
    chunk = 4096
    for p0 in range(0, pool, chunk):
        p1 = min(pool, p0 + chunk)
        codes[p0:p1] = (torch.randn(p1 - p0, PAGE, D_LATENT, generator=gen, device=device) * 64.0).to(
            torch.float8_e4m3fn).view(torch.uint8)
    rope = torch.randn(pool, PAGE, D_ROPE, generator=gen, device=device).to(torch.bfloat16)
    exps = torch.randint(exp_range[0], exp_range[1] + 1, (pool, PAGE), generator=gen, dtype=torch.int64,
                         device=device).to(torch.int8)
    used = torch.zeros(pool, dtype=torch.bool)
    used[perm[:needed]] = True
    unused = (~used).nonzero().flatten().to(device)
    if unused.numel():
        codes[unused] = E4M3_NAN
        rope[unused] = float("nan")
    for i, (L, n) in enumerate(zip(seqlens, pages_per_row)):
        if n and int(L) % PAGE:
            last = int(table[i, n - 1])
            codes[last, int(L) % PAGE:] = E4M3_MAX
            exps[last, int(L) % PAGE:] = 5
    return Fp8DecodeInputs(q=q, latent_codes=codes.contiguous(), rope=rope, exps=exps, block_table=table.to(device),
                           seqlens=torch.tensor([int(L) for L in seqlens], dtype=torch.int32, device=device),
                           s_q=s_q, h_q=h_q, causal=causal, softmax_scale=softmax_scale)
