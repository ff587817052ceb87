"""Benchmark of the MLA decode hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload I]
                    [--no-cpu-baseline] [--headline-only]

A step is one pass of the whole path over one batch: the split-KV plan
(mla_get_metadata), the split-KV decode kernel and the log-sum-exp combine
(mla_decode), on inputs already resident in HBM.  The workload defaults to the
largest one-GPU configuration: the compute-bound speculative decode, batch
128, s_q 2 (causal within the two new tokens), h_q 128, 4096 cached tokens
per row (64-token pages, 1.25x shuffled pool, bf16 N(0, 1)).  Calls rotate
over several independent pools whose total size is at least 3x the L2 cache,
so each step reads its cache from HBM.  The timed region replays CUDA graphs
of those steps (exactly K steps, no event nodes between the kernels so that
programmatic dependent launch applies), bracketed by a barrier and a device
synchronisation, timed with CUDA events on the launching stream; the split-KV
kernel is also timed on its own, by graphs of the same steps with events
recorded around it, replayed right after the timed region.

The line also carries, for the headline workload:
  * `parity`: the GPU result on the workload's seeded inputs against the fp64
    oracle, element by element (every row when the oracle finishes them in
    about 25 s, else a seeded sample of at least 8 rows with the shortest and
    longest), with the parity bars (max-abs 8e-3, mean-abs 1e-3, lse 1e-3);
  * `cpu_baseline`: that same oracle run, timed and scaled to a full call;
  * `e2e`: the public API with pinned host buffers, inputs in and results out
    every step (at least 200 steps, rotating over the pools);
  * the projections either side of the decode and the split of one row over
    emulated ranks;
and, unless --headline-only, the same decode-kernel roofline, step time and
parity sample for the other four workloads (`memory_bound` is the
memory-bound sweep, `other_workloads` the rest).

With --gpus N > 1 (launched by torchrun, one process per GPU, NCCL), every
rank runs its own batch (batch rows are independent: weak scaling, no
collective on the data path); the step time is the maximum over ranks, and
`value` is the whole job's time per call: that step time over the N calls the
ranks make in it.

--impl reference times the fp64 CPU oracle on this host's cores instead (rank
0 only), one batch row per step, scaled to a full call.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_decode_attention_13_b200 import binding, inputs  # noqa: E402

METRIC = "MLA decode µs/call, achieved HBM GB/s and TFLOPS vs B200 roofline (1 GPU)"
DEFAULT_WORKLOAD = 3  # b128_s2_h128_L4k_causal: the largest configuration by bytes and FLOPs
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES = ("mla_decode.cu", "sm100_ptx.cuh", "mla_internal.h")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "mla_decode_kernel_traffic.json")
TOL_MAX, TOL_MEAN, TOL_LSE = 8e-3, 1e-3, 1e-3
# How every workload keeps its reads out of L2 between timed steps (the same
# words in both arms' config).
L2_NOTE = "inputs larger than L2: calls rotate over cache pools totalling at least 3x the L2 size"


# ----------------------------------------------------------------------------
# work accounting
# ----------------------------------------------------------------------------

def visible_pairs(lens, h_q, s_q, causal):
    n = 0
    for L in lens:
        for t in range(s_q):
            vis = min(max((L - s_q + t + 1) if causal else L, 0), L)
            n += h_q * vis
    return n


def algorithmic_work_fp8(lens, h_q, s_q, causal):
    """As algorithmic_work for an FP8 latent cache: every cached token once as
    512 E4M3 codes, 64 bf16 rope values and one exponent byte (641 B instead
    of 1152 B); the rest (Q, output, lse, table, lengths) and the FLOPs are
    unchanged."""
    rows = s_q * h_q
    tokens = sum(lens)
    pages = sum((L + 63) // 64 for L in lens)
    nbytes = tokens * (512 + 64 * 2 + 1) + len(lens) * rows * (576 * 2 + 512 * 2 + 4) + pages * 4 + len(lens) * 4
    flops = 2 * (576 + 512) * visible_pairs(lens, h_q, s_q, causal)
    return nbytes, flops


def algorithmic_work(lens, h_q, s_q, causal):
    """Bytes the decode kernel must move and FLOPs it must do.

    Bytes: every cached row once (576 bf16), Q (576 bf16 per query row), the
    bf16 output (512 per row), fp32 lse, one block-table entry per page and one
    length per row.  FLOPs: 2 * (576 + 512) per visible (query row, token).
    """
    rows = s_q * h_q
    tokens = sum(lens)
    pages = sum((L + 63) // 64 for L in lens)
    nbytes = tokens * 576 * 2 + len(lens) * rows * (576 * 2 + 512 * 2 + 4) + pages * 4 + len(lens) * 4
    flops = 2 * (576 + 512) * visible_pairs(lens, h_q, s_q, causal)
    return nbytes, flops


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def roofline_entry(nbytes, flops, k2_s, hbm_peak, tf_peak, peak_kind, traffic, timing):
    """The decode kernel against the roof that bounds its workload.

    The bound is the larger of the two ideal times: algorithmic bytes at the
    measured HBM copy bandwidth, or FLOPs at the measured bf16 GEMM rate (the
    burst figure: the kernel is timed on its own).  The other fraction is
    reported beside it.
    """
    t_hbm = nbytes / (hbm_peak * 1e9)
    t_tc = flops / (tf_peak * 1e12)
    ok = k2_s > 0
    gbs = nbytes / k2_s / 1e9 if ok else None
    tfs = flops / k2_s / 1e12 if ok else None
    entry = {"kernel": "mla_decode_kernel", "algorithmic_bytes_per_launch": nbytes, "flops_per_launch": flops,
             "traffic": traffic, "timing": timing}
    if t_tc > t_hbm:
        entry.update({"bound": "tensor", "achieved": round(tfs, 1) if ok else None, "peak": tf_peak,
                      "unit": "TFLOP/s", "frac": round(tfs / tf_peak, 4) if ok else None,
                      "peak_source": f"{peak_kind} bf16_tflops",
                      "hbm_frac": round(gbs / hbm_peak, 4) if ok else None})
    else:
        entry.update({"bound": "hbm", "achieved": round(gbs, 1) if ok else None, "peak": hbm_peak,
                      "unit": "GB/s", "frac": round(gbs / hbm_peak, 4) if ok else None,
                      "peak_source": f"{peak_kind} hbm_gbs",
                      "tensor_frac_of_measured_bf16": round(tfs / tf_peak, 4) if ok else None})
    return {k: entry[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic", "kernel",
                                  "algorithmic_bytes_per_launch", "flops_per_launch", "peak_source",
                                  "hbm_frac" if "hbm_frac" in entry else "tensor_frac_of_measured_bf16",
                                  "timing")}


def strip_comments(src):
    """C/C++/CUDA source without its comments and blank lines, trailing
    spaces dropped (string and character literals are kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        ch = src[i]
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif ch in "\"'":
            j = i + 1
            while j < n and src[j] != ch:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(ch)
            i += 1
    lines = (line.rstrip() for line in "".join(out).split("\n"))
    return "\n".join(line for line in lines if line)


def kernel_source_sha():
    """Hash of the decode kernel's code (its comments and blank lines
    removed): the ncu figures in TRAFFIC_FILE hold while it is unchanged."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "mla_decode_attention_13_b200", "csrc", name), encoding="utf-8") as f:
            h.update(strip_comments(f.read()).encode("utf-8"))
    return h.hexdigest()[:16]


def committed_traffic(workload_name):
    """DRAM bytes (read + write) per decode-kernel launch from the ncu capture
    recorded in profiles/mla_decode_kernel_traffic.json, if that capture was
    taken on the current kernel source (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("source_sha") != kernel_source_sha():
        return None
    v = d.get("workloads", {}).get(workload_name)
    return int(v) if v is not None else None


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML (read-only)."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            try:
                nvml_index = torch.cuda._get_nvml_device_index(index)
            except Exception:
                nvml_index = index
            self._h = pynvml.nvmlDeviceGetHandleByIndex(nvml_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= self._reasons(self._h)
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        s = sorted(self.samples)
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(s)}


# ----------------------------------------------------------------------------
# distributed plumbing (one process per GPU)
# ----------------------------------------------------------------------------

def dist_setup(backend="nccl"):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def dist_teardown(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


# ----------------------------------------------------------------------------
# the oracle: the reference arm, the CPU baseline and the parity check
# ----------------------------------------------------------------------------

def cpu_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle_rows(x, rows_per_step, steps, warmup):
    from oracle import mla_oracle

    times = []
    b = x.batch
    for k in range(warmup + steps):
        rows = [(k * rows_per_step + j) % b for j in range(rows_per_step)]
        t0 = time.perf_counter()
        mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, rows=rows)
        dt = time.perf_counter() - t0
        if k >= warmup:
            times.append(dt)
    return times


def workload_config(wl, idx, lens):
    """The workload's description, the same in both arms."""
    rec = wl.lengths
    return {"workload": wl.name, "batch": wl.batch, "s_q": wl.s_q, "h_q": wl.h_q, "h_kv": 1, "d_qk": 576,
            "d_v": 512, "page": 64, "causal": wl.causal, "lengths": str(rec[0]) + str(list(rec[1:]))[:60],
            "tokens": int(sum(lens)), "seed": 1000 + idx, "l2": L2_NOTE}


def workload_lengths(idx):
    wl = inputs.WORKLOADS[idx]
    gen = torch.Generator()
    gen.manual_seed(1000 + idx)
    return inputs.draw_lengths(wl.lengths, wl.batch, gen)


def reference_arm(args, world, rank):
    if rank != 0:
        return
    idx = args.workload
    wl = inputs.WORKLOADS[idx]
    x = inputs.workload_inputs(idx)
    lens = x.seqlens.tolist()
    # calibrate one row, then keep the whole run within a few minutes
    t_row = min(time_oracle_rows(x, 1, 2, 0))
    steps, warmup = args.steps, args.warmup
    t0 = time.perf_counter()
    times = time_oracle_rows(x, 1, steps, warmup)
    elapsed = time.perf_counter() - t0
    per_row = sum(times) / len(times)
    us_per_call = per_row * x.batch * 1e6
    nbytes, flops = algorithmic_work(lens, wl.h_q, wl.s_q, wl.causal)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(us_per_call, 3), "unit": "us/call", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(per_row * 1e3, 4), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, idx, lens),
        "achieved_gbs": round(nbytes / (us_per_call * 1e-6) / 1e9, 3),
        "achieved_tflops": round(flops / (us_per_call * 1e-6) / 1e12, 6),
        "cpu_baseline": {"value": round(us_per_call, 3), "unit": "us/call", "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"one batch row per step (of {x.batch}), {steps} timed steps, scaled x{x.batch}; "
                                   f"calibration {t_row * 1e3:.1f} ms/row, run {elapsed:.1f} s"},
        "e2e": {"value": round(us_per_call, 3), "unit": "us/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def sample_rows(lens, k, seed):
    """A seeded sample of k batch rows that includes the shortest and the longest."""
    order = sorted(range(len(lens)), key=lambda i: (lens[i], i))
    rows = {order[0], order[-1]}
    rng = np.random.default_rng(seed)
    for i in rng.permutation(len(lens)):
        if len(rows) >= k:
            break
        rows.add(int(i))
    return sorted(rows)


def parity_check(idx, dev, budget_s, min_rows=8, all_rows_ok=True):
    """The GPU result on the workload's seeded inputs (drawn on the CPU, as the
    tests draw them) against the fp64 oracle on the same inputs.

    Rows: all of them if the oracle's estimated time fits budget_s (and
    all_rows_ok), else a seeded sample of at least min_rows with the shortest
    and longest.  Returns (parity entry, oracle seconds per batch row, rows)."""
    from oracle import mla_oracle

    x = inputs.workload_inputs(idx)
    lens = [int(v) for v in x.seqlens]
    g = x.to(dev)
    meta = binding.mla_get_metadata(g.seqlens, g.h_q, g.s_q)
    out, lse = binding.mla_decode(g.q, g.kv_cache, g.block_table, g.seqlens, g.softmax_scale, g.causal, meta)
    torch.cuda.synchronize(dev)
    err = binding.mla_check_device_error(meta)
    got_o = out.cpu().double().numpy()
    got_l = lse.cpu().double().numpy()
    del g, meta, out, lse
    # the longest row first: it calibrates the oracle's cost per row
    longest = max(range(len(lens)), key=lambda i: (lens[i], i))
    t0 = time.perf_counter()
    mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, rows=[longest])
    t_longest = time.perf_counter() - t0
    if all_rows_ok and t_longest * x.batch <= budget_s:
        rows = list(range(x.batch))
    else:
        k = max(min_rows, min(x.batch, int(budget_s / max(t_longest, 1e-6))))
        rows = sample_rows(lens, min(k, x.batch), seed=idx)
    t0 = time.perf_counter()
    want_o, want_l = mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal,
                                       rows=rows)
    t_oracle = time.perf_counter() - t0
    go, gl, wo, wl_ = got_o[rows], got_l[rows], want_o[rows], want_l[rows]
    d = np.abs(go - wo)
    inf = np.isneginf(wl_)
    neg_inf_match = bool(np.array_equal(np.isneginf(gl), inf))
    lse_max = float(np.abs(gl[~inf] - wl_[~inf]).max()) if (~inf).any() else 0.0
    finite = bool(np.isfinite(go).all())
    entry = {
        "max_abs": float(d.max()), "mean_abs": float(d.mean()), "lse_max_abs": lse_max,
        "neg_inf_match": neg_inf_match, "finite": finite, "device_error_word": int(err),
        "rows": len(rows) if len(rows) == x.batch else rows, "of_rows": x.batch,
        "elements": int(d.size),
        "tolerance": {"max_abs": TOL_MAX, "mean_abs": TOL_MEAN, "lse_max_abs": TOL_LSE},
        "pass": bool(d.max() <= TOL_MAX and d.mean() <= TOL_MEAN and lse_max <= TOL_LSE and neg_inf_match
                     and finite and err == 0),
        "inputs": "the workload's seeded inputs (seed 1000 + index, drawn on the CPU), one mla_decode call",
    }
    return entry, t_oracle / len(rows), rows


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

class Bench:
    """One workload's rotating pools, buffers and step graphs on this GPU
    (bf16 cache, or with fp8 the FP8 latent cache of mla_decode_fp8)."""

    def __init__(self, idx, dev, rank, stream, fp8=False):
        self.idx = idx
        self.fp8 = fp8
        self.wl = wl = inputs.WORKLOADS[idx]
        self.dev = dev
        self.stream = stream
        self.lens = workload_lengths(idx)
        self.l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        pools, total = [], 0
        while len(pools) < 2 or total < 3 * self.l2:
            seed = 1000 + idx + 7919 * (len(pools) + 1) + 104729 * rank
            if fp8:
                one = inputs.make_fp8_inputs(self.lens, wl.h_q, wl.s_q, seed=seed, causal=wl.causal,
                                             softmax_scale=wl.softmax_scale, pool_factor=wl.pool_factor,
                                             device=str(dev))
                total += sum(t.numel() * t.element_size() for t in (one.latent_codes, one.rope, one.exps, one.q))
            else:
                one = inputs.make_inputs(self.lens, wl.h_q, wl.s_q, seed=seed, causal=wl.causal,
                                         softmax_scale=wl.softmax_scale, pool_factor=wl.pool_factor, device=str(dev),
                                         name=wl.name)
                total += one.kv_cache.numel() * 2 + one.q.numel() * 2
            pools.append(one)
            if len(pools) >= 64:
                break
        self.pools, self.total = pools, total
        self.npool = len(pools)
        ws_bytes = max(binding.mla_workspace_bytes(wl.batch, wl.h_q, wl.s_q), 16)
        with torch.cuda.stream(stream):
            self.metas = [torch.empty(binding.mla_metadata_bytes(wl.batch, wl.h_q, wl.s_q) // 4, dtype=torch.int32,
                                      device=dev) for _ in range(self.npool)]
            self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
            self.out = torch.empty(wl.batch, wl.s_q, wl.h_q, 512, dtype=torch.bfloat16, device=dev)
            self.lse = torch.empty(wl.batch, wl.h_q, wl.s_q, dtype=torch.float32, device=dev)
        torch.cuda.synchronize(dev)

    def step(self, r, events=None):
        x = self.pools[r]
        binding.mla_get_metadata(x.seqlens, x.h_q, x.s_q, metadata=self.metas[r], stream=self.stream)
        if self.fp8:
            binding.mla_decode_fp8(x.q, x.latent_codes, x.rope, x.exps, x.block_table, x.seqlens, x.softmax_scale,
                                   x.causal, self.metas[r], workspace=self.ws, out=self.out, lse=self.lse,
                                   stream=self.stream, events=events)
        else:
            binding.mla_decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, self.metas[r],
                               workspace=self.ws, out=self.out, lse=self.lse, stream=self.stream, events=events)

    def warm_up(self, n):
        for k in range(max(n, 1)):
            self.step(k % self.npool)
        self.stream.synchronize()
        for m in self.metas:
            err = binding.mla_check_device_error(m, stream=self.stream)
            if err:
                raise RuntimeError(f"device error word {err:#x} during warm-up ({self.wl.name})")
        err = binding.mla_take_device_errors(stream=self.stream)  # each plan rewrites its own word: the sticky bits
        if err:
            raise RuntimeError(f"device error bits {err:#x} during warm-up ({self.wl.name})")

    def capture(self):
        """One graph cycling over the pools, the same with events around each
        split-KV kernel, and one single-step graph per pool (so that exactly K
        steps can run)."""
        s = self.stream
        self.ev_pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                         for _ in range(self.npool)]
        for a, b in self.ev_pairs:
            a.record(s)
            b.record(s)
        s.synchronize()
        # The timed graphs hold no event nodes between the kernels, so that each
        # kernel can launch while its predecessor finishes (programmatic
        # dependent launch); the graph with events times the split-KV kernel.
        self.cycle = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.cycle, stream=s):
            for r in range(self.npool):
                self.step(r)
        self.cycle_k2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.cycle_k2, stream=s):
            for r in range(self.npool):
                self.step(r, events=self.ev_pairs[r])
        self.singles = []
        for r in range(self.npool):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                self.step(r)
            self.singles.append(g)
        with torch.cuda.stream(s):
            for _ in range(2):
                self.cycle.replay()
                self.cycle_k2.replay()
        s.synchronize()

    def timed_steps(self, K, world, local):
        """Exactly K steps, bracketed by a barrier and a device sync; max over ranks."""
        reps, rem = divmod(K, self.npool)
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        s = self.stream
        barrier(world)
        torch.cuda.synchronize(self.dev)
        with ClockSampler(local) as clocks:
            with torch.cuda.stream(s):
                start.record(s)
                for _ in range(reps):
                    self.cycle.replay()
                for r in range(rem):
                    self.singles[r].replay()
                end.record(s)
            s.synchronize()
        torch.cuda.synchronize(self.dev)
        barrier(world)
        ms_total = max_over_ranks(start.elapsed_time(end), world, self.dev)
        return ms_total / K, clocks.summary()

    def decode_kernel_timing(self, K, local):
        """The split-KV kernel alone: events around it in graph replays of the
        same steps, started from an idle GPU (the power cap lowers the SM clock
        within a tenth of a second of sustained load), median of the launches."""
        n_cycles = max(1, min(max(K // self.npool, 1), 20))
        source = ("events around the split-KV kernel, graph replays of the same steps after a 0.3 s idle pause "
                  "(median of %d launches: %d cycles over the pools)" % (n_cycles * self.npool, n_cycles))
        k2_ms = []
        time.sleep(0.3)
        with ClockSampler(local) as clk:
            for _ in range(n_cycles):
                with torch.cuda.stream(self.stream):
                    self.cycle_k2.replay()
                self.stream.synchronize()
                k2_ms += [a.elapsed_time(b) for a, b in self.ev_pairs]
        return sorted(k2_ms)[len(k2_ms) // 2], source, clk.summary()

    def release(self):
        for name in ("cycle", "cycle_k2", "singles", "pools", "metas", "ws", "out", "lse"):
            if hasattr(self, name):
                delattr(self, name)
        torch.cuda.synchronize(self.dev)
        torch.cuda.empty_cache()


def per_layer_timing(B, K, world):
    """The plan is made once per decode step and reused by every layer: one
    graph of a plan on the shared lengths, then a decode call over each pool in
    turn (a pool stands for a layer's cache; all pools share the lengths),
    timed whole and divided by the calls."""
    n_layers = max(8, B.npool)
    s = B.stream
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        x0 = B.pools[0]
        binding.mla_get_metadata(x0.seqlens, x0.h_q, x0.s_q, metadata=B.metas[0], stream=s)
        for layer in range(n_layers):
            x = B.pools[layer % B.npool]
            binding.mla_decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, B.metas[0],
                               workspace=B.ws, out=B.out, lse=B.lse, stream=s)
    l0 = torch.cuda.Event(enable_timing=True)
    l1 = torch.cuda.Event(enable_timing=True)
    time.sleep(0.3)
    with torch.cuda.stream(s):
        g.replay()
        l0.record(s)
        n_rep = max(1, min(20, K // n_layers))
        for _ in range(n_rep):
            g.replay()
        l1.record(s)
    s.synchronize()
    us = max_over_ranks(l0.elapsed_time(l1) * 1e3 / (n_rep * n_layers), world, B.dev)
    del g
    return {"value": round(us, 3), "unit": "us/call",
            "note": (f"one plan, then {n_layers} decode calls (split-KV + combine) on it over the rotating pools, "
                     f"graph-replayed {n_rep} times; the plan's cost spread over the calls")}


def e2e_timing(B, K, world):
    """End to end through the public API: every step copies its inputs (q,
    block table, lengths) in from pinned host memory and its result (out, lse)
    back, as a serving loop would, rotating over the pools (each pool's inputs
    have a pinned host copy of their own).  Copies run on two copy streams,
    double-buffered, so that step n + 1's inputs go in and step n - 1's result
    comes out while step n computes."""
    dev, stream = B.dev, B.stream
    steps = max(200, min(K, 2000))

    def layout(tensors):
        offs, n = [], 0
        for t in tensors:
            offs.append(n)
            n += (t.numel() * t.element_size() + 15) // 16 * 16
        return offs, n

    def views(buf, offs, like):
        return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for o, t in zip(offs, like)]

    like_in = [B.pools[0].q, B.pools[0].block_table, B.pools[0].seqlens]
    in_offs, in_bytes = layout(like_in)
    h_in = []
    for x in B.pools:
        h = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
        for v, t in zip(views(h, in_offs, like_in), (x.q, x.block_table, x.seqlens)):
            v.copy_(t.cpu())
        h_in.append(h)
    res_like = [B.out, B.lse]
    res_offs, res_bytes = layout(res_like)
    h_res = [torch.empty(res_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
    d_in = [torch.empty(in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    d_res = [torch.empty(res_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    d_q, d_table, d_lens = zip(*[views(d, in_offs, like_in) for d in d_in])
    d_out, d_lse = zip(*[views(d, res_offs, res_like) for d in d_res])
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    in_done = [torch.cuda.Event(), torch.cuda.Event()]
    comp_done = [torch.cuda.Event(), torch.cuda.Event()]
    out_done = [torch.cuda.Event(), torch.cuda.Event()]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    wl = B.wl

    def run(n):
        b, r = n & 1, n % B.npool
        with torch.cuda.stream(s_in):
            if n >= 2:
                s_in.wait_event(comp_done[b])  # step n - 2 no longer reads these inputs
            d_in[b].copy_(h_in[r], non_blocking=True)
            in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        if n >= 2:
            stream.wait_event(out_done[b])  # step n - 2's result has left this buffer
        binding.mla_get_metadata(d_lens[b], wl.h_q, wl.s_q, metadata=B.metas[b % B.npool], stream=stream)
        binding.mla_decode(d_q[b], B.pools[r].kv_cache, d_table[b], d_lens[b], wl.softmax_scale, wl.causal,
                           B.metas[b % B.npool], workspace=B.ws, out=d_out[b], lse=d_lse[b], stream=stream)
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            h_res[b].copy_(d_res[b], non_blocking=True)
            out_done[b].record(s_out)

    for n in range(4):  # untimed: first calls of the copy streams and of the API on these buffers
        run(n)
    torch.cuda.synchronize(dev)
    barrier(world)
    time.sleep(0.3)  # start from an idle GPU, as the other timed phases do
    e0.record(s_in)
    for n in range(steps):
        run(n)
    s_out.wait_event(comp_done[(steps - 1) & 1])
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    err = binding.mla_take_device_errors(stream=stream)
    if err:
        raise RuntimeError(f"device error bits {err:#x} in the end-to-end steps")
    # the last step's result, as it came back, against a call on that pool's device-resident inputs
    last = steps - 1
    x = B.pools[last % B.npool]
    binding.mla_get_metadata(x.seqlens, x.h_q, x.s_q, metadata=B.metas[0], stream=stream)
    binding.mla_decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, B.metas[0],
                       workspace=B.ws, out=B.out, lse=B.lse, stream=stream)
    stream.synchronize()
    got = views(h_res[last & 1], res_offs, res_like)
    same = bool(torch.equal(got[0], B.out.cpu()) and torch.equal(got[1], B.lse.cpu()))
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
    return {"value": round(ms * 1e3 / world, 3), "unit": "us/call", "h2d_bytes_per_step": in_bytes,
            "d2h_bytes_per_step": res_bytes, "steps": steps,
            "pcie_gbs_each_way": round(max(in_bytes, res_bytes) / (ms * 1e-3) / 1e9, 1),
            "last_result_equals_device_call": same,
            "note": ("pinned q/block_table/seqlens in (one packed copy per step, from the step's pool), out/lse "
                     "back (one packed copy), every step, on copy streams of their own, double-buffered so that "
                     "copies overlap the neighbouring steps' compute; calls rotate over the cache pools, which stay "
                     "resident in HBM (the model state a decode step appends to)")}


def roofline_for(B, k2_ms, k2_source, peaks):
    hbm_peak, tf_peak, _, peak_kind = peaks
    work = algorithmic_work_fp8 if B.fp8 else algorithmic_work
    nbytes, flops = work(B.lens, B.wl.h_q, B.wl.s_q, B.wl.causal)
    traffic = committed_traffic(("fp8:" if B.fp8 else "") + B.wl.name)
    entry = roofline_entry(nbytes, flops, k2_ms * 1e-3, hbm_peak, tf_peak, peak_kind, traffic, k2_source)
    if B.fp8:
        entry["kernel"] = "mla_decode_kernel (FP8 latent cache)"
    return entry, nbytes, flops


def parity_check_fp8(idx, dev, min_rows=8):
    """The FP8-cache decode on seeded inputs of the workload's shape (drawn on
    the CPU) against the oracle's decode_fp8, on a seeded sample of at least
    min_rows rows with the shortest and longest (every row when there are
    no more)."""
    from oracle import mla_oracle

    wl = inputs.WORKLOADS[idx]
    lens = workload_lengths(idx)
    x = inputs.make_fp8_inputs(lens, wl.h_q, wl.s_q, seed=3000 + idx, causal=wl.causal,
                               softmax_scale=wl.softmax_scale, pool_factor=wl.pool_factor)
    g = x.to(dev)
    meta = binding.mla_get_metadata(g.seqlens, g.h_q, g.s_q)
    out, lse = binding.mla_decode_fp8(g.q, g.latent_codes, g.rope, g.exps, g.block_table, g.seqlens,
                                      g.softmax_scale, g.causal, meta)
    torch.cuda.synchronize(dev)
    err = binding.mla_check_device_error(meta)
    got_o = out.cpu().double().numpy()
    got_l = lse.cpu().double().numpy()
    del g, meta, out, lse
    rows = sample_rows(lens, min(min_rows, wl.batch), seed=idx)
    want_o, want_l = mla_oracle.decode_fp8(x.q, x.latent_codes, x.rope, x.exps, x.block_table, x.seqlens,
                                           x.softmax_scale, x.causal, rows=rows)
    go, gl, wo, wl_ = got_o[rows], got_l[rows], want_o[rows], want_l[rows]
    d = np.abs(go - wo)
    inf = np.isneginf(wl_)
    neg_inf_match = bool(np.array_equal(np.isneginf(gl), inf))
    lse_max = float(np.abs(gl[~inf] - wl_[~inf]).max()) if (~inf).any() else 0.0
    finite = bool(np.isfinite(go).all())
    return {"max_abs": float(d.max()), "mean_abs": float(d.mean()), "lse_max_abs": lse_max,
            "neg_inf_match": neg_inf_match, "finite": finite, "device_error_word": int(err),
            "rows": rows, "of_rows": wl.batch, "elements": int(d.size),
            "tolerance": {"max_abs": TOL_MAX, "mean_abs": TOL_MEAN, "lse_max_abs": TOL_LSE},
            "pass": bool(d.max() <= TOL_MAX and d.mean() <= TOL_MEAN and lse_max <= TOL_LSE and neg_inf_match
                         and finite and err == 0),
            "inputs": "seeded FP8 inputs of the workload's shape (seed 3000 + index, drawn on the CPU): E4M3 codes "
                      "of N(0, 64^2) values, token exponents uniform in [-8, -6], bf16 rope and q ~ N(0, 1)"}


def fp8_workload(idx, args, world, rank, local, dev, stream, peaks):
    """The FP8 latent cache (mla_decode_fp8) on a workload's shape: step
    time, decode-kernel roofline on the FP8 bytes, and a parity sample."""
    B = Bench(idx, dev, rank, stream, fp8=True)
    B.warm_up(args.warmup)
    B.capture()
    K = max(B.npool, min(args.steps, 200))
    ms_step, clocks = B.timed_steps(K, world, local)
    k2_ms, k2_source, k2_clocks = B.decode_kernel_timing(K, local)
    roof, nbytes, _ = roofline_for(B, k2_ms, k2_source, peaks)
    entry = {"config": {**workload_config(B.wl, idx, B.lens), "cache": "fp8 e4m3 latent + per-token 2^e + bf16 rope"},
             "step_us": round(ms_step * 1e3 / world, 3), "steps": K, "decode_kernel_us": round(k2_ms * 1e3, 3),
             "roofline": roof, "decode_kernel_clocks": k2_clocks, "clocks": clocks,
             "pools": f"{B.npool} rotating pools, {B.total / 2**20:.0f} MiB"}
    B.release()
    if world == 1 and not args.no_cpu_baseline:
        entry["parity"] = parity_check_fp8(idx, dev)
    return entry


def other_workload(idx, args, world, rank, local, dev, stream, peaks):
    """Another workload's step time, decode-kernel roofline and parity sample."""
    B = Bench(idx, dev, rank, stream)
    B.warm_up(args.warmup)
    B.capture()
    K = max(B.npool, min(args.steps, 200))
    ms_step, clocks = B.timed_steps(K, world, local)
    k2_ms, k2_source, k2_clocks = B.decode_kernel_timing(K, local)
    roof, _, _ = roofline_for(B, k2_ms, k2_source, peaks)
    entry = {"config": workload_config(B.wl, idx, B.lens), "step_us": round(ms_step * 1e3 / world, 3),
             "steps": K, "decode_kernel_us": round(k2_ms * 1e3, 3), "roofline": roof,
             "decode_kernel_clocks": k2_clocks, "clocks": clocks}
    B.release()
    if world == 1 and not args.no_cpu_baseline:
        entry["parity"], _, _ = parity_check(idx, dev, budget_s=3.0, min_rows=8, all_rows_ok=False)
    return entry


def ours(args, world, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    idx = args.workload
    stream = torch.cuda.Stream(dev)
    peaks = measured_peaks()
    K = args.steps

    B = Bench(idx, dev, rank, stream)
    wl = B.wl
    B.warm_up(args.warmup)
    B.capture()
    ms_step, clocks = B.timed_steps(K, world, local)
    k2_ms, k2_source, k2_clocks = B.decode_kernel_timing(K, local)
    layer = per_layer_timing(B, K, world)
    proj = split = None
    if not args.headline_only:
        proj = projection_timing(wl, B.pools, B.metas[0], B.ws, B.out, B.lse, stream, dev, B.l2, world, local,
                                 max(8, B.npool))
        split = long_row_timing(wl, B.pools, stream, dev, world, local)
    # The sticky bits cover every call since warm-up (each plan rewrites the
    # word in its own metadata, so those only show the last cycle).
    err = binding.mla_take_device_errors(stream=stream)
    if err:
        raise RuntimeError(f"device error bits {err:#x} in the timed region or the kernel timing replays")
    e2e = e2e_timing(B, K, world)
    roof, nbytes, flops = roofline_for(B, k2_ms, k2_source, peaks)
    npool, total, l2 = B.npool, B.total, B.l2
    B.release()

    line = {
        "metric": METRIC,
        # Whole job: the calls all ranks made over the time they took (each
        # rank makes one call per step; with one GPU this is the step time).
        "value": round(ms_step * 1e3 / world, 3),
        "unit": "us/call",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 6),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(wl, idx, B.lens),
        "pools": f"{npool} rotating pools, {total / 2**20:.0f} MiB > 3x {l2 / 2**20:.0f} MiB L2; timed via CUDA "
                 f"graph replay",
        "achieved_gbs": round(world * nbytes / (ms_step * 1e-3) / 1e9, 1),
        "achieved_tflops": round(world * flops / (ms_step * 1e-3) / 1e12, 2),
        "calls_per_s_all_ranks": round(world / (ms_step * 1e-3), 1),
        "decode_kernel_us": round(k2_ms * 1e3, 3),
        "roofline": roof,
        "decode_kernel_clocks": k2_clocks,
        "e2e": e2e,
        "per_layer": layer,
        "gpu_launches": 3 * K,
        "clocks": clocks,
    }
    if proj is not None:
        line["projections"] = proj
        line["long_row_split"] = split
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        par, t_row, rows = parity_check(idx, dev, budget_s=25.0)
        line["parity"] = par
        line["cpu_baseline"] = {
            "value": round(t_row * wl.batch * 1e6, 1), "unit": "us/call", "cores": cpu_threads(), "kind": "oracle",
            "sample": (f"the parity check's oracle run (fp64 NumPy) over {len(rows)} of {wl.batch} batch rows of the "
                       f"same workload, scaled to all {wl.batch} rows")}
        if proj is not None:
            line["projections"]["cpu_baseline"] = oracle_projection_and_merge(wl)
    if not args.headline_only:
        others = {}
        for j in range(len(inputs.WORKLOADS)):
            if j != idx:
                others[inputs.WORKLOADS[j].name] = other_workload(j, args, world, rank, local, dev, stream, peaks)
        mb = inputs.WORKLOADS[2].name
        if mb in others:
            line["memory_bound"] = others.pop(mb)
        line["other_workloads"] = others
        # The FP8 latent cache on the memory-bound sweep's shape and the
        # headline's.
        line["fp8_cache"] = {inputs.WORKLOADS[j].name: fp8_workload(j, args, world, rank, local, dev, stream, peaks)
                             for j in (2, idx) if j < len(inputs.WORKLOADS)}
    if rank == 0:
        print(json.dumps(line), flush=True)


def ours_fp8(args, world, rank, local):
    """--fp8: the workload's step on the FP8 latent cache, one JSON line (for
    profiling runs of that kernel; the default line carries the same entry
    under fp8_cache)."""
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(dev)
    e = fp8_workload(args.workload, args, world, rank, local, dev, stream, measured_peaks())
    if rank == 0:
        print(json.dumps({"metric": METRIC, "value": e["step_us"], "unit": "us/call", "n_gpus": world,
                          "steps": e["steps"], "warmup": args.warmup, "higher_is_better": False, "scaling": "weak",
                          "vs_baseline": None, "dtype": "fp8 cache, f16/bf16 MMAs", "data": "synthetic", **e}),
              flush=True)


def projection_work(tokens, h_q):
    """Algorithmic bytes of one absorb and one up-projection launch: the head
    weights once, the tokens' inputs once, the outputs once (bf16)."""
    w = h_q * 512 * 128 * 2
    absorb = w + tokens * h_q * (128 + 64) * 2 + tokens * h_q * 576 * 2
    up = w + tokens * h_q * 512 * 2 + tokens * h_q * 128 * 2
    return absorb, up


def projection_timing(wl, pools, meta, ws, out, lse, stream, dev, l2, world, local, n_layers):
    """The projections either side of the decode, on the workload's tokens.

    Each kernel is timed as the mean launch of a graph that runs it over
    rotating weight sets (more than 3x L2 in all, so the weights come from
    HBM), back to back; then one layer call (absorb -> decode -> up-project)
    is timed the same way, with the plan made once per graph."""
    tokens = wl.batch * wl.s_q
    sets, total = [], 0
    while len(sets) < 2 or total < 3 * l2:
        x = inputs.make_projection_inputs(tokens, wl.h_q, seed=5000 + len(sets)).to(dev)
        sets.append(x)
        total += sum(t.numel() * 2 for t in (x.w_uk, x.w_uv, x.q_nope, x.q_rope, x.o_latent))
        if len(sets) >= 128:
            break
    n = len(sets)
    with torch.cuda.stream(stream):
        q_abs = torch.empty(tokens, wl.h_q, 576, dtype=torch.bfloat16, device=dev)
        o_up = torch.empty(tokens, wl.h_q, 128, dtype=torch.bfloat16, device=dev)
    graphs = {}
    for name in ("absorb", "up_project"):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for x in sets:
                if name == "absorb":
                    binding.mla_absorb_q(x.q_nope, x.q_rope, x.w_uk, out=q_abs, stream=stream)
                else:
                    binding.mla_up_project(x.o_latent, x.w_uv, out=o_up, stream=stream)
        graphs[name] = g
    layer = torch.cuda.CUDAGraph()
    q_layer = [torch.empty_like(p.q) for p in pools[:2]]
    with torch.cuda.graph(layer, stream=stream):
        x0 = pools[0]
        binding.mla_get_metadata(x0.seqlens, x0.h_q, x0.s_q, metadata=meta, stream=stream)
        for k in range(n_layers):
            x, w = pools[k % len(pools)], sets[k % n]
            qb = q_layer[k & 1]
            binding.mla_absorb_q(w.q_nope, w.q_rope, w.w_uk, out=qb.view(tokens, wl.h_q, 576), stream=stream)
            binding.mla_decode(qb, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, meta,
                               workspace=ws, out=out, lse=lse, stream=stream)
            binding.mla_up_project(out.view(tokens, wl.h_q, 512), w.w_uv, out=o_up, stream=stream)
    graphs["layer"] = layer
    with torch.cuda.stream(stream):
        for g in graphs.values():
            g.replay()
    stream.synchronize()
    res = {}
    for name, g in graphs.items():
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        reps = 10
        time.sleep(0.3)  # from an idle GPU, as the other timed phases
        with ClockSampler(local) as clk:
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            stream.synchronize()
        per = n_layers if name == "layer" else n
        res[name] = (max_over_ranks(e0.elapsed_time(e1) * 1e3 / (reps * per), world, dev), clk.summary())
    del graphs, layer
    hbm_peak = measured_peaks()[0]
    b_abs, b_up = projection_work(tokens, wl.h_q)
    entry = {}
    for name, nbytes in (("absorb", b_abs), ("up_project", b_up)):
        us = res[name][0]
        gbs = nbytes / (us * 1e-6) / 1e9
        entry[name] = {"us": round(us, 3), "bytes": nbytes,
                       "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                                    "frac": round(gbs / hbm_peak, 3)},
                       "clocks": res[name][1]}
    entry["layer_with_projections"] = {
        "value": round(res["layer"][0], 3), "unit": "us/call", "clocks": res["layer"][1],
        "note": (f"one plan, then {n_layers} calls of absorb -> decode (split-KV + combine) -> up-project, "
                 f"graph-replayed; weights rotate over {n} sets")}
    entry["note"] = (f"{tokens} tokens x {wl.h_q} heads; each kernel is the mean launch of a graph over {n} weight "
                     f"sets ({total / 2**20:.0f} MiB > 3x L2), launched back to back")
    return entry


def oracle_projection_and_merge(wl, budget_s=4.0):
    """The oracle, as it stands, on bounded samples of the same shapes: the two
    projections on one token of every head (scaled to the step's tokens), and
    the merge of 4 splits over a sample of query rows (scaled to all rows)."""
    from oracle import mla_oracle

    tokens = wl.batch * wl.s_q
    x = inputs.make_projection_inputs(1, wl.h_q, seed=99)
    res = {}
    for name, fn in (("absorb", lambda: mla_oracle.absorb_query(x.q_nope[0], x.q_rope[0], x.w_uk)),
                     ("up_project", lambda: mla_oracle.expand_output(x.o_latent[0], x.w_uv))):
        times = []
        t_start = time.perf_counter()
        while not times or (time.perf_counter() - t_start < budget_s / 3 and len(times) < 20):
            t0 = time.perf_counter()
            fn()
            times.append(time.perf_counter() - t0)
        res[name + "_us"] = round(sum(times) / len(times) * tokens * 1e6, 1)
    rows = wl.batch * wl.s_q * wl.h_q
    sample = min(rows, 256)
    gen = torch.Generator()
    gen.manual_seed(98)
    parts = [((torch.randn(sample, 512, generator=gen) * 0.25).double().numpy(),
              torch.randn(sample, generator=gen).double().numpy()) for _ in range(4)]
    t0 = time.perf_counter()
    mla_oracle.combine_partials(parts)
    res["merge_4_splits_us"] = round((time.perf_counter() - t0) * rows / sample * 1e6, 1)
    res.update(unit="us/call", cores=cpu_threads(), kind="oracle",
               sample=(f"projections: one token of all {wl.h_q} heads, x {tokens} tokens; merge: {sample} of "
                       f"{rows} query rows, x {rows / sample:g}"))
    return res


def long_row_timing(wl, pools, stream, dev, world, local):
    """The split of each row across W ranks (longrow), with the ranks emulated
    one after another on this GPU: each rank's plan + decode call on its share
    of the pages (graph over the rotating pools, mean per call), and the merge
    of the W partial results.  The exchange between GPUs is not timed here
    (one GPU); its bytes per rank are reported."""
    from mla_decode_attention_13_b200 import longrow

    lens = [int(v) for v in pools[0].seqlens.cpu()]
    rows = wl.batch * wl.s_q * wl.h_q
    res = {}
    for W in (2, 4):
        rank_us, outs, lses = [], [], []
        for r in range(W):
            shards = [longrow.shard_block_table(x.block_table, lens, W, r, wl.s_q) for x in pools]
            with torch.cuda.stream(stream):
                meta = torch.empty(binding.mla_metadata_bytes(wl.batch, wl.h_q, wl.s_q) // 4, dtype=torch.int32,
                                   device=dev)
                ws = torch.empty(max(binding.mla_workspace_bytes(wl.batch, wl.h_q, wl.s_q), 16), dtype=torch.uint8,
                                 device=dev)
                o = torch.empty(wl.batch, wl.s_q, wl.h_q, 512, dtype=torch.bfloat16, device=dev)
                l = torch.empty(wl.batch, wl.h_q, wl.s_q, dtype=torch.float32, device=dev)
            causal_r = bool(wl.causal) and r == W - 1

            def call(k):
                x, (tab, ln) = pools[k], shards[k]
                binding.mla_get_metadata(ln, x.h_q, x.s_q, metadata=meta, stream=stream)
                binding.mla_decode(x.q, x.kv_cache, tab, ln, x.softmax_scale, causal_r, meta, workspace=ws, out=o,
                                   lse=l, stream=stream)

            for k in range(len(pools)):
                call(k)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for k in range(len(pools)):
                    call(k)
            with torch.cuda.stream(stream):
                g.replay()
            stream.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 10
            time.sleep(0.3)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            stream.synchronize()
            rank_us.append(max_over_ranks(e0.elapsed_time(e1) * 1e3 / (reps * len(pools)), world, dev))
            del g
            # the last pool's partial result, for the merge
            outs.append(o.clone())
            lses.append(l.clone())
        outs_t, lses_t = torch.stack(outs), torch.stack(lses)
        with torch.cuda.stream(stream):
            m_out = torch.empty_like(outs[0])
            m_lse = torch.empty_like(lses[0])
            binding.mla_merge_splits(outs_t, lses_t, out=m_out, lse=m_lse, stream=stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        n_merge = 20
        with torch.cuda.graph(g, stream=stream):
            for _ in range(n_merge):
                binding.mla_merge_splits(outs_t, lses_t, out=m_out, lse=m_lse, stream=stream)
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        time.sleep(0.3)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(5):
                g.replay()
            e1.record(stream)
        stream.synchronize()
        merge_us = max_over_ranks(e0.elapsed_time(e1) * 1e3 / (5 * n_merge), world, dev)
        del g
        merge_bytes = (W + 1) * rows * (512 * 2 + 4)
        res[f"ranks_{W}"] = {
            "rank_call_us": [round(u, 3) for u in rank_us],
            "max_rank_call_us": round(max(rank_us), 3),
            "merge_us": round(merge_us, 3),
            "merge_bytes": merge_bytes,
            "merge_achieved_gbs": round(merge_bytes / (merge_us * 1e-6) / 1e9, 1),
            "exchange_bytes_per_rank": (W - 1) * rows * (512 * 2 + 4),
        }
    res["note"] = ("each row's pages cut over W ranks (page-aligned, the last rank masks); ranks emulated one after "
                   "another on this GPU, each a plan + decode call on its share (graph over the rotating pools, mean "
                   "per call); merge = mla_merge_splits of the W partials (graph, mean per launch, L2-resident "
                   "inputs as after an exchange); the all-gather between GPUs is not run on one GPU")
    return res


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD,
                    help=f"index into inputs.WORKLOADS ({DEFAULT_WORKLOAD} = headline)")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="run no oracle (no parity, no CPU baseline)")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the headline workload's step (no projections, split or other workloads)")
    ap.add_argument("--fp8", action="store_true",
                    help="time the workload's step on the FP8 latent cache (mla_decode_fp8) only")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup("nccl" if args.impl == "ours" else "gloo")
    try:
        if args.impl == "reference":
            reference_arm(args, world, rank)
        elif args.fp8:
            ours_fp8(args, world, rank, local)
        else:
            ours(args, world, rank, local)
    finally:
        dist_teardown(world)


if __name__ == "__main__":
    main()
