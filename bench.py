"""Benchmark of the MLA decode hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload I]

A step is one pass of the whole path over one batch: the split-KV plan
(mla_get_metadata), the split-KV decode kernel and the log-sum-exp combine
(mla_decode), on inputs already resident in HBM.  The workload defaults to
batch 16, s_q 1, h_q 128, lengths uniform in [1024, 4096] (64-token pages,
1.25x shuffled pool, bf16 N(0, 1)).  Calls rotate over several independent
pools whose total size is at least 3x the L2 cache, so each step reads its
cache from HBM.  The timed region replays CUDA graphs of those steps (exactly
K steps, no event nodes between the kernels so that programmatic dependent
launch applies), bracketed by a barrier and a device synchronisation, timed
with CUDA events on the launching stream; the split-KV kernel is also timed on
its own, by graphs of the same steps with events recorded around it, replayed
right after the timed region.

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
import re
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_decode_attention_13_b200 import binding, inputs  # noqa: E402

METRIC = "MLA decode µs/call, achieved HBM GB/s and TFLOPS vs B200 roofline (1 GPU)"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES = ("mla_decode.cu", "sm100_ptx.cuh", "mla_internal.h")


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


def kernel_source_sha():
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "mla_decode_attention_13_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(workload_name):
    """DRAM bytes per decode-kernel launch from the committed ncu summary, if
    it was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "mla_decode_kernel_traffic.md")
    if not os.path.exists(path):
        return None
    sha = kernel_source_sha()
    pat = re.compile(r"traffic_bytes_per_launch:\s*(\d+)\s+workload:\s*(\S+)\s+source_sha:\s*([0-9a-f]+)")
    for line in open(path):
        m = pat.search(line)
        if m and m.group(2) == workload_name and m.group(3) == sha:
            return int(m.group(1))
    return None


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
# the reference arm: the fp64 CPU oracle
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


def cpu_baseline(idx, budget_s):
    """The oracle, as it stands, on whole calls of the workload for about budget_s."""
    from oracle import mla_oracle

    x = inputs.workload_inputs(idx)
    times = []
    t_start = time.perf_counter()
    while not times or (time.perf_counter() - t_start < budget_s and len(times) < 50):
        t0 = time.perf_counter()
        mla_oracle.decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal)
        times.append(time.perf_counter() - t0)
    per_call = sum(times) / len(times)
    return {"value": round(per_call * 1e6, 1), "unit": "us/call", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{len(times)} whole oracle calls (fp64 NumPy, all {x.batch} rows) of the same workload"}


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
        "config": workload_config(wl, idx, lens, None),
        "achieved_gbs": round(nbytes / (us_per_call * 1e-6) / 1e9, 3),
        "achieved_tflops": round(flops / (us_per_call * 1e-6) / 1e12, 6),
        "cpu_baseline": {"value": round(us_per_call, 3), "unit": "us/call", "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"one batch row per step (of {x.batch}), {steps} timed steps, scaled x{x.batch}; "
                                   f"calibration {t_row * 1e3:.1f} ms/row, run {elapsed:.1f} s"},
        "e2e": {"value": round(us_per_call, 3), "unit": "us/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(wl, idx, lens, l2_note):
    rec = wl.lengths
    c = {"workload": wl.name, "batch": wl.batch, "s_q": wl.s_q, "h_q": wl.h_q, "h_kv": 1, "d_qk": 576, "d_v": 512,
         "page": 64, "causal": wl.causal, "lengths": str(rec[0]) + str(list(rec[1:]))[:60],
         "tokens": int(sum(lens)), "seed": 1000 + idx}
    if l2_note:
        c["l2"] = l2_note
    return c


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def ours(args, world, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    idx = args.workload
    wl = inputs.WORKLOADS[idx]
    gen = torch.Generator()
    gen.manual_seed(1000 + idx)
    lens = inputs.draw_lengths(wl.lengths, wl.batch, gen)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    one = None
    pools = []
    total = 0
    while len(pools) < 2 or total < 3 * l2:
        seed = 1000 + idx + 7919 * (len(pools) + 1) + 104729 * rank
        one = inputs.make_inputs(lens, wl.h_q, wl.s_q, seed=seed, causal=wl.causal, softmax_scale=wl.softmax_scale,
                                 pool_factor=wl.pool_factor, device=str(dev), name=wl.name)
        pools.append(one)
        total += one.kv_cache.numel() * 2 + one.q.numel() * 2
        if len(pools) >= 64:
            break
    npool = len(pools)
    stream = torch.cuda.Stream(dev)
    ws_bytes = max(binding.mla_workspace_bytes(wl.batch, wl.h_q, wl.s_q), 16)
    with torch.cuda.stream(stream):
        metas = [torch.empty(binding.mla_metadata_bytes(wl.batch, wl.h_q, wl.s_q) // 4, dtype=torch.int32, device=dev)
                 for _ in range(npool)]
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        out = torch.empty(wl.batch, wl.s_q, wl.h_q, 512, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(wl.batch, wl.h_q, wl.s_q, dtype=torch.float32, device=dev)
    torch.cuda.synchronize(dev)

    def step(r, events=None):
        x = pools[r]
        binding.mla_get_metadata(x.seqlens, x.h_q, x.s_q, metadata=metas[r], stream=stream)
        binding.mla_decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, metas[r],
                           workspace=ws, out=out, lse=lse, stream=stream, events=events)

    # warm-up (eager), and a check that no device error was raised
    for k in range(max(args.warmup, 1)):
        step(k % npool)
    stream.synchronize()
    for m in metas:
        err = binding.mla_check_device_error(m, stream=stream)
        if err:
            raise RuntimeError(f"device error word {err:#x} during warm-up")
    err = binding.mla_take_device_errors(stream=stream)  # every plan rewrites its metadata word: check the sticky bits
    if err:
        raise RuntimeError(f"device error bits {err:#x} during warm-up")

    # CUDA graphs: one cycle over all pools (with events around each split-KV
    # kernel) and one single-step graph per pool, so that exactly K steps run.
    ev_pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(npool)]
    for a, b in ev_pairs:
        a.record(stream)
        b.record(stream)
    stream.synchronize()
    # The timed graphs hold no event nodes between the kernels, so that each
    # kernel can launch while its predecessor finishes (programmatic dependent
    # launch); a separate graph with events around each split-KV kernel times
    # that kernel alone, replayed right after the timed region.
    cycle = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cycle, stream=stream):
        for r in range(npool):
            step(r)
    cycle_k2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cycle_k2, stream=stream):
        for r in range(npool):
            step(r, events=ev_pairs[r])
    singles = []
    for r in range(npool):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(r)
        singles.append(g)
    with torch.cuda.stream(stream):
        for _ in range(2):
            cycle.replay()
            cycle_k2.replay()
    stream.synchronize()

    K = args.steps
    reps, rem = divmod(K, npool)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(reps):
                cycle.replay()
            for r in range(rem):
                singles[r].replay()
            end.record(stream)
        stream.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    ms_total = start.elapsed_time(end)
    ms_total = max_over_ranks(ms_total, world, dev)
    ms_step = ms_total / K
    n_cycles = max(1, min(reps, 20))
    k2_source = ("events around the split-KV kernel, graph replays of the same steps right after the timed "
                 "region and a 0.3 s idle pause (median of %d launches: %d cycles over the pools)"
                 % (n_cycles * npool, n_cycles))
    k2_ms = []
    # Under sustained load the GPU's power cap lowers the SM clock within a
    # tenth of a second; each timed phase therefore starts from an idle GPU,
    # as the timed region did, and its clocks are sampled too.
    time.sleep(0.3)
    with ClockSampler(local) as k2_clocks:
        try:
            for _ in range(n_cycles):
                with torch.cuda.stream(stream):
                    cycle_k2.replay()
                stream.synchronize()
                k2_ms += [a.elapsed_time(b) for a, b in ev_pairs]
        except Exception:
            k2_ms = []
        if not k2_ms:
            # Eager launches with the same events, right after the timed region.
            k2_source = "events around the split-KV kernel, eager launches after the timed region (median)"
            for _ in range(n_cycles):
                for r in range(npool):
                    step(r, events=ev_pairs[r])
                stream.synchronize()
                k2_ms += [a.elapsed_time(b) for a, b in ev_pairs]
    k2_med_ms = sorted(k2_ms)[len(k2_ms) // 2]

    # Per layer: the plan is made once per decode step and reused by every
    # layer, so a step of a model is one plan and then one decode call (split
    # KV + combine) per layer.  One graph: a plan on the shared lengths, then
    # a decode call over each pool in turn (a pool stands for a layer's
    # cache; all pools share the lengths), timed whole and divided by the
    # calls.
    n_layers = max(8, npool)
    layer_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(layer_graph, stream=stream):
        x0p = pools[0]
        binding.mla_get_metadata(x0p.seqlens, x0p.h_q, x0p.s_q, metadata=metas[0], stream=stream)
        for layer in range(n_layers):
            x = pools[layer % npool]
            binding.mla_decode(x.q, x.kv_cache, x.block_table, x.seqlens, x.softmax_scale, x.causal, metas[0],
                               workspace=ws, out=out, lse=lse, stream=stream)
    l0 = torch.cuda.Event(enable_timing=True)
    l1 = torch.cuda.Event(enable_timing=True)
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        layer_graph.replay()
        l0.record(stream)
        n_rep = max(1, min(20, K // n_layers))
        for _ in range(n_rep):
            layer_graph.replay()
        l1.record(stream)
    stream.synchronize()
    layer_us = max_over_ranks(l0.elapsed_time(l1) * 1e3 / (n_rep * n_layers), world, dev)
    del layer_graph
    proj = projection_timing(wl, pools, metas[0], ws, out, lse, stream, dev, l2, world, local, n_layers)
    split = long_row_timing(wl, pools, stream, dev, world, local)
    # The sticky bits cover every step since warm-up (each plan rewrites the
    # word in its own metadata, so those only show the last cycle).
    err = binding.mla_take_device_errors(stream=stream)
    if err:
        raise RuntimeError(f"device error bits {err:#x} in the timed region or the kernel timing replays")

    # End to end through the API: every step copies its inputs in from pinned
    # host memory and its result (out, lse) back, as a serving loop would:
    # copies run on their own streams, double-buffered, so that step n + 1's
    # inputs go in and step n - 1's result comes out while step n computes.
    e2e_steps = min(K, 500)
    x0 = pools[0]

    def layout(tensors):
        """Byte offsets of the tensors packed back to back, each 16-byte aligned."""
        offs, n = [], 0
        for t in tensors:
            offs.append(n)
            n += (t.numel() * t.element_size() + 15) // 16 * 16
        return offs, n

    def views(buf, offs, like):
        return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for o, t in zip(offs, like)]

    # One pinned buffer per direction: q, block table and lengths go in with
    # one copy, out and lse come back with one copy (the device tensors the
    # API calls take are views into the matching device buffers).
    ins = [x0.q, x0.block_table, x0.seqlens]
    in_offs, in_bytes = layout(ins)
    h_in = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
    for v, t in zip(views(h_in, in_offs, ins), ins):
        v.copy_(t.cpu())
    res_like = [out, lse]
    res_offs, res_bytes = layout(res_like)
    h_res = [torch.empty(res_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
    d_in = [torch.empty(in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    d_res = [torch.empty(res_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    d_q, d_table, d_lens = zip(*[views(d, in_offs, ins) for d in d_in])
    d_out, d_lse = zip(*[views(d, res_offs, res_like) for d in d_res])
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    in_done = [ev(), ev()]
    comp_done = [ev(), ev()]
    out_done = [ev(), ev()]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    time.sleep(0.3)  # start from an idle GPU, as the other timed phases do
    e0.record(s_in)
    for n in range(e2e_steps):
        b = n & 1
        with torch.cuda.stream(s_in):
            if n >= 2:
                s_in.wait_event(comp_done[b])  # step n - 2 no longer reads these inputs
            d_in[b].copy_(h_in, non_blocking=True)
            in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        if n >= 2:
            stream.wait_event(out_done[b])  # step n - 2's result has left this buffer
        binding.mla_get_metadata(d_lens[b], x0.h_q, x0.s_q, metadata=metas[b], stream=stream)
        binding.mla_decode(d_q[b], x0.kv_cache, d_table[b], d_lens[b], x0.softmax_scale, x0.causal, metas[b],
                           workspace=ws, out=d_out[b], lse=d_lse[b], stream=stream)
        comp_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            h_res[b].copy_(d_res[b], non_blocking=True)
            out_done[b].record(s_out)
    s_out.wait_event(comp_done[(e2e_steps - 1) & 1])
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    err = binding.mla_take_device_errors(stream=stream)
    if err:
        raise RuntimeError(f"device error bits {err:#x} in the end-to-end steps")
    # the last step's result, as it came back, against a call on the device-resident inputs
    binding.mla_decode(x0.q, x0.kv_cache, x0.block_table, x0.seqlens, x0.softmax_scale, x0.causal, metas[0],
                       workspace=ws, out=out, lse=lse, stream=stream)
    stream.synchronize()
    last = views(h_res[(e2e_steps - 1) & 1], res_offs, res_like)
    e2e_same = bool(torch.equal(last[0], out.cpu()) and torch.equal(last[1], lse.cpu()))
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    h2d = in_bytes
    d2h = res_bytes

    nbytes, flops = algorithmic_work(lens, wl.h_q, wl.s_q, wl.causal)
    hbm_peak, tf_peak, tf_sustained, peak_kind = measured_peaks()
    k2_s = k2_med_ms * 1e-3
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
        "config": workload_config(wl, idx, lens, f"{npool} rotating pools, {total / 2**20:.0f} MiB > 3x "
                                                 f"{l2 / 2**20:.0f} MiB L2; timed via CUDA graph replay"),
        "achieved_gbs": round(world * nbytes / (ms_step * 1e-3) / 1e9, 1),
        "achieved_tflops": round(world * flops / (ms_step * 1e-3) / 1e12, 2),
        "calls_per_s_all_ranks": round(world / (ms_step * 1e-3), 1),
        "decode_kernel_us": round(k2_med_ms * 1e3, 3),
        "roofline": roofline_entry(nbytes, flops, k2_s, hbm_peak, tf_peak, peak_kind, committed_traffic(wl.name),
                                   k2_source),
        "decode_kernel_clocks": k2_clocks.summary(),
        "e2e": {"value": round(e2e_ms * 1e3 / world, 3), "unit": "us/call", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "last_result_equals_device_call": e2e_same,
                "note": ("pinned q/block_table/seqlens in (one packed copy), out/lse back (one packed copy), "
                         "every step, on copy streams of their own, double-buffered so that copies overlap the "
                         "neighbouring steps' compute; cache resident in HBM")},
        "per_layer": {"value": round(layer_us, 3), "unit": "us/call",
                      "note": (f"one plan, then {n_layers} decode calls (split-KV + combine) on it over the rotating "
                               f"pools, graph-replayed {n_rep} times; the plan's cost spread over the calls")},
        "projections": proj,
        "long_row_split": split,
        "gpu_launches": 3 * K,
        "clocks": clocks.summary(),
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(idx, budget_s=10.0)
        line["projections"]["cpu_baseline"] = oracle_projection_and_merge(wl)
    del cycle, singles
    if rank == 0:
        print(json.dumps(line), flush=True)


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
    ap.add_argument("--workload", type=int, default=1, help="index into inputs.WORKLOADS (1 = headline)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup("nccl" if args.impl == "ours" else "gloo")
    try:
        if args.impl == "reference":
            reference_arm(args, world, rank)
        else:
            ours(args, world, rank, local)
    finally:
        dist_teardown(world)


if __name__ == "__main__":
    main()
