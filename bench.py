"""Benchmark of the IndexCache hot path on B200 GPUs.

One step = one pass of the whole F/S layer stack (indexer + top-k on F
layers, index reuse on S layers, sparse MQA attention on every layer) over
one synthetic sequence of the prefill workload: L = 16384, pattern
FSSSFSSS, H_I = 64, d_I = 128, k = 2048, 16 query heads, d = 128.  Inputs
are resident in HBM when the timed region starts; the L2 is flushed
(a 512 MB write) between timed steps, outside the timed events.

Launch: ``python bench.py [--gpus N --steps K --warmup W]``; for N > 1 under
torchrun, one rank per GPU, each rank running its own independent sequence
(weak scaling, no data-path collective; NCCL carries only the barrier and
the max-over-ranks of the step time).

``--impl reference`` times the CPU oracle (the plain C reference) on the
host cores instead, on a bounded row sample of the same workload.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "indexer scored pairs/s + top-k rows/s; F/S layer-stack prefill & decode ms"
WORKLOAD = "prefill"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLOP_PER_PAIR_PER_HEAD_DIM = 2  # multiply-add


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def scored_pairs(L, k, n_f):
    """Causal pairs (t, s <= t) the F layers must score: rows t >= k (rows
    t < k keep all of 0..t without a score)."""
    per_layer = L * (L + 1) // 2 - k * (k + 1) // 2 if L > k else 0
    return per_layer * n_f


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled every 20 ms by
    NVML in a thread (read-only queries), kept only while the timed region
    runs (mark_start / mark_stop); falls back to nvidia-smi at 200 ms when
    NVML is unavailable."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.samples = []  # (sm_mhz, set of reasons)
        self.smax = None
        self.in_region = False
        self.stop_flag = False
        self.proc = None
        self.nvml = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:  # the CUDA device's own board, when torch reports its PCI bus id
            bus = torch.cuda.get_device_properties(self.dev).pci_bus_id
            h = pynvml.nvmlDeviceGetHandleByPciBusId(
                "%08x:%02x:%02x.0" % (torch.cuda.get_device_properties(self.dev).pci_domain_id,
                                      bus, torch.cuda.get_device_properties(self.dev).pci_device_id))
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.dev]) if vis and vis.split(",")[0].isdigit() else self.dev
            h = pynvml.nvmlDeviceGetHandleByIndex(idx)
        return pynvml, h

    def start(self):
        try:
            pynvml, h = self._nvml_handle()
            self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            masks = [(n, getattr(pynvml, a)) for n, a in self.REASONS]

            def run():
                while not self.stop_flag:
                    if self.in_region:
                        try:
                            mhz = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                            r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                            self.samples.append((mhz, {n for n, m in masks if r & m}))
                        except Exception:
                            pass
                    time.sleep(0.02)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            self.nvml = pynvml
            self.source = "nvml, 20 ms"
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
            self.source = "nvidia-smi, 200 ms"
        except Exception:
            self.proc = None

    def _read_smi(self):
        names = [n for n, _ in self.REASONS]
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.strip().split(",")]
            if len(parts) < 9 or not self.in_region:
                continue
            try:
                mhz, self.smax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            self.samples.append((mhz, {n for n, v in zip(names, parts[5:9])
                                       if v.lower().startswith("active")}))

    def mark_start(self):
        self.in_region = True

    def mark_stop(self):
        self.in_region = False

    def stop(self):
        self.in_region = False
        self.stop_flag = True
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.nvml is None and self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self.thread.join(timeout=2)
        sm = [m for m, _ in self.samples]
        reasons = set()
        for _, r in self.samples:
            reasons |= r
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.smax,
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


# ------------------------------------------------------------- our arm
def make_prefill_inputs(cfg, rank, device):
    """All layer tensors of one sequence; each rank draws its own sequence."""
    from cross_layer_top_b200 import synth
    cfg = rank_config(cfg, rank)
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.prefill_layer(cfg, l, device)
        lay["out"] = torch.empty((cfg.L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=device)
        layers.append(lay)
    return layers


def run_ours(args, rank, world, local_rank):
    from cross_layer_top_b200 import indexcache as ic
    from cross_layer_top_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    cfg = synth.CONFIGS[WORKLOAD]
    L, k = cfg.L, cfg.k
    n_f = cfg.pattern.count("F")
    ctx = ic.Context(local_rank)
    pat = ic.ic_create_pattern(cfg.pattern)
    layers = make_prefill_inputs(cfg, rank, dev)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    cache = torch.empty((L, k), dtype=torch.int32, device=dev)
    arr = ic.make_stack_layers(layers)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ic.ic_run_stack(ctx, pat, None, dims, cache, layer_array=arr)

    # the clock sampler starts before the warm-up; it keeps only the samples
    # taken while the timed steps run
    clocks = ClockSampler(local_rank)
    clocks.start()
    for _ in range(args.warmup):
        step()
    ctx.sync_status()
    dist_barrier(world)
    torch.cuda.synchronize()

    # ------------------------------------------------ timed region (device)
    ctx.reset_timing()
    ctx.set_timing(True)
    launches0 = ctx.launch_count()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    dist_barrier(world)
    torch.cuda.synchronize()
    clocks.mark_start()
    for i in range(args.steps):
        flush.fill_(float(i))  # L2 flush, outside the timed events
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    clocks.mark_stop()
    dist_barrier(world)
    clk = clocks.stop()
    ctx.set_timing(False)
    ctx.sync_status()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(step_ms)
    gpu_launches = ctx.launch_count() - launches0
    ktimes = {}
    for kid, name in enumerate(ic.KERNEL_NAMES):
        ms, n = ctx.get_timing(kid)
        ktimes[name] = {"ms": ms, "launches": n}
    total_ms = dist_max(total_ms, world)

    pairs_step = scored_pairs(L, k, n_f)
    value = weak_scaling_value(pairs_step, args.steps, world, total_ms)
    ms_per_step = total_ms / args.steps

    # ------------------------------------------------ roofline of the dominant kernel
    idx_k = ktimes["index_score"]
    att_k = ktimes["sparse_attn"]
    top_k = ktimes["topk"]
    roof = {}
    if idx_k["launches"]:
        avg_ms = idx_k["ms"] / idx_k["launches"]
        pairs_launch = pairs_step * args.steps / idx_k["launches"]
        tflops = 2 * cfg.H_I * cfg.d_I * pairs_launch / (avg_ms / 1e3) / 1e12
        # a 1.5 ms launch inside a 12 ms step: the burst GEMM figure applies
        peak = peaks["bf16_tflops"]
        sus = peaks.get("bf16_tflops_sustained")
        roof["index_score"] = {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak,
                               "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                               "traffic": INDEX_SCORE_PREFILL_DRAM_BYTES,
                               "peak_kind": "burst bf16 GEMM, " + peak_src,
                               "frac_of_sustained": round(tflops / sus, 4) if sus else None,
                               "avg_launch_ms": round(avg_ms, 4),
                               "flop_per_launch": 2 * cfg.H_I * cfg.d_I * pairs_launch}
    if att_k["launches"]:
        avg_ms = att_k["ms"] / att_k["launches"]
        # algorithmic bytes per launch: the min(t+1, k) gathered K and V rows
        # of each query row t, plus its Q row read and output row written
        keys = sum(min(t + 1, k) for t in range(L))
        bytes_launch = keys * 2 * cfg.d * 2 + L * 2 * cfg.Hq * cfg.d * 2
        gbs = bytes_launch / (avg_ms / 1e3) / 1e9
        # The layer's K/V (8 MB) stays in L2, so the gathered rows come from
        # L2, not HBM: the bound is the L2 random-row gather rate, measured
        # in this run by the gather probe (the same rows, no compute).  HBM
        # is reported on the DRAM bytes ncu counted (Q, idx, out).
        roof["sparse_attn"] = {"bound": "l2", "achieved": round(gbs, 1), "peak": None,
                               "unit": "GB/s", "frac": None,
                               "traffic": ATTN_PREFILL_DRAM_BYTES,
                               "peak_kind": "L2 random-row gather ceiling measured in this run "
                                            "(libindexcache_probe: the same K/V rows gathered "
                                            "with cp.async, no compute); no driver-measured L2 "
                                            "peak exists",
                               "avg_launch_ms": round(avg_ms, 4), "bytes_per_launch": bytes_launch,
                               "hbm_frac_on_dram_traffic": round(
                                   ATTN_PREFILL_DRAM_BYTES / (avg_ms / 1e3) / 1e9
                                   / peaks["hbm_gbs"], 4) if ATTN_PREFILL_DRAM_BYTES else None}
        # Every gathered K/V byte crosses shared memory twice (the cp.async
        # write, the ldmatrix read): against the SMs' nominal shared-memory
        # bandwidth of 128 B per clock at the clock sampled during the timed
        # steps, that is the floor of this staged design.
        mhz = clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0
        sms = torch.cuda.get_device_properties(stream.device).multi_processor_count
        smem_bytes = 2 * keys * 2 * cfg.d * 2
        smem_peak = sms * 128 * mhz * 1e6 / 1e9
        smem_gbs = smem_bytes / (avg_ms / 1e3) / 1e9
        roof["sparse_attn"]["smem_floor"] = {
            "bytes_per_launch": smem_bytes, "peak_gbs": round(smem_peak, 1),
            "achieved_gbs": round(smem_gbs, 1), "frac": round(smem_gbs / smem_peak, 4),
            "floor_ms": round(smem_bytes / smem_peak / 1e6, 4),
            "peak_kind": "nominal 128 B/clock/SM x %d SMs x %.0f MHz (sampled)" % (sms, mhz)}
        ceiling = measure_gather_ceiling(cache, layers[-1], L, k, stream)
        if ceiling:
            roof["sparse_attn"]["peak"] = ceiling["achieved_gbs"]
            roof["sparse_attn"]["frac"] = round(gbs / ceiling["achieved_gbs"], 4)
            extra_ceiling = ceiling
        else:
            extra_ceiling = None
    else:
        extra_ceiling = None
    if top_k["launches"]:
        # algorithmic bytes per F layer: the fp32 scores of every scored row
        # t >= k read once (4(t+1) B), and k int32 indices written for every row
        bytes_f = sum(4 * (t + 1) for t in range(k, L)) + 4 * k * L
        per_f = top_k["ms"] / (args.steps * n_f)
        gbs = bytes_f / (per_f / 1e3) / 1e9
        # The kernel is bound by instruction issue (ncu: issue active 79%):
        # the warp-instructions one launch over the scored rows executes (from
        # the capture of the current kernel), per second, against one
        # instruction per clock on each of the SM's 4 schedulers at the clock
        # sampled during the timed steps.
        mhz = clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0
        sms = torch.cuda.get_device_properties(stream.device).multi_processor_count
        issue_peak = 4 * sms * mhz * 1e6 / 1e9
        roof["topk"] = {"bound": "issue", "achieved": None, "peak": round(issue_peak, 1),
                        "unit": "G warp-instructions/s", "frac": None, "traffic": TOPK_PREFILL_DRAM_BYTES,
                        "peak_kind": "4 schedulers x %d SMs x %.0f MHz (sampled)" % (sms, mhz),
                        "ms_per_f_layer": round(per_f, 4), "bytes_per_f_layer": bytes_f,
                        "hbm": {"achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": round(gbs / peaks["hbm_gbs"], 4),
                                "peak_kind": "HBM copy, " + peak_src}}
        if TOPK_PREFILL_WARP_INSTR:
            ginst = TOPK_PREFILL_WARP_INSTR / (per_f / 1e3) / 1e9
            roof["topk"]["achieved"] = round(ginst, 1)
            roof["topk"]["frac"] = round(ginst / issue_peak, 4)
            roof["topk"]["warp_instructions_per_launch"] = TOPK_PREFILL_WARP_INSTR
    overlap = measure_overlap(ctx, layers, cfg, stream)
    # the same stack with the F layers' indexers issued ahead on a second
    # stream (the multi-layer indexer page's scheduling); not the headline:
    # it relies on each F layer's inputs being given
    ahead = {"ms_per_step": round(time_stack_ahead(ctx, pat, dims, cache, arr, max(args.steps, 5),
                                                   stream, flush), 4),
             "stack_ms_per_step": round(ms_per_step, 4),
             "what": "ic_run_stack_ahead on the same layers, L2 flushed between steps"}
    dominant = max(("index_score", "sparse_attn"), key=lambda n: ktimes[n]["ms"])
    roofline = dict(roof.get(dominant, {}))
    roofline["kernel"] = dominant

    topk_rows = (L - k) * n_f * args.steps
    extra = {
        "kernels_ms_per_step": {n: round(v["ms"] / args.steps, 4) for n, v in ktimes.items()},
        "indexer_pairs_per_s": (pairs_step * args.steps / (idx_k["ms"] / 1e3)) if idx_k["ms"] else None,
        "topk_rows_per_s": (topk_rows / (top_k["ms"] / 1e3)) if top_k["ms"] else None,
        "stack_prefill_ms": round(ms_per_step, 4),
        "step_ms": [round(x, 4) for x in step_ms],
        "roofline_all": roof,
        "l2_gather_ceiling": extra_ceiling,
        "cross_layer_overlap": overlap,
        "stack_ahead": ahead,
    }

    # ------------------------------------------------ e2e through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, ctx, pat, dims, cfg, layers, cache, world, pairs_step, stream)

    # ------------------------------------------------ decode step (extra evidence)
    del layers, arr
    torch.cuda.empty_cache()
    if not args.no_decode:
        extra["decode"] = run_decode(args, ctx, peaks, peak_src, local_rank)
    extra["fp8_indexer"] = run_fp8_indexer(args, ctx, peaks, peak_src, local_rank)
    if not args.no_extended:
        extra["long_prefill"] = run_long_prefill(args, ctx, peaks, local_rank)
        extra["decode_retention_sweep"] = run_decode_sweep(args, ctx, local_rank)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, budget_s=args.cpu_budget)

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "pairs/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "prefill stack: 1 sequence/GPU, L=16384, pattern FSSSFSSS, "
                               "H_I=64, d_I=128, k=2048, 16 query heads, 1 KV head, d=128",
                   "global_batch": world, "seq_len": L, "parallelism": "dp%d" % world,
                   "l2": "flushed between timed steps (512 MB write)"},
        "e2e": e2e,
        "gpu_launches": gpu_launches,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "clocks": clk,
        "extra": extra,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
# the prefill kernels, from one ncu capture of the current kernel each (the
# summaries under profiles/ for the L=16384 prefill attention and indexer);
# None once a kernel changes until it is captured again.
ATTN_PREFILL_DRAM_BYTES = 209.91e6 + 55.03e6
INDEX_SCORE_PREFILL_DRAM_BYTES = 249.13e6 + 487.47e6
TOPK_PREFILL_DRAM_BYTES = 532.31e6 + 107.21e6
# warp-instructions of one prefill top-k launch over the scored rows (the
# same capture: smsp__inst_executed.sum)
TOPK_PREFILL_WARP_INSTR = 291.70e6


def measure_gather_ceiling(cache, lay, L, k, stream):
    """Time the library's gather probe (the attention's K/V row gather alone,
    no compute) over the fully populated index rows t >= k of this step's
    cache: the random-row gather ceiling that bounds attention when K/V sit
    in L2.  Best of 3, after one warm-up."""
    from cross_layer_top_b200 import probe
    if L <= k:
        return None
    idx = cache[k:]
    best = None
    for ctas in (2, 3):
        probe.ic_probe_gather(lay["K"], lay["V"], idx, ctas_per_sm=ctas)
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            probe.ic_probe_gather(lay["K"], lay["V"], idx, ctas_per_sm=ctas)
            b.record(stream)
            b.synchronize()
            ms = a.elapsed_time(b)
            best = ms if best is None else min(best, ms)
    nbytes = (L - k) * k * 2 * lay["K"].shape[-1] * 2
    return {"achieved_gbs": round(nbytes / (best / 1e3) / 1e9, 1), "ms": best, "bytes": nbytes,
            "what": "cp.async gather of the same K/V rows (index rows t >= k), no compute"}


def measure_overlap(ctx, layers, cfg, stream):
    """The cross-layer overlap diagnostic between the stack's two F layers
    (0 and 4): their top-k sets recomputed, then |T_0 ∩ T_4| per row timed
    over all L rows.  The synthetic layers are independent, so the overlap
    is near that of random sets (about k / (t + 1)), not the 70-100% a
    trained model shows between neighbouring layers."""
    from cross_layer_top_b200 import indexcache as ic
    f = [l for l, c in enumerate(cfg.pattern) if c == "F"]
    if len(f) < 2:
        return None
    L, k = cfg.L, cfg.k
    idx = [torch.empty((L, k), dtype=torch.int32, device=layers[0]["Q"].device) for _ in range(2)]
    for t, l in zip(idx, f[:2]):
        ic.ic_index_fp(ctx, layers[l]["qI"], layers[l]["kI"], layers[l]["w"], k, t)
    hits = torch.empty(L, dtype=torch.int32, device=idx[0].device)
    ic.ic_index_overlap(ctx, idx[0], idx[1], hits, L)
    best = None
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ic.ic_index_overlap(ctx, idx[0], idx[1], hits, L)
        b.record(stream)
        b.synchronize()
        best = a.elapsed_time(b) if best is None else min(best, a.elapsed_time(b))
    ctx.sync_status()
    h = hits[k:].double()  # rows with a full k-set in both layers
    return {"layers": f[:2], "mean_overlap_full_rows": round(float(h.mean()) / k, 5),
            "kernel_ms": round(best, 4), "rows_per_s": L / (best / 1e3),
            "bytes_per_launch": 2 * L * k * 4}


def run_split(args, rank, world, local_rank):
    """--prefill-split: ONE prefill sequence split over the ranks by query rows
    (strong scaling).  Each rank holds its rows of every layer (the
    causal-balanced partition of ic_prefill_partition); a step is one NCCL
    all-gather per k_I / K / V tensor of the ranks' rows, then
    ic_run_stack_rows on the rank's rows.  value = the sequence's scored
    pairs per step / the max-over-ranks step time."""
    from cross_layer_top_b200 import indexcache as ic
    from cross_layer_top_b200 import sharding, synth
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = synth.CONFIGS[WORKLOAD]
    L, k = cfg.L, cfg.k
    parts = sharding.partition(L, world)
    mine = parts[rank]
    n = sum(b - a for a, b in mine)
    ctx = ic.Context(local_rank)
    pat = ic.ic_create_pattern(cfg.pattern)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    local, gathered = [], []
    for l in range(cfg.n_layers):
        full = synth.prefill_layer(cfg, l, dev)  # same seed on every rank: take my rows
        loc = {m: sharding.rows_of(t, mine) for m, t in full.items()}
        loc["out"] = torch.empty((n, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=dev)
        local.append(loc)
        del full
    cache = torch.empty((n, k), dtype=torch.int32, device=dev)

    def step():
        lays = []
        for loc in local:
            lay = dict(loc)
            for m in ("kI", "K", "V"):
                if m in loc:
                    lay[m] = sharding.allgather_rows(loc[m], parts, L)
            lays.append(lay)
        ic.ic_run_stack_rows(ctx, pat, lays, dims, mine, cache)
        return lays

    for _ in range(args.warmup):
        step()
    ctx.sync_status()
    dist_barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    launches0 = ctx.launch_count()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    dist_barrier(world)
    ms = dist_max(a.elapsed_time(b), world)
    launches = ctx.launch_count() - launches0
    pairs_step = scored_pairs(L, k, cfg.pattern.count("F"))
    line = {"metric": METRIC, "value": pairs_step * args.steps / (ms / 1e3), "unit": "pairs/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "prefill stack split by query rows: 1 sequence over %d GPUs, "
                                   "L=16384, FSSSFSSS, H_I=64, d_I=128, k=2048, 16 query heads, "
                                   "d=128; per step one all-gather per k_I/K/V tensor" % world,
                       "global_batch": 1, "seq_len": L, "parallelism": "rows%d" % world,
                       "rows_per_rank": n},
            "gpu_launches": launches}
    if rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()


PROFILE_KERNELS = ("index_score", "topk", "sparse_attn", "fp_decode", "sparse_attn_decode")


def run_profile_kernel(args, local_rank):
    """--profile-kernel NAME: a small harness for ncu captures.  It allocates
    only what one kernel of the stack needs, at the workload's size (a few
    GB at most), runs --warmup launches, then --steps launches, and exits:
      index_score         prefill indexer scores, rows [k, L) of one F layer
      topk                prefill top-k of those rows (scores made once first)
      sparse_attn         prefill attention of one layer (indices made once first)
      fp_decode           decode F layer (FP8 scan with its first-digit
                          histograms, then the cluster top-k), 32 x 65537
      sparse_attn_decode  decode attention of one layer, 32 x 65537
    Prints one JSON line with the average time per launch (CUDA events)."""
    from cross_layer_top_b200 import indexcache as ic
    from cross_layer_top_b200 import synth
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    ctx = ic.Context(local_rank)
    name = args.profile_kernel
    if name in ("index_score", "topk", "sparse_attn"):
        cfg = synth.CONFIGS[WORKLOAD]
        L, k = cfg.L, cfg.k
        lay = synth.prefill_layer(cfg, 0, dev)
        ld = (L + 63) // 64 * 64
        if name == "sparse_attn":
            idx = torch.empty((L, k), dtype=torch.int32, device=dev)
            ic.ic_index_fp(ctx, lay["qI"], lay["kI"], lay["w"], k, idx)
            out = torch.empty((L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=dev)
            for m in ("qI", "kI", "w"):
                del lay[m]
            run = lambda: ic.ic_sparse_attn(ctx, lay["Q"], lay["K"], lay["V"], idx, out)
        else:
            scores = torch.empty((L - k, ld), dtype=torch.float32, device=dev)
            score = lambda: ic.ic_index_score(ctx, lay["qI"], lay["kI"], lay["w"], k, L, scores, ld)
            if name == "index_score":
                run = score
            else:
                score()
                for m in ("qI", "kI", "w", "Q", "K", "V"):
                    del lay[m]
                idx = torch.empty((L - k, k), dtype=torch.int32, device=dev)
                run = lambda: ic.ic_topk(ctx, scores, k, idx, causal_base=k, ld=ld)
    elif name in ("fp_decode", "sparse_attn_decode"):
        cfg = synth.CONFIGS["decode"]
        B, S, k = cfg.B, cfg.S, cfg.k
        lay = synth.decode_layer(cfg, 0, dev)
        idx = torch.empty((B, k), dtype=torch.int32, device=dev)
        fp = lambda: ic.ic_index_fp_decode(ctx, lay["q"], lay["w"], lay["kI8"], lay["kI_scale"],
                                           lay["seq_len"], k, idx)
        if name == "fp_decode":
            run = fp
        else:
            fp()
            out = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=dev)
            run = lambda: ic.ic_sparse_attn(ctx, lay["Q"], lay["K"], lay["V"], idx, out,
                                            rows_per_seq=1, kv_seq_stride=S * cfg.d, kv_len=S)
    else:
        raise SystemExit("--profile-kernel: one of %s" % ", ".join(PROFILE_KERNELS))
    ctx.sync_status()
    for _ in range(args.warmup):
        run()
    ctx.sync_status()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        run()
    b.record()
    b.synchronize()
    ctx.sync_status()
    print(json.dumps({"profile_kernel": name, "launches": args.steps,
                      "ms_per_call": a.elapsed_time(b) / max(1, args.steps),
                      "gpu_mem_gb": round(torch.cuda.max_memory_allocated() / 1e9, 2)}), flush=True)
    ctx.close()


def run_e2e(args, ctx, pat, dims, cfg, layers, cache, world, pairs_step, stream):
    """Same metric through the library's host-memory entry point
    (ic_run_stack_host): every step copies all layer inputs host->device from
    pinned memory and every layer output back, the copies of one layer
    overlapping the compute of its neighbours."""
    from cross_layer_top_b200 import indexcache as ic
    host = []
    h2d = d2h = 0
    for lay in layers:
        h = {}
        for n, t in lay.items():
            if n in ("out", "idx_snapshot"):
                continue
            h[n] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            h[n].copy_(t)
            h2d += t.numel() * t.element_size()
        h["out"] = torch.empty(lay["out"].shape, dtype=lay["out"].dtype, pin_memory=True)
        d2h += lay["out"].numel() * lay["out"].element_size()
        host.append(h)
    arr = ic.make_stack_layers(host)

    def step():
        ic.ic_run_stack_host(ctx, pat, None, dims, cache, layer_array=arr)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    dist_barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = dist_max(a.elapsed_time(b), world)
    return {"value": pairs_step * args.steps * world / (ms / 1e3), "unit": "pairs/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / args.steps,
            "api": "ic_run_stack_host (pinned host inputs and outputs, copies overlapped)"}


def run_decode(args, ctx, peaks, peak_src, local_rank):
    """One decode step of the batched-decode workload (32 sequences x 65537
    candidates, 16 layers FSSS x4; --decode-config picks a 200K-context
    workload of the retention sweep instead): step ms, FP8 indexer-key scan
    GB/s and the attention gather GB/s against the HBM peak.  --decode-layers
    N keeps the first N layers (for profiling captures that must stay small)."""
    import dataclasses
    from cross_layer_top_b200 import indexcache as ic
    from cross_layer_top_b200 import synth
    cfg = synth.CONFIGS[getattr(args, "decode_config", "decode")]
    if args.decode_layers:
        cfg = dataclasses.replace(cfg, pattern=cfg.pattern[:args.decode_layers])
    dev = torch.device("cuda", local_rank)
    B, S, k = cfg.B, cfg.S, cfg.k
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.decode_layer(cfg, l, dev)
        lay["out"] = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=dev)
        layers.append(lay)
    seq_len = layers[0]["seq_len"]
    pat = ic.ic_create_pattern(cfg.pattern)
    dims = ic.stack_dims(ic.IC_DECODE, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, B=B, S_max=S,
                         seq_len=seq_len)
    cache = torch.empty((B, k), dtype=torch.int32, device=dev)
    arr = ic.make_stack_layers(layers, ic.IC_DECODE)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        ic.ic_run_stack(ctx, pat, None, dims, cache, layer_array=arr)
    ctx.sync_status()
    steps = max(args.steps, 5)
    t = _time_stack(ctx, pat, dims, cache, arr, steps, torch.cuda.current_stream(), flush,
                    ahead=True)
    kt = t.pop("kernels")
    n_f = cfg.pattern.count("F")
    scan_bytes = B * S * (cfg.d_I + 4) + B * S * 4  # e4m3 keys + scales read, fp32 scores written
    scan_ms, scan_n = kt["index_score_decode"]
    att_ms, att_n = kt["sparse_attn"]
    gather_bytes = B * k * 2 * cfg.d * 2
    res = {"workload": "decode: %d sequences x (%d cached + 1 new) tokens, %d layers %s, "
                       "FP8 e4m3 indexer keys + fp32 per-token scale, k=%d"
                       % (B, S - 1, cfg.n_layers, cfg.pattern, k),
           **t,
           "kernels_ms_per_step": {n: round(v[0] / steps, 4) for n, v in kt.items()}}
    if scan_n:
        # timed like the attention below: the F layers' scans back to back in
        # a CUDA graph (the events of the eager step add host launch gaps)
        f_layers = [lay for lay, c in zip(layers, cfg.pattern) if c == "F"]
        g_ms = _scan_graph_launch_ms(ctx, f_layers, S, steps, flush)
        gbs = scan_bytes / (g_ms / 1e3) / 1e9
        ev_ms = scan_ms / scan_n
        res["scan"] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                       "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                       "bytes_per_launch": scan_bytes, "avg_launch_ms": g_ms,
                       "timing": "%d scan launches (one per F layer) captured in a CUDA graph, "
                                 "L2 flushed before every replay" % len(f_layers),
                       "events_avg_launch_ms": ev_ms,
                       "events_frac": round(scan_bytes / (ev_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                       "peak_kind": "HBM copy, " + peak_src}
    if att_n:
        # the per-kernel events of the eager step include host launch gaps,
        # which a 15 us kernel feels: the kernel's own rate comes from the
        # layers' attention launches captured back to back in a CUDA graph
        g_ms = _attn_graph_launch_ms(ctx, layers, cache, S, cfg.d, steps, flush)
        gbs = gather_bytes / (g_ms / 1e3) / 1e9
        ev_ms = att_ms / att_n
        res["gather"] = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "bytes_per_launch": gather_bytes, "avg_launch_ms": g_ms,
                         "timing": "%d attention launches (one per layer, each layer's own K/V, "
                                   "gathered from HBM) captured in a CUDA graph, L2 flushed "
                                   "before every replay" % len(layers),
                         "events_avg_launch_ms": ev_ms,
                         "events_frac": round(gather_bytes / (ev_ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}
    del layers
    torch.cuda.empty_cache()
    return res


def _graph_launch_ms(ctx, run, n, reps, flush):
    """Average duration of one of the n launches that run() issues, without
    host gaps: run() captured once in a CUDA graph (after one eager call,
    which sets up kernel attributes and cached occupancy answers), replayed
    `reps` times with L2 flushed before each replay; CUDA events on the
    replay stream."""
    run()
    ctx.sync_status()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        run()
    stream = torch.cuda.current_stream()
    g.replay()
    tot = 0.0
    for i in range(reps):
        flush.fill_(float(i))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        b.synchronize()
        tot += a.elapsed_time(b)
    ctx.sync_status()
    del g
    return tot / reps / n


def _scan_graph_launch_ms(ctx, f_layers, S, reps, flush):
    """One decode indexer-key scan launch (ic_index_score_decode), timed over
    the F layers' scans captured back to back."""
    from cross_layer_top_b200 import indexcache as ic
    B = f_layers[0]["q"].shape[0]
    scores = torch.empty((B, (S + 63) // 64 * 64), dtype=torch.float32, device=flush.device)

    def all_scans():
        for lay in f_layers:
            ic.ic_index_score_decode(ctx, lay["q"], lay["w"], lay["kI8"], lay["kI_scale"],
                                     lay["seq_len"], scores)

    return _graph_launch_ms(ctx, all_scans, len(f_layers), reps, flush)


def _attn_graph_launch_ms(ctx, layers, cache, S, d, reps, flush):
    """One decode attention launch (ic_sparse_attn), timed over every layer's
    attention (its own Q/K/V, the current index cache) captured back to
    back."""
    from cross_layer_top_b200 import indexcache as ic

    def all_layers():
        for lay in layers:
            ic.ic_sparse_attn(ctx, lay["Q"], lay["K"], lay["V"], cache, lay["out"], rows_per_seq=1,
                              kv_seq_stride=S * d, kv_len=S)

    return _graph_launch_ms(ctx, all_layers, len(layers), reps, flush)


def _time_stack(ctx, pat, dims, cache, arr, steps, stream, flush=None, graph=True, ahead=False):
    """One step of the stack timed three ways, each over `steps`
    steps with CUDA events around the step only: "step_ms" through
    ic_run_stack, "graph_step_ms" as a replay of the stack captured with
    ic_stack_graph_create, and "events_step_ms" with the library's
    per-kernel timing events on (the per-kernel breakdown, "kernels", comes
    from that pass; its events add launch gaps to a step of many small
    kernels).  `flush`, when given, is rewritten before every step;
    graph=False skips the graph pass; ahead=True adds "ahead_step_ms",
    through ic_run_stack_ahead (F layers' indexers on a second stream), and
    with the graph pass "ahead_graph_step_ms", a replay of its graph."""
    from cross_layer_top_b200 import indexcache as ic

    def timed(run):
        tot = 0.0
        for i in range(steps):
            if flush is not None:
                flush.fill_(float(i))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            run()
            b.record(stream)
            b.synchronize()
            tot += a.elapsed_time(b)
        ctx.sync_status(stream)
        return tot / steps

    def eager():
        ic.ic_run_stack(ctx, pat, None, dims, cache, stream=stream, layer_array=arr)

    plain = timed(eager)
    res = {"step_ms": plain}
    if ahead:
        res["ahead_step_ms"] = time_stack_ahead(ctx, pat, dims, cache, arr, steps, stream, flush)
        if graph:
            cache2 = torch.empty_like(cache)
            g = ic.ic_stack_graph_create_ahead(ctx, pat, None, dims, cache, cache2,
                                               layer_array=arr)
            for _ in range(2):
                g.launch(stream)
            res["ahead_graph_step_ms"] = timed(lambda: g.launch(stream))
            g.close()
            del cache2
    if graph:
        g = ic.ic_stack_graph_create(ctx, pat, None, dims, cache, layer_array=arr)
        for _ in range(2):
            g.launch(stream)
        res["graph_step_ms"] = timed(lambda: g.launch(stream))
        res["kernels_per_step"] = g.kernels()
        g.close()
    ctx.reset_timing()
    ctx.set_timing(True)
    with_events = timed(eager)
    ctx.set_timing(False)
    res["events_step_ms"] = with_events
    res["kernels"] = {n: ctx.get_timing(i) for i, n in enumerate(ic.KERNEL_NAMES)}
    return res


def time_stack_ahead(ctx, pat, dims, cache, arr, steps, stream, flush=None):
    """ms per step of ic_run_stack_ahead on the same layers (a second index
    buffer beside `cache`), after two untimed steps; CUDA events on the
    caller's stream, whose completion covers the side stream's work."""
    from cross_layer_top_b200 import indexcache as ic
    cache2 = torch.empty_like(cache)

    def run():
        ic.ic_run_stack_ahead(ctx, pat, None, dims, cache, cache2, stream=stream, layer_array=arr)

    for _ in range(2):
        run()
    ctx.sync_status(stream)
    tot = 0.0
    for i in range(steps):
        if flush is not None:
            flush.fill_(float(i))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        run()
        b.record(stream)
        b.synchronize()
        tot += a.elapsed_time(b)
    ctx.sync_status(stream)
    del cache2
    return tot / steps


def run_long_prefill(args, ctx, peaks, local_rank):
    """The long-prefill workload (L = 131072, FSSS), and the same layers
    with an all-F pattern: stack ms and the indexer's share of the all-F
    stack (indexer score + top-k time over stack time)."""
    from cross_layer_top_b200 import indexcache as ic
    from cross_layer_top_b200 import synth
    cfg = synth.CONFIGS["long_prefill_allF"]
    dev = torch.device("cuda", local_rank)
    L, k = cfg.L, cfg.k
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.prefill_layer(cfg, l, dev, indexer=True)
        lay["out"] = torch.empty((L, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=dev)
        layers.append(lay)
    dims = ic.stack_dims(ic.IC_PREFILL, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, L=L)
    cache = torch.empty((L, k), dtype=torch.int32, device=dev)
    arr = ic.make_stack_layers(layers)
    stream = torch.cuda.current_stream()
    res = {"workload": "long prefill: 1 sequence, L=131072, 4 layers, H_I=64, d_I=128, k=2048, "
                       "16 query heads, d=128"}
    for pattern in ("FSSS", "FFFF"):
        pat = ic.ic_create_pattern(pattern)
        ic.ic_run_stack(ctx, pat, None, dims, cache, layer_array=arr)  # warm-up
        t = _time_stack(ctx, pat, dims, cache, arr, 2, stream, graph=False)
        ms = t["step_ms"]
        kt = {n: v[0] / 2 for n, v in t["kernels"].items()}
        pairs = scored_pairs(L, k, pattern.count("F"))
        ent = {"stack_ms": ms, "kernels_ms": {n: round(v, 3) for n, v in kt.items()},
               "scored_pairs_per_s": pairs / (ms / 1e3)}
        if kt["index_score"]:
            tf = 2 * cfg.H_I * cfg.d_I * pairs / (kt["index_score"] / 1e3) / 1e12
            ent["indexer_tflops"] = round(tf, 1)
            # steps of 0.17-0.58 s: the sustained GEMM figure applies; burst beside it
            ent["indexer_frac_of_sustained_bf16"] = round(
                tf / peaks.get("bf16_tflops_sustained", 1400.0), 4)
            ent["indexer_frac_of_burst_bf16"] = round(tf / peaks["bf16_tflops"], 4)
        ent["indexer_share"] = round((kt["index_score"] + kt["topk"]) / ms, 4)
        res[pattern] = ent
    res["speedup_FSSS_vs_FFFF"] = res["FFFF"]["stack_ms"] / res["FSSS"]["stack_ms"]
    del layers, arr, cache
    torch.cuda.empty_cache()
    return res


def run_fp8_indexer(args, ctx, peaks, peak_src, local_rank):
    """The FP8 prefill indexer (e4m3 q_I / k_I, per-(token, head) and
    per-token scales) on the prefill workload's F layer: one F layer (scores
    + top-k) per step, 3 warm-up and 10 timed; the score kernel's roofline
    against the fp8 tensor peak (the measured bf16 peak x 2, the nominal
    fp8 / bf16 ratio)."""
    from cross_layer_top_b200 import indexcache as ic
    from cross_layer_top_b200 import synth
    cfg = synth.CONFIGS["prefill"]
    dev = torch.device("cuda", local_rank)
    lay = synth.prefill_indexer_fp8(cfg, 0, dev)
    L, k = cfg.L, cfg.k
    idx = torch.empty((L, k), dtype=torch.int32, device=dev)
    run = lambda: ic.ic_index_fp_fp8(ctx, lay["qI8"], lay["q_scale"], lay["kI8"], lay["k_scale"],
                                     lay["w"], k, idx)
    for _ in range(3):
        run()
    ctx.sync_status()
    ctx.reset_timing()
    ctx.set_timing(True)
    n = 10
    for _ in range(n):
        run()
    torch.cuda.synchronize()
    ctx.set_timing(False)
    ctx.sync_status()
    ms, launches = ctx.get_timing(ic.IC_K_INDEX_SCORE)
    tms, _ = ctx.get_timing(ic.IC_K_TOPK)
    pairs = sum(t + 1 for t in range(k, L))  # rows t >= k are scored
    flop = 2 * cfg.H_I * cfg.d_I * pairs
    avg = ms / launches
    tflops = flop / (avg / 1e3) / 1e12
    # 1.2 ms launches timed apart: the burst figure, x2 for e4m3 (nominal ratio)
    peak = 2 * peaks["bf16_tflops"]
    del lay, idx
    torch.cuda.empty_cache()
    return {"workload": "prefill F layer, FP8 indexer inputs: L=16384, H_I=64, d_I=128, k=2048",
            "score_ms": round(avg, 4), "topk_ms": round(tms / n, 4),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": round(peak, 1),
                         "unit": "TFLOP/s", "frac": round(tflops / peak, 4), "traffic": None,
                         "peak_kind": "2 x burst bf16 GEMM (nominal fp8/bf16 ratio), " + peak_src},
            "flop_per_launch": flop}


def run_decode_sweep(args, ctx, local_rank):
    """200K-context decode: 8 sequences x 200001 candidates, 47 layers, one
    decode step at uniform retention 1/1, 1/2, 1/4, 1/8 and with the searched
    patterns at 1/2, 1/4, 1/8 (the same layer tensors; S layers ignore their
    indexer inputs)."""
    from cross_layer_top_b200 import indexcache as ic
    from cross_layer_top_b200 import synth
    cfg = synth.CONFIGS["decode_sweep_r1"]
    dev = torch.device("cuda", local_rank)
    B, S, k = cfg.B, cfg.S, cfg.k
    layers = []
    for l in range(cfg.n_layers):
        lay = synth.decode_layer(cfg, l, dev, indexer=True)
        lay["out"] = torch.empty((B, cfg.Hq, cfg.d), dtype=torch.bfloat16, device=dev)
        layers.append(lay)
    seq_len = layers[0]["seq_len"]
    dims = ic.stack_dims(ic.IC_DECODE, cfg.H_I, cfg.d_I, k, cfg.Hq, cfg.d, B=B, S_max=S,
                         seq_len=seq_len)
    cache = torch.empty((B, k), dtype=torch.int32, device=dev)
    arr = ic.make_stack_layers(layers, ic.IC_DECODE)
    stream = torch.cuda.current_stream()
    res = {"workload": "decode: 8 sequences x (200000 cached + 1 new) tokens, 47 layers, "
                       "FP8 indexer keys, k=2048"}
    for r in (1, 2, 4, 8):
        pat = ic.ic_pattern_uniform(cfg.n_layers, r)
        for _ in range(2):
            ic.ic_run_stack(ctx, pat, None, dims, cache, layer_array=arr)
        t = _time_stack(ctx, pat, dims, cache, arr, 5, stream, ahead=True)
        kt = t.pop("kernels")
        res["r%d" % r] = {"pattern_F_layers": str(pat).count("F"), **t,
                          "tokens_per_s": B / (t["step_ms"] / 1e3),
                          "tokens_per_s_graph": B / (t["graph_step_ms"] / 1e3),
                          "kernels_ms": {n: round(v[0] / 5, 4) for n, v in kt.items()}}
    # the searched patterns of the 47-layer model (same layer tensors)
    for ret, c in synth.SEARCHED_PATTERNS_47.items():
        pat = ic.ic_create_pattern(c)
        for _ in range(2):
            ic.ic_run_stack(ctx, pat, None, dims, cache, layer_array=arr)
        t = _time_stack(ctx, pat, dims, cache, arr, 5, stream, ahead=True)
        kt = t.pop("kernels")
        res["searched_" + ret.replace("/", "_")] = {
            "pattern_F_layers": c.count("F"), **t, "tokens_per_s": B / (t["step_ms"] / 1e3),
            "tokens_per_s_graph": B / (t["graph_step_ms"] / 1e3),
            "kernels_ms": {n: round(v[0] / 5, 4) for n, v in kt.items()}}
    res["speedup_r4_vs_r1"] = res["r1"]["step_ms"] / res["r4"]["step_ms"]
    res["speedup_r4_vs_r1_graph"] = res["r1"]["graph_step_ms"] / res["r4"]["graph_step_ms"]
    del layers, arr, cache
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------- the oracle on CPU
def cpu_baseline(cfg, budget_s=15.0, rows_idx=None, rows_att=None):
    """Time the CPU oracle on a bounded row sample of the prefill stack and
    scale to the stack's scored pairs/s.  The indexer cost of row t is
    proportional to t+1, attention cost is per row."""
    import oracle
    from cross_layer_top_b200 import synth
    L, k = cfg.L, cfg.k
    n_f, n_l = cfg.pattern.count("F"), cfg.n_layers
    lay = synth.prefill_layer(cfg, 0, "cpu")
    q = synth.bf16_to_f32_numpy(lay["qI"])
    kk = synth.bf16_to_f32_numpy(lay["kI"])
    w = synth.bf16_to_f32_numpy(lay["w"])
    Q = synth.bf16_to_f32_numpy(lay["Q"])
    K = synth.bf16_to_f32_numpy(lay["K"])
    V = synth.bf16_to_f32_numpy(lay["V"])
    rng = np.random.default_rng(0)
    threads = os.cpu_count()
    # indexer: grow the sample until about half the budget is spent
    n_rows = rows_idx or 8
    while True:
        rows = np.sort(rng.integers(k, L, n_rows)).astype(np.int32)
        t0 = time.perf_counter()
        idx = oracle.index_topk(q, kk, w, k, rows)
        dt_idx = time.perf_counter() - t0
        if rows_idx or dt_idx > budget_s / 4 or n_rows >= 4096:
            break
        n_rows *= 4
    pairs_sampled = int(np.sum(rows.astype(np.int64) + 1))
    sec_per_pair = dt_idx / pairs_sampled
    n_att = rows_att or 64
    while True:
        arows = rng.integers(0, L, n_att).astype(np.int32)
        t0 = time.perf_counter()
        oracle.sparse_attn(Q, K, V, np.tile(idx[:1], (n_att, 1)), rows=arows)
        dt_att = time.perf_counter() - t0
        if rows_att or dt_att > budget_s / 4 or n_att >= 65536:
            break
        n_att *= 4
    sec_per_att_row = dt_att / n_att
    pairs = scored_pairs(L, k, n_f)
    est_step_s = pairs * sec_per_pair + n_l * L * sec_per_att_row
    return {"value": pairs / est_step_s, "unit": "pairs/s", "cores": threads, "kind": "oracle",
            "sample": "%d indexer rows (t in [k, L), %d scored pairs) + %d attention rows of the "
                      "prefill workload; stack time extrapolated by pairs and rows"
                      % (n_rows, pairs_sampled, n_att),
            "est_step_s": est_step_s, "measured_s": dt_idx + dt_att}


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle (plain C, fp64, OpenMP over rows)."""
    if rank != 0:
        return
    from cross_layer_top_b200 import synth
    cfg = synth.CONFIGS[WORKLOAD]
    budget = min(16.0, max(4.0, 150.0 / max(1, args.steps + args.warmup)))
    vals, measured = [], []
    cb = None
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(cfg, budget_s=budget)
        if i >= args.warmup:
            vals.append(cb["value"])
            measured.append(cb["measured_s"])
    value = statistics.median(vals) if vals else cb["value"]
    step_ms = scored_pairs(cfg.L, cfg.k, cfg.pattern.count("F")) / value * 1e3
    measured_s = sum(c for c in measured)
    line = {"metric": METRIC, "value": value, "unit": "pairs/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": "prefill stack: 1 sequence, L=16384, pattern FSSSFSSS, H_I=64, "
                                   "d_I=128, k=2048, 16 query heads, 1 KV head, d=128",
                       "global_batch": 1, "seq_len": cfg.L, "parallelism": "host cores"},
            "extrapolated": True,
            "timing": "each of the %d timed steps runs a bounded row sample of the stack on the "
                      "host cores (%.1f s measured in all); ms_per_step is the whole stack's "
                      "time extrapolated from those samples by scored pairs and rows, not a "
                      "timed full step" % (args.steps, measured_s),
            "measured_s": round(measured_s, 2),
            "cpu_baseline": {"value": value, "unit": "pairs/s", "kind": "oracle",
                             "cores": cb["cores"], "sample": cb["sample"]},
            "e2e": {"value": value, "unit": "pairs/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ distributed
def dist_barrier(world):
    if world > 1:
        torch.distributed.barrier()


def dist_max(x, world, device="cuda"):
    """Max over ranks (plumbing only: the step time and nothing else)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_config(cfg, rank):
    """Weak scaling: every rank runs its own independent sequence of the same
    shape (a different seed), with no data-path exchange."""
    import dataclasses
    return dataclasses.replace(cfg, seed=cfg.seed + 7919 * rank)


def weak_scaling_value(units_per_step_per_rank, steps, world, max_rank_ms):
    """Whole-job throughput: units processed by all ranks / max rank time."""
    return units_per_step_per_rank * steps * world / (max_rank_ms / 1e3)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=16.0)
    ap.add_argument("--no-extended", action="store_true",
                    help="skip the long-prefill and 200K-decode retention-sweep timings")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode workload (not the contract line)")
    ap.add_argument("--decode-layers", type=int, default=0)
    ap.add_argument("--decode-config", default="decode",
                    choices=["decode", "decode_sweep_r1", "decode_sweep_r2", "decode_sweep_r4",
                             "decode_sweep_r8"],
                    help="the decode workload of --decode-only")
    ap.add_argument("--profile-kernel", default=None, choices=PROFILE_KERNELS,
                    help="harness for ncu captures: only this kernel's inputs, then exit")
    ap.add_argument("--prefill-split", action="store_true",
                    help="one prefill sequence split over the ranks by query rows (strong "
                         "scaling, an all-gather of k_I/K/V per step) instead of one sequence "
                         "per rank")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours" and not args.profile_kernel:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.profile_kernel:
        run_profile_kernel(args, local_rank)
        return
    if args.decode_only:
        torch.cuda.set_device(local_rank)
        from cross_layer_top_b200 import indexcache as ic
        ctx = ic.Context(local_rank)
        peaks, peak_src = load_peaks()
        res = run_decode(args, ctx, peaks, peak_src, local_rank)
        if rank == 0:
            print(json.dumps({"decode_only": True, "decode": res}), flush=True)
        ctx.close()
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.prefill_split:
            run_split(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
