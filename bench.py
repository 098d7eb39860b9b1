#!/usr/bin/env python
"""Benchmark of the exact-softmax-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--decode-workload NAME] [--no-e2e] [--no-cpu-baseline]

One step = one pass of the whole hot path over one batch of synthetic input:
  * prefill: attn_fwd on the named prefill workload (default gqa_causal_32k:
    B=1, Hq=32, Hkv=8, S=32768, d=128, causal), and
  * decode: attn_decode_paged (split kernel + merge kernel) on paged_decode
    (B=64, Hq=32, Hkv=8, d=128, pages of 16, lengths U[512, 8192]).
Each kernel is timed with CUDA events on the stream it is launched on; L2 is
flushed (a 256 MiB write) before each timed kernel.  The headline `value` is
prefill TFLOPS (FLOPs = 4*B*Hq*Sq*Sk*d, halved when causal) over all ranks;
`decode` reports KV GB/s (K+V bytes of the attended tokens).  Side legs time
the other prefill workloads, ragged and paged prefill (bf16 and E4M3 caches),
the FP8 prefill, the backward, the E4M3 decode, the host-buffer call
(`e2e`) and the CPU oracle's sample, each on its own.  Under torchrun every
rank runs the same per-GPU workload (weak scaling; the work units are
independent, so there is no data-path collective) and times are the max over
ranks.

--impl reference times the CPU oracle (the only reference implementation this
project has) on the host cores of rank 0, on a bounded seeded sample of the
same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attn fwd TFLOPS (prefill) and decode KV GB/s on 1 B200, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gqa_causal_32k")
    ap.add_argument("--prefill-legs",
                    default="mha_causal_2k,gqa_causal_8k,gqa_causal_8k_padded,tiny_mha",
                    help="prefill configurations timed on their own after the headline "
                         "('none' for no leg)")
    ap.add_argument("--decode-workload", default="paged_decode")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-ragged", action="store_true")
    ap.add_argument("--ragged-workload", default="ragged_gqa_causal")
    ap.add_argument("--no-decode-fp8", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--backward-workloads", default="mha_causal_2k,gqa_causal_8k")
    ap.add_argument("--no-prefill-fp8", action="store_true")
    ap.add_argument("--prefill-fp8-workload", default="gqa_causal_8k")
    ap.add_argument("--no-paged-prefill", action="store_true")
    ap.add_argument("--no-paged-prefill-fp8", action="store_true")
    ap.add_argument("--paged-prefill-workload", default="paged_prefill_gqa")
    ap.add_argument("--no-masks", action="store_true")
    ap.add_argument("--masks-workload", default="gqa_causal_8k")
    ap.add_argument("--mask-legs", default="window,blocks",
                    help="which mask legs to time: window, blocks or both")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


# Device-code sources of each kernel family: its ncu counters stay valid while
# these files are unchanged (the other kernels' sources do not affect them).
KERNEL_SOURCES = {
    "attn_prefill_sm100_kernel": ("prefill_sm100.cuh", "varlen_schedule.cuh",
                                  "sm100_primitives.cuh"),
    "attn_prefill_fp8_kernel": ("prefill_fp8_sm100.cuh", "prefill_sm100.cuh",
                                "sm100_primitives.cuh"),
    "attn_decode_split_tma_kernel": ("decode_sm100.cuh", "sm100_primitives.cuh"),
    "attn_decode_split_tma_kernel_e4m3": ("decode_sm100.cuh", "sm100_primitives.cuh"),
    "attn_bwd_dkdv_kernel": ("bwd_sm100.cuh", "sm100_primitives.cuh"),
    "attn_bwd_dq_kernel": ("bwd_sm100.cuh", "sm100_primitives.cuh"),
}


def kernel_source_sha(kernel: str = None) -> str:
    """Hash of a kernel family's CUDA sources (of every .cu/.cuh when kernel is
    None): ncu traffic figures are valid only for this hash."""
    csrc = os.path.join(ROOT, "exact_softmax_attention_fwd_b200", "csrc")
    names = (sorted(KERNEL_SOURCES[kernel]) if kernel is not None else
             sorted(n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh"))))
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str, config_name: str):
    """Per-launch DRAM bytes of a kernel from profiles/traffic.json, if current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(kernel_key, {}).get(config_name)
    if not e or e.get("source_sha") != kernel_source_sha(kernel_key):
        return None
    return float(e["dram_bytes_per_launch"])


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    def __init__(self, device, period_s: float = 0.005):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nv = nv
            self._h = None
            try:  # NVML numbering can differ from CUDA's: match the PCI bus id
                import torch
                pr = torch.cuda.get_device_properties(device)
                bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
                self._h = nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self._h = nv.nvmlDeviceGetHandleByIndex(device.index or 0)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self._nv = None
        self._names = {
            "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
            "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4, "sync_boost": 0x10,
            "gpu_idle": 0x1, "applications_clocks_setting": 0x2,
        }

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                for name, bit in self._names.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The largest x over all ranks (times are reported as the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, ms_per_rank: float, world: int,
                       device: str = "cuda"):
    """Whole-job throughput under weak scaling: every rank processes the same
    number of independent units; the job takes as long as its slowest rank.
    Returns (units of all ranks per second, slowest rank's ms)."""
    ms = max_over_ranks(ms_per_rank, world, device)
    return world * units_per_rank / (ms * 1e-3), ms


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------------- reference arm


def run_reference(args, world, rank):
    """Time the CPU oracle on a bounded sample of the prefill workload (rank 0 only)."""
    if rank != 0:
        return None
    import torch

    import oracle
    from exact_softmax_attention_fwd_b200 import workloads as W
    cfg = W.CONFIGS[args.workload]
    dcfg = None if args.no_decode else W.CONFIGS[args.decode_workload]
    q, k, v, k_lens = W.config_inputs(cfg)
    dinp = None if dcfg is None else W.decode_config_inputs(dcfg)
    n_rows = 2048  # prefill rows per step: well under a second of the host's cores
    threads = os.cpu_count() or 1
    oracle.build()
    times, flops, dtimes = [], [], []
    for step in range(args.warmup + args.steps):
        rows = W.sample_rows(cfg.B, cfg.Hq, cfg.S, n_rows, seed=5000 + step)
        f = _visible_pair_flops(cfg, rows, k_lens)
        t0 = time.perf_counter()
        oracle.attn_fwd(q, k, v, cfg.causal, cfg.scale, k_lens=k_lens, rows=rows, n_threads=threads)
        dt = time.perf_counter() - t0
        if dinp is not None:  # the whole decode batch
            t1 = time.perf_counter()
            oracle.decode_paged(dinp.q, dinp.k_cache, dinp.v_cache, dinp.block_table,
                                dinp.seq_lens, dcfg.scale, n_threads=threads)
            ddt = time.perf_counter() - t1
        if step >= args.warmup:
            times.append(dt)
            flops.append(f)
            if dinp is not None:
                dtimes.append(ddt)
    value = sum(flops) / sum(times) / 1e12
    ms = 1e3 * (sum(times) + sum(dtimes)) / len(times)
    sample = (f"{n_rows} seeded query rows of {cfg.name} per step (of {cfg.B * cfg.Hq * cfg.S})"
              + ("" if dinp is None else f" and the whole {dcfg.name} batch"))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(cfg, dcfg),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    if dinp is not None:
        nbytes = decode_algorithmic_bytes(dcfg, dinp)
        line["decode"] = {"value": nbytes * len(dtimes) / sum(dtimes) / 1e9, "unit": "GB/s",
                          "ms": 1e3 * sum(dtimes) / len(dtimes)}
    return line


# --------------------------------------------------------------------------- our arm


def config_dict(cfg, dcfg):
    d = {"workload": cfg.name, "B": cfg.B, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "Sq": cfg.S, "Sk": cfg.S,
         "d": cfg.d, "causal": cfg.causal,
         "inputs": f"bf16 N(0,1){' x ' + str(cfg.value_scale) if cfg.value_scale != 1.0 else ''} "
                   f"seeded{', key padding 0-25%' if cfg.padded else ''}",
         "l2": "flushed before every timed kernel (256 MiB write)"}
    if dcfg is not None:
        d["decode_workload"] = dcfg.name
        d["decode"] = {"B": dcfg.B, "Hq": dcfg.Hq, "Hkv": dcfg.Hkv, "d": dcfg.d,
                       "page_size": dcfg.page_size, "seq_lens": f"U[{dcfg.len_lo},{dcfg.len_hi}]"}
    return d


# The oracle's sample per prefill configuration for the CPU baseline: None =
# every row; an int = that many seeded rows (the 32k configuration: the 512
# (head, row) pairs its parity test checks, timed and extrapolated).
CPU_SAMPLE_ROWS = {"tiny_mha": None, "mha_causal_2k": None, "gqa_causal_8k": None,
                   "gqa_causal_8k_padded": None, "gqa_causal_32k": 24576}
CPU_SAMPLE_SEED = {"gqa_causal_32k": 41}


def _visible_pair_flops(cfg, rows, k_lens):
    """4*d per visible (row, key) pair over the given flat rows (None = all)."""
    import torch
    S = cfg.S
    if rows is None:
        i = torch.arange(S, dtype=torch.float64).repeat(cfg.B * cfg.Hq)
        b = torch.arange(cfg.B).repeat_interleave(cfg.Hq * S)
    else:
        i = (rows % S).double()
        b = rows // (cfg.Hq * S)
    kl = (torch.full((cfg.B,), float(S), dtype=torch.float64) if k_lens is None
          else k_lens.double())[b]
    if cfg.causal:  # bottom-right: row i sees keys j <= i + kl - S, j < kl
        vis = torch.clamp(torch.minimum(i + kl - S + 1, kl), min=0)
    else:
        vis = kl
    return float(4.0 * cfg.d * vis.sum())


def cpu_baseline_prefill(cfg, q, k, v, k_lens):
    """The oracle as it stands on this host's cores, on the configuration's
    sample: every row, or the seeded sample of CPU_SAMPLE_ROWS (then the full
    problem's time is extrapolated from the sample's share of visible pairs
    and labelled as such).  `value` counts the metric's FLOPs (the nominal
    causal formula for full runs, visible-pair FLOPs for a sample)."""
    import oracle
    from exact_softmax_attention_fwd_b200 import workloads as W
    threads = os.cpu_count() or 1
    n = CPU_SAMPLE_ROWS.get(cfg.name)
    rows = None if n is None else W.sample_rows(cfg.B, cfg.Hq, cfg.S, n,
                                                seed=CPU_SAMPLE_SEED.get(cfg.name, 78))
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, cfg.causal, cfg.scale, k_lens=k_lens, rows=rows, n_threads=threads)
    dt = time.perf_counter() - t0
    out = {"unit": "TFLOPS", "cores": threads, "kind": "oracle", "seconds": dt}
    if rows is None:
        out["value"] = cfg.flops() / dt / 1e12
        out["sample"] = f"all {cfg.B * cfg.Hq * cfg.S} query rows of {cfg.name} ({dt:.1f} s)"
    else:
        f_sample = _visible_pair_flops(cfg, rows, k_lens)
        f_all = _visible_pair_flops(cfg, None, k_lens)
        out["value"] = f_sample / dt / 1e12
        out["sample"] = (f"{rows.numel()} seeded (head, query row) pairs of {cfg.name} "
                         f"({dt:.2f} s)")
        out["extrapolated_full_problem_s"] = dt * f_all / f_sample
        out["extrapolation"] = ("EXTRAPOLATED, not measured: the sample's time scaled by "
                                "the full problem's visible pairs over the sample's")
    return out


def cpu_baseline_decode(dcfg, dinp):
    """The decode oracle on the whole paged_decode batch (GB/s of the same
    algorithmic bytes the GPU figure counts)."""
    import oracle
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle.decode_paged(dinp.q, dinp.k_cache, dinp.v_cache, dinp.block_table, dinp.seq_lens,
                        dcfg.scale, n_threads=threads)
    dt = time.perf_counter() - t0
    nbytes = decode_algorithmic_bytes(dcfg, dinp)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "seconds": dt, "sample": f"the whole {dcfg.name} batch ({dcfg.B} sequences, {dt:.2f} s)"}


def decode_algorithmic_bytes(dcfg, dinp) -> int:
    """K+V of the attended tokens, q, o, the block-table entries used, lengths, LSE."""
    from exact_softmax_attention_fwd_b200 import workloads as W
    kv = W.decode_kv_bytes(dinp.seq_lens, dcfg.Hkv, dcfg.d)
    table = int(sum(-(-int(n) // dcfg.page_size) for n in dinp.seq_lens.tolist())) * 4
    return kv + 2 * dinp.q.numel() * 2 + table + dinp.seq_lens.numel() * 4 + dcfg.B * dcfg.Hq * 4


def leg_calls(args, est_ms: float, world: int, floor_ms: float = 200.0, cap: int = 4000) -> int:
    """Calls to time in a leg: at least --steps, and enough for the region to
    last about floor_ms so that the clock sampler sees it (the estimate is
    the slowest rank's, so every rank makes the same number of calls)."""
    est = max_over_ranks(max(est_ms, 1e-3), world)
    return int(max(args.steps, min(cap, math.ceil(floor_ms / est))))


def timed_calls(args, dev, world, one, est_calls: int = 3):
    """Warm up, estimate the call time, then time n calls of `one` (L2 flushed
    before each, CUDA events on the launch stream around each) with NVML clock
    samples over the region.  Returns (per-call ms, clocks summary)."""
    import torch

    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        flush.fill_(1.0)
        one()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(est_calls):
        one()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    n = leg_calls(args, e0.elapsed_time(e1) / est_calls + 0.05, world)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    sampler = ClockSampler(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    with sampler:
        for a, b in evs:
            flush.fill_(1.0)
            a.record(stream)
            one()
            b.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    return [a.elapsed_time(b) for a, b in evs], sampler.summary()


def tensor_roofline(flops, ms, peaks, kernel, config_name, world):
    """Roofline object of a tensor-bound launch from its per-call times."""
    mean = sum(ms) / len(ms)
    med = statistics.median(ms)
    mean_all = max_over_ranks(mean, world)
    achieved = flops / (mean_all * 1e-3) / 1e12
    achieved_med = flops / (med * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
            "achieved_median": achieved_med, "frac_median": achieved_med / peaks["bf16_tflops"],
            "traffic": ncu_traffic(kernel, config_name), "kernel": kernel,
            "peak_source": f"{peaks['source']} bf16 burst (kernel timed alone)",
            "per_launch_flops": flops, "mean_ms": mean_all, "median_ms": med, "calls": len(ms)}


def prefill_leg(args, cfg, dev, world, peaks, cpu: bool):
    """One prefill configuration timed on its own (attn_fwd_masked; inputs
    resident; L2 flushed before each call), with its own clock record and, on
    rank 0 of a 1-GPU run, the oracle's time on the same inputs."""
    import torch

    from exact_softmax_attention_fwd_b200 import attn_fwd_masked, attn_get_device_error
    from exact_softmax_attention_fwd_b200 import workloads as W

    q_h, k_h, v_h, kl_h = W.config_inputs(cfg)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    kl = None if kl_h is None else kl_h.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((cfg.B, cfg.Hq, cfg.S), dtype=torch.float32, device=dev)

    def one():
        attn_fwd_masked(q, k, v, cfg.causal, cfg.scale, k_lens=kl, out=o, lse=lse)

    ms, clocks = timed_calls(args, dev, world, one)
    st, fl = attn_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word set in the {cfg.name} leg: {fl:#x}")
    flops = cfg.flops()
    rl = tensor_roofline(flops, ms, peaks, "attn_prefill_sm100_kernel", cfg.name, world)
    leg = {"workload": cfg.name, "value": world * rl["achieved"], "unit": "TFLOPS",
           "ms": rl["mean_ms"], "median_ms": rl["median_ms"], "calls": len(ms),
           "gpu_launches_per_call": 1, "config": config_dict(cfg, None), "roofline": rl,
           "clocks": clocks}
    if cfg.padded:
        leg["flops_counted"] = "nominal 4*B*Hq*S*S*d/2 (padded keys included), as the metric states"
    del q, k, v, o, lse
    if cpu:
        leg["cpu_baseline"] = cpu_baseline_prefill(cfg, q_h, k_h, v_h, kl_h)
    return leg


def run_ours(args, world, rank, local):
    import torch

    from exact_softmax_attention_fwd_b200 import (attn_decode_paged, attn_decode_workspace_size,
                                                  attn_fwd_masked, attn_get_device_error)
    from exact_softmax_attention_fwd_b200 import workloads as W

    dev = torch.device("cuda", local if world > 1 else 0)
    peaks = load_peaks()
    cfg = W.CONFIGS[args.workload]
    dcfg = None if args.no_decode else W.CONFIGS[args.decode_workload]
    cpu = rank == 0 and world == 1 and not args.no_cpu_baseline

    # ---- inputs resident in HBM before the timed region
    q_h, k_h, v_h, kl_h = W.config_inputs(cfg)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    k_lens = None if kl_h is None else kl_h.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((cfg.B, cfg.Hq, cfg.S), dtype=torch.float32, device=dev)
    flops = cfg.flops()
    if dcfg is not None:
        dinp = W.decode_config_inputs(dcfg)
        dq, dk, dv = dinp.q.to(dev), dinp.k_cache.to(dev), dinp.v_cache.to(dev)
        dtbl, dlens = dinp.block_table.to(dev), dinp.seq_lens.to(dev)
        ws = torch.empty(attn_decode_workspace_size(dcfg.B, dcfg.Hq, dcfg.max_pages_per_seq,
                                                    dcfg.page_size, dcfg.d),
                         dtype=torch.uint8, device=dev)
        do = torch.empty((dcfg.B, dcfg.Hq, dcfg.d), dtype=torch.bfloat16, device=dev)
        dlse = torch.empty((dcfg.B, dcfg.Hq), dtype=torch.float32, device=dev)
        decode_bytes = decode_algorithmic_bytes(dcfg, dinp)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def prefill():
        attn_fwd_masked(q, k, v, cfg.causal, cfg.scale, k_lens=k_lens, out=o, lse=lse)

    def decode():
        attn_decode_paged(dq, dk, dv, dtbl, dlens, dcfg.scale, out=do, lse=dlse, workspace=ws)

    def step(evs=None):
        flush.fill_(1.0)
        if evs is not None:
            evs[0].record(stream)
        prefill()
        if evs is not None:
            evs[1].record(stream)
        if dcfg is not None:
            flush.fill_(2.0)
            if evs is not None:
                evs[2].record(stream)
            decode()
            if evs is not None:
                evs[3].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    st, fl = attn_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word set during warm-up: {fl:#x}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    with sampler:
        t_all0.record(stream)
        for s in range(args.steps):
            step(evs[s])
        t_all1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    st, fl = attn_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word set in the timed region: {fl:#x}")

    pre_ms = [e[0].elapsed_time(e[1]) for e in evs]
    step_ms = max_over_ranks(t_all0.elapsed_time(t_all1) / args.steps, world)
    rl = tensor_roofline(flops, pre_ms, peaks, "attn_prefill_sm100_kernel", cfg.name, world)
    line = {
        "metric": METRIC, "value": world * rl["achieved"], "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config_dict(cfg, dcfg), "roofline": rl,
    }
    launches_per_step = 1
    if dcfg is not None:
        dec_ms = [e[2].elapsed_time(e[3]) for e in evs]
        bytes_per_s, dec_avg = weak_scaling_value(decode_bytes, sum(dec_ms) / len(dec_ms), world)
        gbs = decode_bytes / (dec_avg * 1e-3) / 1e9
        dmed = statistics.median(dec_ms)
        line["decode"] = {
            "value": bytes_per_s / 1e9, "unit": "GB/s", "ms": dec_avg, "median_ms": dmed,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "achieved_median": decode_bytes / (dmed * 1e-3) / 1e9,
                         "traffic": ncu_traffic("attn_decode_split_tma_kernel", dcfg.name),
                         "kernel": "attn_decode_split_tma_kernel + attn_decode_merge_kernel",
                         "peak_source": f"{peaks['source']} copy bandwidth",
                         "algorithmic_bytes": decode_bytes},
        }
        launches_per_step += 2
    line["gpu_launches"] = launches_per_step * args.steps
    line["clocks"] = sampler.summary()
    del q, k, v, o, lse

    # ---- the other prefill configurations, each timed on its own
    legs = {}
    for name in args.prefill_legs.split(","):
        name = name.strip()
        if name and name != "none" and name != cfg.name:
            legs[name] = prefill_leg(args, W.CONFIGS[name], dev, world, peaks, cpu)
    if legs:
        line["prefill_legs"] = legs
    if not args.no_masks:
        line["masks"] = masks_leg(args, W.CONFIGS[args.masks_workload], dev, world, peaks)
    if not args.no_prefill_fp8:
        line["prefill_fp8"] = prefill_fp8_leg(args, W.CONFIGS[args.prefill_fp8_workload], dev,
                                              world, peaks)
    if not args.no_ragged:
        line["ragged"] = ragged_leg(args, dev, world, peaks)
    if not args.no_paged_prefill:
        line["paged_prefill"] = paged_prefill_leg(args, dev, world, peaks)
    if not args.no_paged_prefill_fp8:
        line["paged_prefill_fp8"] = paged_prefill_leg(args, dev, world, peaks, fp8=True)
    if not args.no_backward:
        line["backward"] = {name.strip(): backward_leg(args, W.CONFIGS[name.strip()], dev, world,
                                                       peaks)
                            for name in args.backward_workloads.split(",") if name.strip()}
    if not args.no_decode and not args.no_decode_fp8:
        line["decode_fp8"] = decode_fp8_leg(args, dev, world, peaks)
    if not args.no_e2e:
        line["e2e"] = e2e_leg(args, cfg, q_h, k_h, v_h, kl_h, dev, world)
    if cpu:
        line["cpu_baseline"] = cpu_baseline_prefill(cfg, q_h, k_h, v_h, kl_h)
        if dcfg is not None:
            line["decode"]["cpu_baseline"] = cpu_baseline_decode(dcfg, dinp)
    return line if rank == 0 else None


# The programmable-mask legs: a sliding window and a block mask shared by the
# heads, causal, on a fixed-length configuration's inputs.
MASK_WINDOW = 1024
MASK_DENSITY = 0.25


def visible_pairs_window(S: int, window: int) -> int:
    """(query row, key) pairs a causal sliding window of `window` keys leaves
    for Sq = Sk = S: row i sees min(i + 1, window) keys."""
    w = min(window, S)
    return w * (w + 1) // 2 + (S - w) * w


def visible_pairs_blocks(mask, S: int, causal: bool) -> int:
    """Pairs a block mask uint8 [B, 1, n, n] (Sq = Sk = S, 128 x 128 blocks)
    leaves per query head, summed over the batch: each kept block contributes
    its (row, key) pairs, causal ones only below the diagonal."""
    import numpy as np

    n = -(-S // 128)
    edge = np.minimum(np.arange(n) * 128 + 128, S) - np.arange(n) * 128  # rows (keys) per tile
    full = np.outer(edge, edge)
    if causal:
        qt, kt = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        # a diagonal tile of m rows and keys holds m (m + 1) / 2 causal pairs
        diag = np.diag(edge * (edge + 1) // 2)
        full = np.where(kt < qt, full, 0) + diag
    m = np.asarray(mask, dtype=np.int64)[:, 0]
    return int((m * full[None]).sum())


def masks_leg(args, cfg, dev, world, peaks):
    """attn_fwd_window (window MASK_WINDOW) and attn_fwd_block_sparse (a mask of
    density MASK_DENSITY shared by the heads, causal) on a configuration's
    inputs, timed like the other legs; FLOPs counted over the visible (query,
    key) pairs only, 4 d per pair and query head."""
    import torch

    from exact_softmax_attention_fwd_b200 import (attn_fwd_block_sparse, attn_fwd_window,
                                                 attn_get_device_error)
    from exact_softmax_attention_fwd_b200 import workloads as W

    assert cfg.causal and not cfg.padded
    q_h, k_h, v_h, _ = W.config_inputs(cfg)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((cfg.B, cfg.Hq, cfg.S), dtype=torch.float32, device=dev)
    bm_h = W.block_mask(cfg.B, 1, cfg.S, cfg.S, MASK_DENSITY)
    bm = bm_h.to(dev)
    cases = {
        f"window_{MASK_WINDOW}": (
            lambda: attn_fwd_window(q, k, v, cfg.scale, window=MASK_WINDOW, out=o, lse=lse),
            cfg.B * visible_pairs_window(cfg.S, MASK_WINDOW),
            f"causal sliding window of {MASK_WINDOW} keys"),
        f"blocks_{MASK_DENSITY}": (
            lambda: attn_fwd_block_sparse(q, k, v, bm, True, cfg.scale, out=o, lse=lse),
            visible_pairs_blocks(bm_h, cfg.S, True),
            f"causal, 128 x 128 block mask shared by the heads, density {MASK_DENSITY} "
            f"(seed {W.SEED_BLOCK_MASK})"),
    }
    wanted = {x.strip() for x in args.mask_legs.split(",") if x.strip()}
    legs = {}
    for name, (one, pairs, what) in cases.items():
        if name.split("_")[0] not in wanted:
            continue
        ms, clocks = timed_calls(args, dev, world, one)
        st, fl = attn_get_device_error()
        if st != 0:
            raise RuntimeError(f"device error word set in the {name} leg: {fl:#x}")
        flops = 4.0 * cfg.d * cfg.Hq * pairs
        rl = tensor_roofline(flops, ms, peaks, "attn_prefill_sm100_kernel",
                             f"{cfg.name}_{name}", world)
        legs[name] = {"workload": f"{cfg.name}, {what}", "value": world * rl["achieved"],
                      "unit": "TFLOPS", "flops_counted": "visible (query, key) pairs x 4 d x Hq",
                      "visible_fraction": pairs / (cfg.B * cfg.S * (cfg.S + 1) / 2),
                      "ms": rl["mean_ms"], "median_ms": rl["median_ms"], "calls": len(ms),
                      "gpu_launches_per_call": 1, "clocks": clocks, "roofline": rl}
    del q, k, v, o, lse, bm
    return legs


def prefill_fp8_leg(args, cfg, dev, world, peaks):
    """attn_fwd_fp8 on a prefill configuration's inputs quantised to E4M3 with one
    scale per (batch, head, 128-row block), timed like the other legs.  FLOPs as
    the bf16 prefill.  Roofline: Q K^T runs on E4M3 MMAs, P V on bf16 ones, so at
    the tensor peaks the launch would take (F/2)/(2 P) + (F/2)/P = 0.75 F / P
    with P the measured bf16 peak and 2 P the E4M3 rate (the nominal 2:1
    ratio): the peak reported is P / 0.75."""
    import torch

    from exact_softmax_attention_fwd_b200 import attn_fwd_fp8, attn_get_device_error
    from exact_softmax_attention_fwd_b200 import workloads as W

    q8, k8, v8, qs, ks, vs = (t.to(dev) for t in W.fp8_prefill_inputs(
        cfg.B, cfg.Hq, cfg.Hkv, cfg.S, cfg.S, cfg.d, cfg.seed, cfg.value_scale))
    kl = None if not cfg.padded else W.key_padding(cfg.B, cfg.S).to(dev)
    o = torch.empty(q8.shape, dtype=torch.bfloat16, device=dev)
    lse = torch.empty((cfg.B, cfg.Hq, cfg.S), dtype=torch.float32, device=dev)

    def one():
        attn_fwd_fp8(q8, k8, v8, qs, ks, vs, cfg.causal, cfg.scale, k_lens=kl, out=o, lse=lse)

    ms, clocks = timed_calls(args, dev, world, one)
    st, fl = attn_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word set in the FP8 prefill leg: {fl:#x}")
    peaks_mixed = dict(peaks)
    peaks_mixed["bf16_tflops"] = peaks["bf16_tflops"] / 0.75
    rl = tensor_roofline(cfg.flops(), ms, peaks_mixed, "attn_prefill_fp8_kernel", cfg.name, world)
    rl["peak_source"] = (f"{peaks['source']} bf16 burst / 0.75 (Q K^T at twice the bf16 rate, "
                         "P V at the bf16 rate)")
    rl["frac_of_bf16_peak"] = rl["achieved"] / peaks["bf16_tflops"]
    return {"workload": cfg.name + " (E4M3 Q, K, V; one scale per 128-row block)",
            "value": world * rl["achieved"], "unit": "TFLOPS", "ms": rl["mean_ms"],
            "median_ms": rl["median_ms"], "calls": len(ms), "gpu_launches_per_call": 1,
            "clocks": clocks, "roofline": rl}


def decode_fp8_leg(args, dev, world, peaks):
    """Paged decode over the same workload with its cache quantised to E4M3
    (one scale per page and KV head): the split kernel reads half the K/V bytes.
    Algorithmic bytes: the FP8 K/V of the attended tokens and their pages'
    scales, plus q, o, lse, the block-table entries and the lengths."""
    import torch

    from exact_softmax_attention_fwd_b200 import (attn_decode_paged_fp8,
                                                  attn_decode_workspace_size,
                                                  attn_get_device_error)
    from exact_softmax_attention_fwd_b200 import workloads as W

    dcfg = W.CONFIGS[args.decode_workload]
    base = W.decode_config_inputs(dcfg)
    k8, ks = W.quantize_e4m3_per_page(base.k_cache)
    v8, vs = W.quantize_e4m3_per_page(base.v_cache)
    q, tbl, lens = base.q.to(dev), base.block_table.to(dev), base.seq_lens.to(dev)
    k8, v8, ks, vs = k8.to(dev), v8.to(dev), ks.to(dev), vs.to(dev)
    ws = torch.empty(attn_decode_workspace_size(dcfg.B, dcfg.Hq, dcfg.max_pages_per_seq,
                                                dcfg.page_size, dcfg.d),
                     dtype=torch.uint8, device=dev)
    o = torch.empty((dcfg.B, dcfg.Hq, dcfg.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((dcfg.B, dcfg.Hq), dtype=torch.float32, device=dev)

    def one():
        attn_decode_paged_fp8(q, k8, v8, ks, vs, tbl, lens, dcfg.scale, out=o, lse=lse,
                              workspace=ws)

    ms, clocks = timed_calls(args, dev, world, one)
    st, fl = attn_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word set in the FP8 decode leg: {fl:#x}")
    pages = int(sum(-(-int(n) // dcfg.page_size) for n in base.seq_lens.tolist()))
    nbytes = (W.fp8_kv_bytes(base.seq_lens, dcfg.Hkv, dcfg.d, dcfg.page_size) + 2 * q.numel() * 2
              + pages * 4 + lens.numel() * 4 + lse.numel() * 4)
    bytes_per_s, avg = weak_scaling_value(nbytes, sum(ms) / len(ms), world)
    gbs = nbytes / (avg * 1e-3) / 1e9
    tokens = int(base.seq_lens.sum())
    return {"workload": dcfg.name + " (E4M3 cache, per-page scales)", "value": bytes_per_s / 1e9,
            "unit": "GB/s", "ms": avg, "median_ms": statistics.median(ms), "calls": len(ms),
            "gpu_launches_per_call": 2, "tokens_per_s": world * tokens / (avg * 1e-3),
            "clocks": clocks,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes": nbytes,
                         "achieved_median": nbytes / (statistics.median(ms) * 1e-3) / 1e9,
                         "kernel": "attn_decode_split_tma_kernel (E4M3) + attn_decode_merge_kernel",
                         "traffic": ncu_traffic("attn_decode_split_tma_kernel_e4m3", dcfg.name)}}


def backward_leg(args, cfg, dev, world, peaks):
    """The backward pass from the saved LSE (attn_bwd: the row-statistics kernel, the
    dK/dV kernel and the dQ kernel) on a prefill workload, timed on its own: the
    forward outputs are computed once before timing, inputs resident, L2 flushed
    before each call.  FLOPs are the backward's five products (2.5x the forward's
    count, halved when causal); the two-kernel design executes seven (3.5x)."""
    import torch

    from exact_softmax_attention_fwd_b200 import (attn_bwd, attn_bwd_workspace_size,
                                                  attn_fwd_masked, attn_get_device_error)
    from exact_softmax_attention_fwd_b200 import workloads as W

    q_h, k_h, v_h, kl_h = W.config_inputs(cfg)
    do_h = W.grad_output(cfg.B, cfg.Hq, cfg.S, cfg.d, seed=cfg.seed)
    q, k, v, do = q_h.to(dev), k_h.to(dev), v_h.to(dev), do_h.to(dev)
    kl = None if kl_h is None else kl_h.to(dev)
    o, lse = attn_fwd_masked(q, k, v, cfg.causal, cfg.scale, k_lens=kl)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(attn_bwd_workspace_size(cfg.B, cfg.Hq, cfg.S), dtype=torch.uint8,
                     device=dev)

    def one():
        attn_bwd(q, k, v, o, lse, do, cfg.causal, cfg.scale, k_lens=kl, dq=dq, dk=dk, dv=dv,
                 workspace=ws)

    ms, clocks = timed_calls(args, dev, world, one)
    st, fl = attn_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word set in the backward leg: {fl:#x}")
    flops = 2.5 * cfg.flops()
    rl = tensor_roofline(flops, ms, peaks, "attn_bwd_dkdv_kernel", cfg.name, world)
    rl["kernel"] = "attn_bwd_prep_kernel + attn_bwd_dkdv_kernel + attn_bwd_dq_kernel"
    rl["traffic_kernel"] = "attn_bwd_dkdv_kernel"
    rl["executed_flops_per_call"] = 3.5 * cfg.flops()
    return {"workload": cfg.name, "value": world * rl["achieved"], "unit": "TFLOPS",
            "ms": rl["mean_ms"], "median_ms": rl["median_ms"], "calls": len(ms),
            "gpu_launches_per_call": 3,
            "flops_counted": "2.5x forward (dV, dP, dQ, dK and the recomputed S)",
            "clocks": clocks, "roofline": rl}


def paged_prefill_leg(args, dev, world, peaks, fp8: bool = False):
    """Chunked prefill over a paged cache (attn_fwd_paged: the unit-list kernel and the
    prefill kernel reading K/V page by page), timed on its own like the ragged leg.
    fp8: the same over the cache quantised to E4M3 with one scale per (page, KV head)
    (attn_fwd_paged_fp8: the referenced pages dequantised, then the bf16 kernels)."""
    import torch

    from exact_softmax_attention_fwd_b200 import (attn_fwd_paged, attn_fwd_paged_fp8,
                                                  attn_fwd_paged_fp8_workspace_size,
                                                  attn_fwd_varlen_workspace_size,
                                                  attn_get_device_error)
    from exact_softmax_attention_fwd_b200 import workloads as W

    pc = W.CONFIGS[args.paged_prefill_workload]
    q_h, cu_q_h, cache, lq, lk = W.paged_prefill_config_inputs(pc)
    q, cu_q = q_h.to(dev), cu_q_h.to(dev)
    tbl, lens = cache.block_table.to(dev), cache.seq_lens.to(dev)
    max_q = int(lq.max())
    o = torch.empty_like(q)
    lse = torch.empty((pc.Hq, q.shape[0]), dtype=torch.float32, device=dev)
    if fp8:
        k8, ks = W.quantize_e4m3_per_page(cache.k_cache)
        v8, vs = W.quantize_e4m3_per_page(cache.v_cache)
        k8, v8, ks, vs = k8.to(dev), v8.to(dev), ks.to(dev), vs.to(dev)
        ws = torch.empty(attn_fwd_paged_fp8_workspace_size(pc.B, q.shape[0], max_q, tbl.shape[1],
                                                           pc.page_size, pc.Hkv, pc.d),
                         dtype=torch.uint8, device=dev)

        def one():
            attn_fwd_paged_fp8(q, k8, v8, ks, vs, tbl, cu_q, lens, max_q, True, pc.scale, out=o,
                               lse=lse, workspace=ws)
    else:
        kc, vc = cache.k_cache.to(dev), cache.v_cache.to(dev)
        ws = torch.empty(attn_fwd_varlen_workspace_size(pc.B, q.shape[0], max_q),
                         dtype=torch.uint8, device=dev)

        def one():
            attn_fwd_paged(q, kc, vc, tbl, cu_q, lens, max_q, True, pc.scale, out=o, lse=lse,
                           workspace=ws)

    ms, clocks = timed_calls(args, dev, world, one)
    st, fl = attn_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word set in the paged-prefill leg: {fl:#x}")
    rl = tensor_roofline(pc.flops(), ms, peaks, "attn_prefill_sm100_kernel",
                         pc.name + ("_e4m3" if fp8 else ""), world)
    return {"workload": pc.name + (" (E4M3 cache, one scale per page and KV head)" if fp8 else ""),
            "value": world * rl["achieved"], "unit": "TFLOPS",
            "ms": rl["mean_ms"], "median_ms": rl["median_ms"], "calls": len(ms),
            "gpu_launches_per_call": 3 if fp8 else 2,
            "sequences": pc.B, "new_tokens": int(q.shape[0]), "page_size": pc.page_size,
            "keys": f"cached uniform {pc.cached_lo}..{pc.cached_hi} + {pc.new_tokens} new (seed {pc.seed})",
            "clocks": clocks, "roofline": rl}


def ragged_leg(args, dev, world, peaks):
    """Prefill over a packed ragged batch (attn_fwd_varlen: the unit-list kernel and
    the prefill kernel), timed on its own after the headline region: inputs resident,
    L2 flushed before each call, CUDA events around each call, max over ranks."""
    import torch

    from exact_softmax_attention_fwd_b200 import (attn_fwd_varlen,
                                                  attn_fwd_varlen_workspace_size,
                                                  attn_get_device_error)
    from exact_softmax_attention_fwd_b200 import workloads as W

    rc = W.CONFIGS[args.ragged_workload]
    q_h, k_h, v_h, cu_q_h, cu_k_h, lens = W.varlen_config_inputs(rc)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    cu_q, cu_k = cu_q_h.to(dev), cu_k_h.to(dev)
    max_q = int(lens.max())
    ws = torch.empty(attn_fwd_varlen_workspace_size(rc.B, q.shape[0], max_q), dtype=torch.uint8,
                     device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((rc.Hq, q.shape[0]), dtype=torch.float32, device=dev)
    def one():
        attn_fwd_varlen(q, k, v, cu_q, cu_k, max_q, rc.causal, rc.scale, out=o, lse=lse,
                        workspace=ws)

    ms, clocks = timed_calls(args, dev, world, one)
    st, fl = attn_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word set in the ragged leg: {fl:#x}")
    rl = tensor_roofline(rc.flops(lens), ms, peaks, "attn_prefill_sm100_kernel", rc.name, world)
    return {"workload": rc.name, "value": world * rl["achieved"], "unit": "TFLOPS",
            "ms": rl["mean_ms"], "median_ms": rl["median_ms"], "calls": len(ms),
            "gpu_launches_per_call": 2, "sequences": rc.B, "total_tokens": int(q.shape[0]),
            "lengths": f"uniform {rc.len_lo}..{rc.len_hi} (seed {rc.seed})",
            "clocks": clocks, "roofline": rl}


def e2e_leg(args, cfg, q_h, k_h, v_h, kl_h, dev, world):
    """Same metric through the public host-buffer call, attn_fwd_host: Q, K, V in
    pinned host memory, O and LSE written back to pinned host memory, every copy
    inside the timed region (the call overlaps the copies of one chunk of
    (sequence, KV head) pairs with the kernels of another)."""
    import torch

    from exact_softmax_attention_fwd_b200 import attn_fwd_host, attn_fwd_host_workspace_size
    qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    op = torch.empty_like(q_h).pin_memory()
    lp = torch.empty((cfg.B, cfg.Hq, cfg.S), dtype=torch.float32).pin_memory()
    kl = None if kl_h is None else kl_h.to(torch.int32).contiguous()
    ws = torch.empty(attn_fwd_host_workspace_size(cfg.B, cfg.Hq, cfg.Hkv, cfg.S, cfg.S, cfg.d),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def one():
        attn_fwd_host(qp, kp, vp, cfg.causal, cfg.scale, k_lens=kl, out=op, lse=lp, workspace=ws,
                      device=dev, stream=stream)

    for _ in range(3):
        one()
    torch.cuda.synchronize(dev)
    n = max(5, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    for _ in range(n):
        one()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / n, world)
    h2d = (qp.numel() + kp.numel() + vp.numel()) * 2
    d2h = op.numel() * 2 + lp.numel() * 4
    return {"value": world * cfg.flops() / (ms * 1e-3) / 1e12, "unit": "TFLOPS",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "call": "attn_fwd_host (pinned host buffers, copies overlapped with the kernels)"}


def main():
    args = parse_args()
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores; other ranks have nothing to do
        if int(os.environ.get("RANK", "0")) != 0:
            return
        line = run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), 0)
        print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup(args)
    try:
        line = run_ours(args, world, rank, local)
        if line is not None and rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
