#!/usr/bin/env python
"""Benchmark of the GQA hot path on B200: prefill TFLOP/s and decode KV-cache GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...      (one process per GPU)

One step is one pass of the whole hot path: a causal prefill over the largest single-GPU prefill
workload, Qwen2-7B-shaped long context (B=1, L=32768, 28/4 heads, d=128), followed by one decode step
over the Qwen2-7B-shaped decode workload (B=64 sequences, cache lengths uniform in [1, 32768]).  The
headline `value` is the prefill's causal-effective TFLOP/s (4*B*h_q*d*L(L+1)/2 per step, summed over
ranks, divided by the slowest rank's device time); the decode step is reported beside it in GB/s of KV
cache.  The other prefill workloads (Qwen2-0.5B L=128, Qwen2-7B L=4096, Qwen2-72B B=4 L=8192) are timed
the same way before the headline and reported under `configs`, each with its step and kernel times, its
roofline fraction and a CPU-oracle sample.  Inputs are synthetic (seeded N(0,1) bf16, drawn on the
device) and resident in HBM when the timed region starts; the L2 is flushed (a 256 MiB write) before
every prefill, and the decode cache (~2.1 GB) is far larger than L2.  Each rank of an N-GPU run
processes its own copy of the workload (independent batches, no collective on the data path: weak
scaling).

`--impl reference` times the plain fp64 CPU oracle (the only reference that exists for this method) on a
bounded sample of the same prefill workload, on the host cores of rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import gqa_inputs as gi  # noqa: E402

METRIC = "GQA prefill TFLOP/s & decode KV GB/s, as % of B200 tensor/HBM peak"
PREFILL_WORKLOAD = "qwen2-7b-prefill-L32768"   # the largest prefill workload that fits one GPU
# The other prefill workloads, each timed before the headline and reported under `configs`.
CONFIG_WORKLOADS = ("qwen2-0.5b-prefill-L128", "qwen2-7b-prefill-L4096", "qwen2-72b-prefill-B4-L8192")
DECODE_WORKLOAD = "qwen2-7b-decode-B64"
FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_BF16_TFLOPS = 2250.0   # dense bf16 of one B200, data sheet (context only)


# ------------------------------------------------------------------------------------------ helpers
def prefill_flops(w) -> float:
    return 4.0 * w.B * w.h_q * w.d * w.L * (w.L + 1) / 2.0


def decode_kv_bytes(total_rows: int, w) -> float:
    return float(total_rows) * w.h_kv * w.d * 2 * 2


def decode_bytes(total_rows: int, w) -> float:
    return decode_kv_bytes(total_rows, w) + 2.0 * w.B * w.h_q * w.d * 2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "attn_kernel": ["prefill_sm100.cuh", "sm100_ptx.cuh", "rope.cuh"],
    "qkv_kernel": ["qkv_sm100.cuh", "sm100_ptx.cuh", "rope.cuh"],
    "proj_kernel": ["qkv_sm100.cuh", "sm100_ptx.cuh"],
    "split_kernel": ["decode_sm100.cuh", "sm100_ptx.cuh", "rope.cuh"],
}


def source_sha(kernel: str) -> str:
    """Hash of the sources a kernel is built from; a profile's DRAM traffic counts only while it matches."""
    h = hashlib.sha256()
    for fn in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "grouped_query_attention_gqa_b200", "csrc", fn), "rb") as f:
            h.update(fn.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def profile_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summaries, if still current."""
    sha = source_sha(kernel)
    key = f"{kernel}_{workload}"
    for fn in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        txt = open(fn, encoding="utf-8").read()
        m_sha = re.search(r"source_sha256_16\[" + kernel + r"\]:\s*([0-9a-f]{16})", txt)
        m_tr = re.search(r"traffic_bytes_per_launch\[" + re.escape(key) + r"\]:\s*([0-9.eE+]+)", txt)
        if m_sha and m_tr and m_sha.group(1) == sha:
            return float(m_tr.group(1))
    return None


class ClockSampler:
    """Polls NVML for SM clock and clock-event reasons on a background thread."""

    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
             0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
             0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report that instead of clocks
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        rs = [n for bit, n in self.NAMES.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples), "reasons": rs}


def clean(x):
    """NaN/inf (a leg that did not run) -> None, so the line stays strict JSON."""
    if isinstance(x, dict):
        return {k: clean(v) for k, v in x.items()}
    if isinstance(x, (list, tuple)):
        return [clean(v) for v in x]
    if isinstance(x, float) and (x != x or x in (float("inf"), float("-inf"))):
        return None
    return x


# ------------------------------------------------------------------------------------------ ranks
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def dist_init(world: int, backend: str = "nccl"):
    if world > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def reduce_max(x: float, device) -> float:
    """Max of a scalar over all ranks (identity when not distributed)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, seconds_this_rank: float, device) -> float:
    """Units processed by all ranks per second of the slowest rank (weak scaling: same work per rank)."""
    world = torch.distributed.get_world_size() if torch.distributed.is_initialized() else 1
    return world * units_per_rank / reduce_max(seconds_this_rank, device)


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


# ------------------------------------------------------------------------------------------ CPU oracle
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


ORACLE_ROW_BLOCK = 1024   # query rows per CPU-oracle sample (bounds one sample to about a second at L=32768)


def oracle_prefill_sample(w, budget_s: float, max_steps: int | None = None):
    """Time the fp64 oracle on samples of the prefill workload: one query head of batch row 0 and a block
    of up to ORACLE_ROW_BLOCK query rows against all keys before them, the heaviest (last) block first,
    then the next head, and so on.  Returns the causal-effective FLOP of each sample and its seconds."""
    from oracle import gqa_ref as R
    q, k, v = gi.prefill_inputs(w)
    blocks = [(r0, min(w.L, r0 + ORACLE_ROW_BLOCK)) for r0 in range(0, w.L, ORACLE_ROW_BLOCK)][::-1]
    flops, times, t0, i = [], [], time.perf_counter(), 0
    while True:
        t = (i // len(blocks)) % w.h_q
        r0, r1 = blocks[i % len(blocks)]
        rows = list(range(r0, r1))
        a = time.perf_counter()
        R.prefill_rows_ref(q, k, v, w.theta, 0, t, rows)
        times.append(time.perf_counter() - a)
        flops.append(4.0 * w.d * sum(r + 1 for r in rows))   # each row r sees keys 0..r
        i += 1
        if max_steps is not None and len(times) >= max_steps:
            break
        if max_steps is None and time.perf_counter() - t0 >= budget_s:
            break
    return flops, times


def cpu_baseline(w, budget_s: float = 12.0) -> dict:
    flops, times = oracle_prefill_sample(w, budget_s=budget_s)
    return {"value": sum(flops) / sum(times) / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"fp64 NumPy oracle, {len(times)} samples of one query head x up to {ORACLE_ROW_BLOCK} query "
                      f"rows (b=0, L={w.L}, d={w.d}, heaviest rows first) of the {w.name} workload, "
                      f"{sum(times):.1f} s of host time"}


def bench_config(wp, wd):
    return {"workload": wp.desc, "B": wp.B, "L": wp.L, "h_q": wp.h_q, "h_kv": wp.h_kv, "d": wp.d,
            "theta": wp.theta, "causal": True, "per_rank": "independent copy of the workload",
            "l2": "flushed before every prefill (256 MiB write); decode cache 2.1 GB > L2",
            "decode_workload": wd.desc}


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    w = gi.BY_NAME[args.prefill_workload]
    flops, times = oracle_prefill_sample(w, 0.0, max_steps=args.warmup + args.steps)
    timed = times[args.warmup:]
    value = sum(flops[args.warmup:]) / sum(timed) / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * sum(timed) / len(timed), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(bench_config(w, gi.BY_NAME[DECODE_WORKLOAD]),
                           step=f"one query head of batch row 0 x up to {ORACLE_ROW_BLOCK} query rows through "
                                "the fp64 oracle on the host"),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{len(timed)} samples of one query head x up to {ORACLE_ROW_BLOCK} "
                                       f"query rows of {w.name}"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------ GPU arm
def ev():
    e = torch.cuda.Event(enable_timing=True)
    e.record()   # creates the CUDA event so its handle can be handed to the library
    return e


def measure_prefill(G, w, K: int, W: int, flush, dev):
    """Time gqa_prefill on workload w: W warm-up steps, then K headline steps (no per-kernel events, so
    the attention kernel stays a programmatic dependent of the rotation pass) interleaved with K steps
    that record events around the attention kernel alone; the L2 is flushed before every step.
    Returns (mean step ms, max over ranks; mean attention-kernel ms on this rank; wall seconds of the loop)."""
    q, k, v = gi.prefill_inputs(w, device=str(dev))
    out = torch.empty_like(q)

    def step(e, inner):
        flush.zero_()
        e[0].record()
        if inner:
            G.set_timing_events(e[1], e[2])
        G.prefill(q, k, v, theta=w.theta, out=out)
        if inner:
            G.set_timing_events(None, None)
        e[3].record()

    for _ in range(W):
        step([ev() for _ in range(4)], False)
    evs = [[ev() for _ in range(4)] for _ in range(K)]
    kevs = [[ev() for _ in range(4)] for _ in range(K)]
    torch.cuda.synchronize()
    barrier()
    t0 = time.perf_counter()
    for i in range(K):
        step(evs[i], False)
        step(kevs[i], True)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    barrier()
    if G.last_error() != 0:
        raise RuntimeError(f"device error while timing {w.name}")
    step_ms = reduce_max(sum(e[0].elapsed_time(e[3]) for e in evs) / K, dev)
    attn_ms = sum(e[1].elapsed_time(e[2]) for e in kevs) / K
    del q, k, v, out
    return step_ms, attn_ms, wall


LONG_RUN_S = 0.1   # a timed loop this long under the power cap counts as "a kernel timed inside a long step"


def tensor_peak(peaks, clocks, wall_s):
    """The bf16 peak a tensor-bound kernel is measured against: the measured burst figure for a kernel timed
    alone, the measured sustained figure (cuBLAS back to back for seconds, under the 1 kW power cap) for a
    kernel timed inside a long run whose clock record shows the power cap active."""
    capped = isinstance(clocks, dict) and "sw_power_cap" in (clocks.get("reasons") or [])
    if capped and wall_s == wall_s and wall_s >= LONG_RUN_S:
        return peaks["bf16_tflops_sustained"], "sustained"
    return peaks["bf16_tflops"], "burst"


def config_entry(w, *, world, step_ms, attn_ms, peaks, peak_src, cpu_base, clocks=None, wall_s=float("nan")):
    """The `configs` entry of one prefill workload from its measured step and kernel times (ms)."""
    fl = prefill_flops(w)
    step_t = fl / (step_ms * 1e-3) / 1e12
    ach = fl / (attn_ms * 1e-3) / 1e12
    peak, kind = tensor_peak(peaks, clocks, wall_s)
    return {"workload": w.desc, "B": w.B, "L": w.L, "h_q": w.h_q, "h_kv": w.h_kv, "d": w.d,
            "value": world * step_t, "unit": "TFLOP/s", "ms_per_step": step_ms,
            "step_frac": step_t / peaks["bf16_tflops"],
            "kernel_ms_per_launch": attn_ms,
            "roofline": {"kernel": "attn_kernel (prefill)", "bound": "tensor", "achieved": ach,
                         "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                         "peak_source": f"{peak_src} bf16 dense ({kind})",
                         "frac_of_burst": ach / peaks["bf16_tflops"],
                         "frac_of_sustained": ach / peaks["bf16_tflops_sustained"],
                         "traffic": profile_traffic("attn_kernel", w.name),
                         "algorithmic_flops_per_launch": fl, "ms_per_launch": attn_ms},
            "cpu_baseline": cpu_base, "clocks": clocks, "wall_s_timed_region": wall_s}


def build_line(*, world, K, W, only, do_p, do_d, wp, wd, value_tflops, pre_mean, attn_mean, dec_mean, split_mean,
               total_rows, page, peaks, peak_src, cpu_base, e2e_pre, e2e_dec, pre_io, dec_io, qkv_line, clocks,
               t_wall, configs=None, dec_alone=(float("nan"), float("nan")), dec_rot=(float("nan"), float("nan")),
               k_cache="raw"):
    """The JSON line of the `ours` arm from the measured numbers (no device work, so the CPU tests cover it).
    Times in ms; pre_io / dec_io = (host->device, device->host) bytes of one end-to-end prefill / decode
    step; a leg that did not run carries NaN, which clean() turns into null."""
    fl = prefill_flops(wp)
    kvb = decode_kv_bytes(total_rows, wd)
    allb = decode_bytes(total_rows, wd)
    # --only decode: attn_mean is NaN, and the prefill roofline below is dropped from the line
    achieved_t = fl / (attn_mean * 1e-3) / 1e12
    peak_t, peak_kind = tensor_peak(peaks, clocks, t_wall)
    achieved_b = allb / (split_mean * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": value_tflops,
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": pre_mean,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) bf16 Q/K/V and caches drawn on the device; decode lengths U[1,32768]",
        "config": dict(bench_config(wp, wd),
                       timing=f"{K} headline steps without per-kernel events, interleaved with {K} steps "
                              "with CUDA events around the attention / split kernels for the roofline"),
        "roofline": {"kernel": "attn_kernel (prefill)", "bound": "tensor", "achieved": achieved_t,
                     "peak": peak_t, "unit": "TFLOP/s", "frac": achieved_t / peak_t,
                     "peak_source": f"{peak_src} bf16 dense ({peak_kind}: "
                                    + ("timed inside a long run with the power cap active)" if peak_kind == "sustained"
                                       else "no long power-capped run)"),
                     "traffic": profile_traffic("attn_kernel", wp.name),
                     "algorithmic_flops_per_launch": fl, "ms_per_launch": attn_mean,
                     # both measured peaks, the 2.25 PFLOP/s data-sheet number, and the exponentials per
                     # launch (one per unmasked score)
                     "frac_of_burst": achieved_t / peaks["bf16_tflops"],
                     "frac_of_sustained": achieved_t / peaks["bf16_tflops_sustained"],
                     "frac_of_spec": achieved_t / SPEC_BF16_TFLOPS,
                     "exp_per_launch": wp.B * wp.h_q * wp.L * (wp.L + 1) // 2,
                     "exp_per_s": wp.B * wp.h_q * wp.L * (wp.L + 1) / 2 / (attn_mean * 1e-3)},
        "cpu_baseline": cpu_base,
        "only": only,
        "e2e": {"value": world * fl / (e2e_pre * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": pre_io[0], "d2h_bytes_per_step": pre_io[1], "ms_per_step": e2e_pre,
                "note": "steps pipelined over three streams (copy in, gqa_prefill, copy out) with two buffer "
                        "sets; every step copies its own inputs in and its output out"},
        "gpu_launches": (2 * do_p + 3 * do_d) * 2 * K + (6 * K if qkv_line else 0)
                        + 2 * 2 * K * sum(1 for n in (configs or {}) if n != wp.name)
                        + (3 * 2 * K if dec_alone[0] == dec_alone[0] else 0)
                        + ((2 + 3) * K if dec_rot[0] == dec_rot[0] else 0)
                        + ((2 + 3) * K if e2e_pre == e2e_pre else 0),
        "qkv": qkv_line,
        "clocks": clocks,
        "decode": {
            "workload": wd.desc, "total_cache_rows": total_rows,
            "layout": f"paged: {page} rows per page, pages scattered in a seeded random order" if page
                      else "packed",
            "k_cache": "keys kept after RoPE (gqa_set_decode_cache_rotated(1)): only the query is rotated"
                       if k_cache == "rotated" else "raw keys, each rotated on load at its position",
            "value": world * allb / (dec_mean * 1e-3) / 1e9, "unit": "GB/s",
            "kv_gbs": world * kvb / (dec_mean * 1e-3) / 1e9,
            "ms_per_step": dec_mean,
            "roofline": {"kernel": "split_kernel (decode)", "bound": "hbm", "achieved": achieved_b,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved_b / peaks["hbm_gbs"],
                         "peak_source": f"{peak_src} HBM copy",
                         "traffic": profile_traffic("split_kernel", DECODE_WORKLOAD + (f"-paged{page}" if page else "")
                                                    + ("-rotated" if k_cache == "rotated" else "")),
                         "algorithmic_bytes_per_launch": allb, "ms_per_launch": split_mean},
            "alone": {"ms_per_step": dec_alone[0], "value": world * allb / (dec_alone[0] * 1e-3) / 1e9, "unit": "GB/s",
                      "split_ms_per_launch": dec_alone[1],
                      "split_frac": allb / (dec_alone[1] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                      "note": "the same decode in steps of its own (L2 flushed before each), timed before the "
                              "prefill legs, on a GPU not yet warm"},
            "rotated_cache": {"ms_per_step": dec_rot[0], "value": world * allb / (dec_rot[0] * 1e-3) / 1e9,
                              "unit": "GB/s", "split_ms_per_launch": dec_rot[1],
                              "split_frac": allb / (dec_rot[1] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                              "traffic": profile_traffic("split_kernel", DECODE_WORKLOAD
                                                         + (f"-paged{page}" if page else "") + "-rotated"),
                              "note": "the same decode over a cache that keeps its keys after RoPE "
                                      "(gqa_set_decode_cache_rotated(1)): only the query is rotated; each step "
                                      "follows the prefill as in the headline step (events around the decode)"},
            "e2e": {"value": world * allb / (e2e_dec * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": dec_io[0], "d2h_bytes_per_step": dec_io[1],
                    "note": "the KV cache is resident device state; the step's inputs are q, the lengths"
                            + (" and the block table" if page else "")},
        },
        "wall_s_timed_region": t_wall,
        "impl": "ours",
        # every prefill workload: the headline's own figures, then the others (timed before it)
        "configs": dict({wp.name: config_entry(wp, world=world, step_ms=pre_mean, attn_ms=attn_mean, peaks=peaks,
                                               peak_src=peak_src, cpu_base=cpu_base, clocks=clocks,
                                               wall_s=t_wall)} if do_p else {},
                        **(configs or {})),
    }
    if not do_p:   # --only decode: the line carries the decode half alone
        line["roofline"] = line["e2e"] = line["cpu_baseline"] = None
    if not do_d:   # --only prefill
        line["decode"] = None
    return line


def run_ours(args):
    rank, local, world = dist_env()
    dist_init(world)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from grouped_query_attention_gqa_b200 import build
    if rank == 0 or world == 1:
        build.build()
    barrier()
    import grouped_query_attention_gqa_b200 as G
    G.load()

    wp = gi.BY_NAME[args.prefill_workload]
    wd = gi.BY_NAME[DECODE_WORKLOAD]
    if args.decode_batch:
        wd = wd.with_(B=args.decode_batch, desc=wd.desc.replace("B=64", f"B={args.decode_batch}"))
    do_p, do_d = args.only in (None, "prefill"), args.only in (None, "decode")
    if do_p:
        q, k, v = gi.prefill_inputs(wp, device=str(dev))
    else:   # placeholders of the right shape; the prefill does not run
        q, k, v = (torch.empty(1, 1, 1, 8, dtype=torch.bfloat16, device=dev) for _ in range(3))
    out = torch.empty_like(q)
    page = args.decode_page_size
    # --decode-cache rotated: every decode of the run reads a cache that keeps its keys after RoPE (random
    # keys serve as rotated keys as well as raw ones, so the same cache is used)
    rotated_run = args.decode_cache == "rotated"
    G.set_decode_cache_rotated(rotated_run)
    table = None
    if do_d and page:   # the same logical cache, scattered over pages of `page` rows
        s, qd, kc, vc, table, _, _, _ = gi.decode_paged_inputs(wd, page, device=str(dev))
    elif do_d:
        s, qd, kc, vc = gi.decode_inputs(wd, device=str(dev))
    else:
        s = torch.ones(1, dtype=torch.int32, device=dev)
        qd, kc, vc = (torch.empty(1, 1, 8, dtype=torch.bfloat16, device=dev) for _ in range(3))
    outd = torch.empty_like(qd)

    def dec_call(qx, sx, tx):
        if tx is None:
            G.decode(qx, kc, vc, sx, theta=wd.theta, out=outd)
        else:
            G.decode_paged(qx, kc, vc, tx, sx, theta=wd.theta, out=outd)
    total_rows = int(s.sum().item())
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    K, W = args.steps, args.warmup

    # ---- the decode alone, first, on a GPU not yet heated by the long prefills: K steps of decode only (L2
    # flushed before each), beside the in-step figure.  The same decode runs ~20 % slower once the GPU is
    # warm (measured: right after the long prefill, after it and 2 ms idle, and alone again later with the
    # SM clock lowered under the power cap), so the step's decode half is reported as measured and this
    # one beside it.
    dec_alone_ms = split_alone_ms = float("nan")
    if do_d and do_p:
        for _ in range(W):
            flush.zero_()
            dec_call(qd, s, table)
        da = [[ev() for _ in range(4)] for _ in range(K)]
        torch.cuda.synchronize()
        barrier()
        for i in range(K):
            flush.zero_()
            da[i][0].record()
            dec_call(qd, s, table)
            da[i][3].record()
            flush.zero_()
            G.set_timing_events(da[i][1], da[i][2])
            dec_call(qd, s, table)
            G.set_timing_events(None, None)
        torch.cuda.synchronize()
        barrier()
        dec_alone_ms = reduce_max(sum(e[0].elapsed_time(e[3]) for e in da) / K, dev)
        split_alone_ms = sum(e[1].elapsed_time(e[2]) for e in da) / K

    peaks, peak_src = load_peaks()
    # ---- the other prefill workloads, one after another (each rank its own copy), each with its own
    # step and kernel times, roofline fraction and (rank 0 of a 1-GPU run) a bounded CPU-oracle sample.
    # Timed before the headline, like the decode alone: after seconds of the long prefill the GPU runs
    # its short workloads at a lower SM clock under the power cap (L=4096: ~1790 against 1965 MHz).
    configs = {}
    names = [] if args.configs in ("", "none") or not do_p else [n for n in args.configs.split(",") if n != wp.name]
    for name in names:
        wc = gi.BY_NAME[name]
        with ClockSampler(local) as c_clk:
            c_step, c_attn, c_wall = measure_prefill(G, wc, K, W, flush, dev)
        c_cpu = cpu_baseline(wc, budget_s=4.0) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
        configs[name] = config_entry(wc, world=world, step_ms=c_step, attn_ms=c_attn, peaks=peaks,
                                     peak_src=peak_src, cpu_base=c_cpu, clocks=c_clk.summary(), wall_s=c_wall)

    def step(evs=None, inner=False):
        """One step; with `inner` the library also records events around its main kernels (separate steps
        time the kernels, so the headline steps carry no events between the prep and attention kernels)."""
        flush.zero_()
        if evs:
            evs[0].record()
        if evs and inner:
            G.set_timing_events(evs[1], evs[2])
        if do_p:
            G.prefill(q, k, v, theta=wp.theta, out=out)
        if evs:
            evs[3].record()
        if evs and inner:
            G.set_timing_events(evs[4], evs[5])
        if do_d:
            dec_call(qd, s, table)
        if evs:
            evs[6].record()
        if evs and inner:
            G.set_timing_events(None, None)

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    if G.last_error() != 0:
        raise RuntimeError("device error during warm-up")
    evs = [[ev() for _ in range(7)] for _ in range(K)]       # headline steps
    kevs = [[ev() for _ in range(7)] for _ in range(K)]      # kernel-timing steps
    torch.cuda.synchronize()

    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    with sampler:
        t_wall = time.perf_counter()
        for i in range(K):   # interleaved, so both kinds of step see the same clocks and temperature
            step(evs[i])
            step(kevs[i], inner=True)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    barrier()
    torch.cuda.synchronize()
    if G.last_error() != 0:
        raise RuntimeError("device error in the timed region")

    pre_ms = [e[0].elapsed_time(e[3]) for e in evs]
    attn_ms = [e[1].elapsed_time(e[2]) if do_p else float("nan") for e in kevs]
    dec_ms = [e[3].elapsed_time(e[6]) for e in evs]
    split_ms = [e[4].elapsed_time(e[5]) if do_d else float("nan") for e in kevs]
    fl = prefill_flops(wp)
    value_tflops = whole_job_rate(fl, 1e-3 * sum(pre_ms) / K, dev) / 1e12   # every rank: same collectives
    pre_mean = reduce_max(sum(pre_ms) / K, dev)
    if not do_p:   # --only decode: no prefill was timed, so there is no headline value
        value_tflops = pre_mean = None
    dec_mean = reduce_max(sum(dec_ms) / K, dev)
    attn_mean = sum(attn_ms) / K
    split_mean = sum(split_ms) / K

    # ---- the same decode over a cache that keeps its keys after RoPE (gqa_set_decode_cache_rotated): the
    # decode rotates only the query.  Random keys serve as rotated keys as well as raw ones, so the same
    # cache is used.  Each step follows the prefill, as the headline step's decode half does.
    dec_rot_ms = split_rot_ms = float("nan")
    if do_d and do_p and not rotated_run:
        rv = [[ev() for _ in range(4)] for _ in range(K)]
        torch.cuda.synchronize()
        barrier()
        G.set_decode_cache_rotated(True)
        try:
            for i in range(K):
                flush.zero_()
                G.prefill(q, k, v, theta=wp.theta, out=out)
                rv[i][0].record()
                G.set_timing_events(rv[i][1], rv[i][2])
                dec_call(qd, s, table)
                G.set_timing_events(None, None)
                rv[i][3].record()
            torch.cuda.synchronize()
        finally:
            G.set_decode_cache_rotated(False)
        barrier()
        if G.last_error() != 0:
            raise RuntimeError("device error in the rotated-cache decode leg")
        dec_rot_ms = reduce_max(sum(e[0].elapsed_time(e[3]) for e in rv) / K, dev)
        split_rot_ms = sum(e[1].elapsed_time(e[2]) for e in rv) / K

    # ---- end to end through the public API: every step copies its inputs in from pinned host memory, runs
    # the call and copies its result out to pinned host memory.  The prefill steps are pipelined as a
    # serving process would run them: copies in on one stream, the call on another, copies out on a third,
    # with two sets of device buffers, so step i+1's inputs travel while step i computes and step i-1's
    # output travels back.  The rate is taken over K steps in steady state (after W), from the output copy
    # of step W-1 to that of step W+K-1.  The decode steps (inputs and outputs of a few hundred KB) run one
    # after another on one stream.
    run_e2e = not args.no_e2e and do_p and do_d
    e2e_pre = e2e_dec = float("nan")
    if run_e2e:
        qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
        outh = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        dins = [tuple(torch.empty_like(x) for x in (q, k, v)) for _ in range(2)]
        douts = [torch.empty_like(out) for _ in range(2)]
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        n = W + K
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_cmp = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        torch.cuda.synchronize()
        barrier()
        for i in range(n):
            j = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[i - 2])        # buffer set j no longer read
                for dst, src in zip(dins[j], (qh, kh, vh)):
                    dst.copy_(src, non_blocking=True)
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[i])
                if i >= 2:
                    s_cmp.wait_event(ev_out[i - 2])       # output buffer j copied out
                G.prefill(*dins[j], theta=wp.theta, out=douts[j])
                ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                outh[j].copy_(douts[j], non_blocking=True)
                ev_out[i].record(s_out)
        torch.cuda.synchronize()
        barrier()
        e2e_pre = reduce_max(ev_out[W - 1].elapsed_time(ev_out[W + K - 1]) / K, dev)

        qdh, sh_ = qd.cpu().pin_memory(), s.cpu().pin_memory()
        outdh = torch.empty(outd.shape, dtype=outd.dtype).pin_memory()
        qdx, sx = torch.empty_like(qd), torch.empty_like(s)
        th = table.cpu().pin_memory() if table is not None else None
        tx = torch.empty_like(table) if table is not None else None

        def e2e_dec_step(e):
            flush.zero_()
            e[0].record()
            qdx.copy_(qdh, non_blocking=True)
            sx.copy_(sh_, non_blocking=True)
            if tx is not None:
                tx.copy_(th, non_blocking=True)
            dec_call(qdx, sx, tx)
            outdh.copy_(outd, non_blocking=True)
            e[1].record()

        for _ in range(max(1, W)):
            e2e_dec_step([ev() for _ in range(2)])
        e2e_evs = [[ev() for _ in range(2)] for _ in range(K)]
        torch.cuda.synchronize()
        barrier()
        for i in range(K):
            e2e_dec_step(e2e_evs[i])
        torch.cuda.synchronize()
        barrier()
        e2e_dec = reduce_max(sum(e[0].elapsed_time(e[1]) for e in e2e_evs) / K, dev)
        del dins, douts, outh

    # ---- the fused route from hidden states: QKV projection + bias + RoPE (writing Q', K' and the cache
    # rows K, V), then the attention on the rotated inputs -- no prep pass.  Timed like the headline
    # steps, plus K steps with events around the projection kernel alone.
    qkv_line = None
    if do_p and not args.no_qkv:
        dm = gi.D_MODEL[(wp.h_q, wp.h_kv, wp.d)]
        xq, wqkv, bqkv = gi.qkv_inputs(wp, d_model=dm, device=str(dev))
        _, w_o, x_in = gi.out_proj_inputs(wp, d_model=dm, device=str(dev))
        y_out = torch.empty_like(x_in)
        qo = (q.new_empty(wp.B, wp.h_q, wp.L, wp.d), q.new_empty(wp.B, wp.h_kv, wp.L, wp.d),
              q.new_empty(wp.B, wp.L, wp.h_kv, wp.d), q.new_empty(wp.B, wp.L, wp.h_kv, wp.d))

        def qstep(e, inner=False):
            flush.zero_()
            e[0].record()
            if inner:
                G.set_timing_events(e[1], e[2])
            G.qkv_rope(xq, wqkv, bqkv, wp.h_q, wp.h_kv, theta=wp.theta, out=qo)
            if inner:
                G.set_timing_events(None, None)
            G.prefill_rotated(qo[0], qo[1], qo[3], out=out)
            if inner:
                G.set_timing_events(e[4], e[5])
            G.out_proj(out, w_o, x_in, out=y_out)
            if inner:
                G.set_timing_events(None, None)
            e[3].record()

        for _ in range(W):
            qstep([ev() for _ in range(6)])
        qe = [[ev() for _ in range(6)] for _ in range(K)]
        qke = [[ev() for _ in range(6)] for _ in range(K)]
        torch.cuda.synchronize()
        barrier()
        with ClockSampler(local) as q_clk:
            q_wall = time.perf_counter()
            for i in range(K):
                qstep(qe[i])
                qstep(qke[i], inner=True)
            torch.cuda.synchronize()
            q_wall = time.perf_counter() - q_wall
        barrier()
        if G.last_error() != 0:
            raise RuntimeError("device error in the QKV leg")
        qfl = 2.0 * wp.B * wp.L * dm * (wp.h_q + 2 * wp.h_kv) * wp.d
        ofl = 2.0 * wp.B * wp.L * (wp.h_q * wp.d) * dm
        route_ms = reduce_max(sum(e[0].elapsed_time(e[3]) for e in qe) / K, dev)
        qkv_ms = sum(e[1].elapsed_time(e[2]) for e in qke) / K
        proj_ms = sum(e[4].elapsed_time(e[5]) for e in qke) / K
        peaks_q, src_q = load_peaks()
        # The same peak rule as the attention kernel's: the sustained figure for a leg that ran long under
        # the power cap, else the burst one; both fractions are carried.
        q_clocks = q_clk.summary()
        q_peak, q_kind = tensor_peak(peaks_q, q_clocks, q_wall)
        q_ach, o_ach = qfl / (qkv_ms * 1e-3) / 1e12, ofl / (proj_ms * 1e-3) / 1e12
        qkv_line = {
            "workload": f"{wp.desc}, d_model={dm}: X [{wp.B * wp.L}, {dm}] x W_qkv^T [{dm}, {(wp.h_q + 2 * wp.h_kv) * wp.d}]"
                        " + bias, RoPE on Q and K, Q'/K' head-major and K/V cache rows written",
            "flops_per_step": qfl,
            "roofline": {"kernel": "qkv_kernel", "bound": "tensor", "achieved": q_ach,
                         "peak": q_peak, "unit": "TFLOP/s", "frac": q_ach / q_peak,
                         "peak_source": f"{src_q} bf16 dense ({q_kind})",
                         "frac_of_burst": q_ach / peaks_q["bf16_tflops"],
                         "frac_of_sustained": q_ach / peaks_q["bf16_tflops_sustained"],
                         "traffic": profile_traffic("qkv_kernel", wp.name),
                         "algorithmic_flops_per_launch": qfl, "ms_per_launch": qkv_ms},
            "out_proj": {"kernel": "proj_kernel", "bound": "tensor", "flops_per_launch": ofl,
                         "traffic": profile_traffic("proj_kernel", wp.name),
                         "peak": q_peak, "peak_source": f"{src_q} bf16 dense ({q_kind})",
                         "ms_per_launch": proj_ms, "achieved": o_ach, "frac": o_ach / q_peak, "unit": "TFLOP/s",
                         "frac_of_burst": o_ach / peaks_q["bf16_tflops"],
                         "frac_of_sustained": o_ach / peaks_q["bf16_tflops_sustained"],
                         "note": "attn [T, h_q d] x W_O^T [h_q d, d_model] + residual"},
            "clocks": q_clocks,
            "wall_s_timed_region": q_wall,
            "sublayer": {"ms_per_step": route_ms,
                         "value": world * (qfl + fl + ofl) / (route_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                         "note": "the attention sub-layer from hidden states: QKV projection + bias + RoPE, "
                                 "attention on the rotated inputs, W_O + residual (no prep pass)"},
        }
        del xq, wqkv, bqkv, qo, w_o, x_in, y_out

    line = None
    if rank == 0:
        line = build_line(
            world=world, K=K, W=W, only=args.only, do_p=do_p, do_d=do_d, wp=wp, wd=wd, value_tflops=value_tflops,
            pre_mean=pre_mean, attn_mean=attn_mean, dec_mean=dec_mean, split_mean=split_mean, total_rows=total_rows,
            page=page, peaks=peaks, peak_src=peak_src,
            cpu_base=cpu_baseline(wp) if (world == 1 and do_p and not args.no_cpu_baseline) else None,
            e2e_pre=e2e_pre, e2e_dec=e2e_dec,
            pre_io=(sum(x.numel() * x.element_size() for x in (q, k, v)), out.numel() * out.element_size()),
            dec_io=(qd.numel() * 2 + s.numel() * 4 + (table.numel() * 4 if page else 0), outd.numel() * 2),
            qkv_line=qkv_line, clocks=sampler.summary(), t_wall=t_wall, configs=configs,
            dec_alone=(dec_alone_ms, split_alone_ms), dec_rot=(dec_rot_ms, split_rot_ms), k_cache=args.decode_cache)
    if torch.distributed.is_initialized():
        barrier()
        torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(clean(line)), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours",
                    help="ours: the CUDA path; reference: the fp64 oracle on the host")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the host oracle timing")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffer) leg")
    ap.add_argument("--only", choices=["prefill", "decode"], default=None,
                    help="run one half of the step only (profiling; the line then carries that half)")
    ap.add_argument("--prefill-workload", default=PREFILL_WORKLOAD, choices=[w.name for w in gi.WORKLOADS if w.kind == "prefill"],
                    help="prefill workload of the step (default: the Qwen2-7B L=32768 headline workload)")
    ap.add_argument("--configs", default=",".join(CONFIG_WORKLOADS),
                    help="comma list of further prefill workloads timed before the headline and reported under "
                         "`configs` ('none' for none)")
    ap.add_argument("--no-qkv", action="store_true", help="skip the fused QKV projection leg")
    ap.add_argument("--decode-cache", choices=["raw", "rotated"], default="raw",
                    help="what the decode's K cache holds: raw keys rotated on load (default), or keys kept after "
                         "RoPE (gqa_set_decode_cache_rotated)")
    ap.add_argument("--decode-page-size", type=int, default=None,
                    help="decode through gqa_decode_paged, the cache in pages of this many rows")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="decode with this many sequences instead of 64 (smaller profiling case)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
