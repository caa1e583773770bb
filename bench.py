#!/usr/bin/env python
"""Benchmark of the paged E4M3 decode attention on B200.

Metric: KV-read HBM GB/s per decode call (algorithmic K+V bytes of the attended
tokens / call time), with % of the measured HBM peak and us/call.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl native|reference]

One step = one decode call (the persistent split kernel and, when a sequence spans
several splits, the combine kernel) over the whole batch
of the named synthetic workload (default: the large mixed batch, B=256, Hq=64,
Hkv=8, D=128, 32-token pages, lognormal lengths of median 2048, window 4096,
sinks: the largest single-GPU workload).  The same run then measures the other
four workloads the same way and adds them to the line under "per_config"
(long context, Llama-3-8B-shaped, sliding window + sinks, tiny).  Inputs are
resident in HBM; consecutive steps read different replicas of the KV cache so
that the bytes of one step are not in L2 for the next (replicas x KV bytes >
2 x L2).  Timing: CUDA events on the launching stream around exactly K steps,
barrier + synchronize on both sides, max over ranks.  Multi-GPU (torchrun) runs
independent replicas, one per GPU (weak scaling): the path has no exchange.

`--impl reference` times the fp64 CPU oracle (on the host cores, bounded
samples of the same workload) and prints the same JSON line with
"impl": "reference".

`--op cache_write` instead measures the FP8 KV-cache write (bf16 K/V of new
tokens quantised and scattered into the paged caches): HBM GB/s of its bytes
(4 read + 2 written per element) on a prefill-sized batch larger than L2
(`--write-tokens`, default 65536 tokens of the Llama-3-8B shape: 384 MB per
call) and the latency of a decode-step batch (one token per sequence of the
decode workload), timed as replays of a CUDA graph of 100 calls so that host
launch overhead is excluded.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV-read HBM GB/s and % of B200 peak per decode call; µs/call"
UNIT = "GB/s"
DEFAULT_CONFIG = "large_mixed"
# measured beside the default workload in the same run (per_config)
PER_CONFIG_DEFAULT = ("tiny", "llama3_8b", "swa_sinks", "long_context")
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--per-config", default="",
                    help="comma-separated workloads measured after the headline one in the same "
                         "run ('none': only the headline; default: every other workload when "
                         "the headline is the default E4M3 single-query decode)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--chunk-pages", type=int, default=0, help="force pages per split (tuning)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU baseline sample budget")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="skip the CUDA-graph replay timing (L2 flushed before each replay)")
    ap.add_argument("--kernels-only", action="store_true",
                    help="only run warm-up + K plain calls (for ncu launch lists and captures)")
    ap.add_argument("--json-out", default=None)
    ap.add_argument("--op", default="decode", choices=["decode", "cache_write", "cp"])
    ap.add_argument("--cp-fused", action="store_true",
                    help="--op cp: the exchange fused into the decode (peer-memory stores and "
                         "flags) instead of an NCCL all-gather")
    ap.add_argument("--cp-ranks", type=int, default=8,
                    help="--op cp on one process: the context-parallel width whose rank "
                         "step is timed (under torchrun the world size is the width)")
    ap.add_argument("--kv-format", default="e4m3", choices=["e4m3", "nvfp4"],
                    help="page format: E4M3 (token-major) or NVFP4 (head-major) pages")
    ap.add_argument("--q-len", type=int, default=1,
                    help="query tokens per sequence (speculative decode of the same workload)")
    ap.add_argument("--write-tokens", type=int, default=65536)
    return ap.parse_args()


def whole_job_value(world_size, kv_bytes_per_call, steps, max_total_ms):
    """Whole-job KV GB/s: every rank ran `steps` calls of `kv_bytes_per_call`; the
    time is the maximum over ranks."""
    return world_size * kv_bytes_per_call * steps / (max_total_ms / 1e3) / 1e9


def max_over_ranks(value_ms, device=None):
    """Max of a per-rank time over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value_ms)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (earlier measurement on this pool)"


# The device code of the split and combine kernels; the ncu traffic record is
# valid only for this exact code and, per workload, for the launch plan it
# records (checked in ncu_traffic).
KERNEL_SOURCES = ("fpd_kernels.cuh", "fpd_ptx.cuh")


def cudart():
    """The CUDA runtime library torch loads (raw async copies and event calls
    for the end-to-end host loop)."""
    from fp8_paged_decode_b200 import cp
    return cp._cudart()


def _code_lines(text):
    """The source without // comments and blank lines (a line holding a string
    literal keeps its text after //), so that comment edits keep the hash."""
    out = []
    for line in text.splitlines():
        if '"' not in line and "//" in line:
            line = line[:line.index("//")]
        line = line.rstrip()
        if line:
            out.append(line)
    return "\n".join(out)


def kernel_source_hash():
    """sha256 of the split kernel's device code (fpd_kernels.cuh, fpd_ptx.cuh)
    without comments: the key of the committed DRAM-traffic record."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fp8_paged_decode_b200", "csrc")
    for fn in KERNEL_SOURCES:
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            h.update(fn.encode())
            h.update(_code_lines(f.read()).encode())
    return h.hexdigest()


def traffic_key(config_name, q_len, kv_format="e4m3"):
    key = config_name if q_len == 1 else f"{config_name}/q{q_len}"
    return key if kv_format == "e4m3" else f"{key}/{kv_format}"


def ncu_traffic(config_name, kv_bytes, plan=None, q_len=1, kv_format="e4m3"):
    """DRAM bytes per split-kernel launch from the committed ncu summary, scaled
    to this launch's KV bytes; None when absent, taken on other kernel code or
    recorded for another launch plan."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_sha256") != kernel_source_hash():
        return None
    e = d.get("workloads", {}).get(traffic_key(config_name, q_len, kv_format))
    if not e:
        return None
    if plan is not None and e.get("plan") is not None and e["plan"] != plan:
        return None
    return int(round(e["dram_bytes_per_launch"] * kv_bytes / e["kv_bytes_per_launch"]))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max((num(r[3]) or 0) for r in rows)}


class RawEvents:
    """CUDA events created and read through the CUDA runtime directly, so that
    events recorded inside the C library can be timed."""

    def __init__(self, n):
        from cuda.bindings import runtime as rt
        self.rt = rt
        self.ev = []
        for _ in range(n):
            err, e = rt.cudaEventCreate()
            assert int(err) == 0, err
            self.ev.append(e)

    def handle(self, i):
        return int(self.ev[i])

    def record(self, i, stream_handle):
        err, = self.rt.cudaEventRecord(self.ev[i], stream_handle)
        assert int(err) == 0, err

    def ms(self, i, j):
        err, v = self.rt.cudaEventElapsedTime(self.ev[i], self.ev[j])
        assert int(err) == 0, err
        return float(v)

    def close(self):
        for e in self.ev:
            self.rt.cudaEventDestroy(e)
        self.ev = []


# ------------------------------------------------------------ CPU oracle --

def make_wl(args):
    from fp8_paged_decode_b200 import workloads as W
    if args.kv_format == "nvfp4":
        return W.make_workload_nvfp4(args.config, q_len=args.q_len)
    return W.make_workload(args.config, q_len=args.q_len)


def oracle_rows(wl, rows, threads=None):
    import oracle
    if wl.kv_format == "nvfp4":
        return oracle.decode_nvfp4_workload(wl, rows=rows, threads=threads)
    return oracle.decode_workload(wl, rows=rows, threads=threads)


def rows_kv_bytes(wl, rows):
    """The workload's algorithmic KV bytes that the given output rows stand
    for: a sequence's K+V bytes are shared by its q_len * Hq rows, so each row
    is credited with that share (the metric counts each KV byte once)."""
    import numpy as np
    att = wl.attended().astype(np.float64)
    per_seq = wl.q_len * wl.Hq
    seq_bytes = att / max(att.sum(), 1.0) * wl.kv_bytes()
    return sum(float(seq_bytes[int(r) // per_seq]) for r in rows) / per_seq


def oracle_sample(wl, budget_s, rng_seed=0, threads=None, min_rows=1):
    """Run the oracle on random (sequence, head) rows until about budget_s of
    wall time is spent; returns (seconds, kv_bytes_read, rows, threads)."""
    import numpy as np
    import oracle
    threads = threads or (os.cpu_count() or 1)
    rng = np.random.default_rng(rng_seed)
    order = rng.permutation(wl.B * wl.q_len * wl.Hq)
    # calibrate on a few rows
    probe = order[:max(min_rows, min(len(order), threads))]
    t0 = time.perf_counter()
    oracle_rows(wl, probe, threads=threads)
    t_probe = time.perf_counter() - t0
    per_row = t_probe / len(probe)
    n = int(max(min_rows, min(len(order), budget_s / max(per_row, 1e-6))))
    rows = order[:n]
    t0 = time.perf_counter()
    oracle_rows(wl, rows, threads=threads)
    dt = time.perf_counter() - t0
    return dt, rows_kv_bytes(wl, rows), n, threads


def run_reference(args):
    """The oracle as the reference arm: every step runs it on a bounded random
    sample of (sequence, head) rows of the same workload, using all host cores."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np
    from fp8_paged_decode_b200 import workloads as W
    import oracle
    wl = make_wl(args)
    threads = os.cpu_count() or 1
    total_steps = args.steps + args.warmup
    budget_s = 120.0
    # calibrate: wall time of one parallel batch of `threads` rows
    n_rows = wl.B * wl.q_len * wl.Hq
    probe = np.arange(min(n_rows, threads))
    t0 = time.perf_counter()
    oracle_rows(wl, probe, threads=threads)
    per_row_wall = (time.perf_counter() - t0) / len(probe)
    rows_per_step = int(budget_s / total_steps / max(per_row_wall, 1e-7))
    rows_per_step = max(1, min(rows_per_step, n_rows))
    rng = np.random.default_rng(7)
    t_sum, kv_sum = 0.0, 0
    for step in range(total_steps):
        rows = rng.choice(n_rows, size=rows_per_step, replace=False)
        t0 = time.perf_counter()
        oracle_rows(wl, rows, threads=min(threads, rows_per_step))
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            t_sum += dt
            kv_sum += rows_kv_bytes(wl, rows)
    value = kv_sum / t_sum / 1e9
    hbm, _ = measured_peaks()
    sample = (f"{rows_per_step} random (sequence, query token, head) rows of the workload per "
              f"step, each credited with its share of the sequence's KV bytes")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_sum / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": W.describe(args.config), "q_len": wl.q_len,
                   "kv_format": wl.kv_format, "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(threads, rows_per_step),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "pct_of_peak": 100.0 * value / hbm,
    }
    print(json.dumps(line))
    if args.json_out:
        with open(args.json_out, "w") as f:
            f.write(json.dumps(line) + "\n")
    return 0


# ---------------------------------------------------------------- native --

def per_config_names(args):
    """Workloads measured beside the headline one, in the same run: every other
    configuration when the headline is the default E4M3 single-query decode."""
    if args.per_config == "none":
        return []
    if args.per_config:
        names = [n for n in args.per_config.split(",") if n]
    elif args.config == DEFAULT_CONFIG and args.q_len == 1 and args.kv_format == "e4m3":
        names = list(PER_CONFIG_DEFAULT)
    else:
        names = []
    return [n for n in names if n != args.config]


def per_config_entry(line):
    """The figures of one workload's line that the per-configuration table keeps."""
    rf = line["roofline"]
    return {"workload": line["config"]["workload"], "kv_bytes_per_call":
            line["config"]["kv_bytes_per_call"], "us_per_call": line["us_per_call"],
            "kv_gbs": line["value"], "pct_of_peak": line["pct_of_peak"],
            "split_kernel_us": line["split_kernel_us"],
            "combine_kernel_us": line["combine_kernel_us"],
            "roofline_frac": rf["frac"], "roofline_traffic": rf["traffic"],
            "graph_replay_cold_l2": line["graph_replay_cold_l2"], "e2e": line["e2e"],
            "parity_guard": line["parity_guard"], "clocks": line["clocks"],
            "steps": line["steps"], "warmup": line["warmup"], "plan": line["config"]["plan"]}


def run_native(args):
    import torch
    import torch.distributed as dist

    import fp8_paged_decode_b200 as fpd

    ws, rank, local = dist_env()
    assert ws == args.gpus, f"--gpus {args.gpus} but WORLD_SIZE={ws}"
    torch.cuda.set_device(local)
    if ws > 1:
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=120))

    def barrier():
        if ws > 1:
            dist.barrier()

    lib = fpd.load_library()
    line = measure_native(args, lib, ws, rank, local, barrier)
    if line is not None and not args.kernels_only:
        others = per_config_names(args)
        if others:
            # every other workload in the same run, the same way, with at
            # least 2000 timed calls after 50 warm-up calls (short workloads
            # need that many to leave the launch ramp; the entries record
            # their counts), and no CPU baseline (quoted once, on the headline)
            table = {args.config: per_config_entry(line)} if rank == 0 else None
            for name in others:
                sub_args = argparse.Namespace(**{**vars(args), "config": name,
                                                 "no_cpu_baseline": True,
                                                 "steps": max(args.steps, 2000),
                                                 "warmup": max(args.warmup, 50)})
                sub = measure_native(sub_args, lib, ws, rank, local, barrier)
                if rank == 0:
                    table[name] = per_config_entry(sub)
                torch.cuda.empty_cache()
            if rank == 0:
                line["per_config"] = table
        if rank == 0:
            print(json.dumps(line))
            if args.json_out:
                with open(args.json_out, "w") as f:
                    f.write(json.dumps(line) + "\n")
    if ws > 1:
        dist.destroy_process_group()
    return 0


def measure_native(args, lib, ws, rank, local, barrier):
    """One workload: warm-up, K timed calls, the per-kernel event pass, the
    cold-L2 graph replay and the end-to-end loop.  Returns rank 0's JSON line
    (a dict; None on other ranks and for --kernels-only)."""
    import numpy as np
    import torch

    import fp8_paged_decode_b200 as fpd
    from fp8_paged_decode_b200 import workloads as W

    wl = make_wl(args)
    dev = torch.device("cuda", local)
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    kv_bytes = wl.kv_bytes()
    replicas = max(1, min(8, math.ceil(2 * l2 / kv_bytes) + (1 if kv_bytes < 4 * l2 else 0)))

    q = torch.from_numpy(wl.q.view(np.int16)).view(torch.bfloat16).to(dev)
    table = torch.from_numpy(wl.block_table).to(dev)
    lens = torch.from_numpy(wl.seq_lens).to(dev)
    sinks = None if wl.sinks is None else torch.from_numpy(wl.sinks).to(dev)
    nvfp4 = wl.kv_format == "nvfp4"
    if nvfp4:   # one tensor of pages [K data | K scales | V data | V scales] per replica
        kc = [torch.from_numpy(wl.kv_cache).to(dev) for _ in range(replicas)]
        vc = kc
    else:
        kc = [torch.from_numpy(wl.k_cache).to(dev) for _ in range(replicas)]
        vc = [torch.from_numpy(wl.v_cache).to(dev) for _ in range(replicas)]
    lead = tuple(wl.q.shape[:-2])   # (B,) or (B, q_len)
    out = torch.empty(lead + (wl.Hq, wl.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty(lead + (wl.Hq,), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    vp = ctypes.c_void_p

    def descriptor(i, io=None):
        """The call on replica i, as the C ABI's descriptor; io: other device
        buffers for (q, table, lens, sinks, out, lse)."""
        q_, table_, lens_, sinks_, out_, lse_ = io or (q, table, lens, sinks, out, lse)
        a = fpd.fpd_decode_args()
        a.q, a.q_dtype = q_.data_ptr(), fpd.FPD_Q_BF16
        if nvfp4:
            lay = fpd.nvfp4_page_layout(wl.Hkv, wl.block_tokens, wl.D)
            base = kc[i].data_ptr()
            a.k_cache, a.v_cache = base + lay["k_data"], base + lay["v_data"]
            a.k_scales, a.v_scales = base + lay["k_sf"], base + lay["v_sf"]
            a.kv_page_stride = a.sf_page_stride = lay["page_bytes"]
            a.kv_format, a.kv_layout = fpd.FPD_KV_NVFP4, fpd.FPD_KV_HND
        else:
            a.k_cache, a.v_cache = kc[i].data_ptr(), vc[i].data_ptr()
            a.kv_format, a.kv_layout = fpd.FPD_KV_E4M3, fpd.FPD_KV_NHD
        a.block_table, a.seq_lens = table_.data_ptr(), lens_.data_ptr()
        a.B, a.q_len, a.Hq, a.Hkv, a.D = wl.B, wl.q_len, wl.Hq, wl.Hkv, wl.D
        a.num_blocks, a.block_tokens, a.max_blocks = wl.num_blocks, wl.block_tokens, wl.max_blocks
        a.k_scale, a.v_scale, a.sm_scale = wl.k_scale, wl.v_scale, wl.sm_scale
        a.window_left = wl.window_left
        a.sinks = sinks_.data_ptr() if sinks_ is not None else None
        a.out, a.lse = out_.data_ptr(), lse_.data_ptr()
        a.chunk_pages_override = args.chunk_pages
        return a

    descs = [descriptor(i) for i in range(replicas)]
    refs = [ctypes.byref(d) for d in descs]
    need = fpd.fp8_paged_decode_workspace_bytes_args(descs[0])
    assert need > 0
    wsp = torch.zeros(need, dtype=torch.uint8, device=dev)
    plan_s = fpd.fpd_plan()
    assert lib.fp8_paged_decode_plan_args(refs[0], ctypes.byref(plan_s)) == 0
    plan = {f: getattr(plan_s, f) for f, _ in fpd.fpd_plan._fields_}
    ws_ptr, ws_n = vp(wsp.data_ptr()), ctypes.c_size_t(wsp.numel())
    f_args = lib.fp8_paged_decode_attention_args
    f_args_prof = lib.fp8_paged_decode_attention_args_profiled

    def f_plain(i):
        return f_args(refs[i % replicas], ws_ptr, ws_n, sh)

    def f_prof(i, e0, e1, e2):
        return f_args_prof(refs[i % replicas], ws_ptr, ws_n, sh, e0, e1, e2)

    if args.kernels_only:
        for i in range(args.warmup + args.steps):
            st = f_plain(i)
            assert st == 0, fpd.fp8_paged_decode_status_string(st)
        torch.cuda.synchronize()
        assert fpd.fp8_paged_decode_check_status(wsp) == 0
        if rank == 0:
            print(json.dumps({"kernels_only": True, "config": args.config, "calls":
                              args.warmup + args.steps, "launches_per_call":
                              1 + (1 if plan["max_splits"] > 1 else 0), "plan": plan,
                              "kv_bytes_per_call": kv_bytes, "replicas": replicas}))
        return None

    # correctness guard on this exact launch configuration (sampled rows vs oracle)
    st = f_plain(0)
    assert st == 0, fpd.fp8_paged_decode_status_string(st)
    torch.cuda.synchronize()
    guard = None
    if rank == 0:
        import oracle
        rng = np.random.default_rng(0)
        n_rows = wl.B * wl.q_len * wl.Hq
        rows = rng.choice(n_rows, size=min(16, n_rows), replace=False)
        ro, rl = oracle_rows(wl, rows)
        # rows index (sequence, query token, head) in that order
        o = out.float().cpu().numpy().reshape(n_rows, wl.D)
        l = lse.cpu().numpy().reshape(n_rows)
        ro = ro.reshape(n_rows, wl.D)
        rl = rl.reshape(n_rows)
        err = np.abs(o[rows] - ro[rows])
        ok = bool((err <= 1e-2 + 1e-2 * np.abs(ro[rows])).all() and
                  (np.abs(l[rows] - rl[rows]) <= 1e-3).all())
        guard = {"rows_checked": int(len(rows)), "max_abs_dout": float(err.max()),
                 "max_abs_dlse": float(np.abs(l[rows] - rl[rows]).max()), "ok": ok}
        assert ok, guard
    bits = fpd.fp8_paged_decode_check_status(wsp, clear=True)
    assert bits == 0, f"device status {bits}"

    # warm-up
    for i in range(args.warmup):
        st = f_plain(i)
        assert st == 0
    torch.cuda.synchronize()

    K = args.steps
    # Timed region: K back-to-back calls between two events, nothing recorded
    # in between (an event per call costs a few us on the small workloads).
    ev = RawEvents(2)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.25)
    barrier()
    torch.cuda.synchronize()
    ev.record(0, stream.cuda_stream)
    for i in range(K):
        st = f_plain(i)
        if st != 0:
            raise RuntimeError(fpd.fp8_paged_decode_status_string(st))
    ev.record(1, stream.cuda_stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    total_ms = ev.ms(0, 1)
    ev.close()
    # Per-call and per-kernel durations (spread and roofline): a second pass of
    # min(K, 2000) calls with events before the split kernel, between the split
    # kernel and the combine launch, and after the combine.
    Kr = min(K, 2000)
    evr = RawEvents(3 * Kr)
    torch.cuda.synchronize()
    for i in range(Kr):
        st = f_prof(i, vp(evr.handle(3 * i)), vp(evr.handle(3 * i + 1)),
                    vp(evr.handle(3 * i + 2)))
        if st != 0:
            raise RuntimeError(fpd.fp8_paged_decode_status_string(st))
    torch.cuda.synchronize()
    split_ms = [evr.ms(3 * i, 3 * i + 1) for i in range(Kr)]
    combine_ms = [evr.ms(3 * i + 1, 3 * i + 2) for i in range(Kr)]
    call_ms = [evr.ms(3 * i, 3 * i + 2) for i in range(Kr)]
    evr.close()

    max_total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = max_total_ms / K
    value = whole_job_value(ws, kv_bytes, K, max_total_ms)

    # One call captured in a CUDA graph, replayed with the L2 flushed before each
    # replay: a write of 2x L2 bytes, then a read of the same bytes, so that L2
    # holds none of the call's data and the flush's dirty lines are written back
    # before the replay starts, not during it; median and p10/p90 of the replays.
    graph = None
    if not args.no_graph:
        flush = torch.empty(2 * l2 // 4 + 1, dtype=torch.float32, device=dev)
        gstream = torch.cuda.Stream(dev)
        gstream.wait_stream(stream)
        gh = vp(gstream.cuda_stream)
        with torch.cuda.stream(gstream):
            for _ in range(3):
                assert f_args(refs[0], ws_ptr, ws_n, gh) == 0
        torch.cuda.synchronize()
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg, stream=gstream):
            st = f_args(refs[0], ws_ptr, ws_n, gh)
        assert st == 0, fpd.fp8_paged_decode_status_string(st)
        n_rep, n_warm = 1000, 100
        e_a = [torch.cuda.Event(enable_timing=True) for _ in range(n_rep)]
        e_b = [torch.cuda.Event(enable_timing=True) for _ in range(n_rep)]
        with torch.cuda.stream(gstream):
            for i in range(n_warm):
                flush.fill_(float(i))
                torch.amax(flush)
                cg.replay()
            for i in range(n_rep):
                flush.fill_(float(i))
                torch.amax(flush)
                e_a[i].record(gstream)
                cg.replay()
                e_b[i].record(gstream)
        torch.cuda.synchronize()
        tr = sorted(e_a[i].elapsed_time(e_b[i]) * 1e3 for i in range(n_rep))
        graph = {"median_us": tr[n_rep // 2], "p10_us": tr[n_rep // 10],
                 "p90_us": tr[(9 * n_rep) // 10], "replays": n_rep, "warmup_replays": n_warm,
                 "l2_flush_bytes": int(flush.numel() * 4),
                 "l2_flush": "write then read of l2_flush_bytes before each replay",
                 "kv_gbs_at_median": kv_bytes / tr[n_rep // 2] / 1e3}
        del cg
        assert fpd.fp8_paged_decode_check_status(wsp, clear=True) == 0

    # End to end through the C ABI: every step copies its inputs from pinned host
    # memory and reads its result back.  Pipelined as a serving loop would run
    # it: two sets of device inputs and outputs, the host-to-device copies on
    # one side stream and the reads on another, so that step i's copies
    # overlap the kernels of steps i - 1 and i + 1.  The serial form (copies
    # and kernels one after another on one stream) is timed too.
    e2e = None
    if not args.no_e2e:
        # a step's inputs (q, block table, lengths, sinks) sit in one buffer and
        # its results (out, lse) in another, on both sides: one copy each way
        def packed(tensors, pinned):
            offs, total = [], 0
            for t in tensors:
                offs.append(total)
                total += (t.numel() * t.element_size() + 255) // 256 * 256
            buf = (torch.empty(total, dtype=torch.uint8).pin_memory() if pinned else
                   torch.empty(total, dtype=torch.uint8, device=dev))
            views = [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                     for o, t in zip(offs, tensors)]
            return buf, views
        src = [torch.from_numpy(wl.q.view(np.int16)).view(torch.bfloat16),
               torch.from_numpy(wl.block_table), torch.from_numpy(wl.seq_lens)]
        if wl.sinks is not None:
            src.append(torch.from_numpy(wl.sinks))
        h_inbuf, h_inv = packed(src, True)
        for v, t in zip(h_inv, src):
            v.copy_(t)
        res = [out, lse]
        h_outbuf = [packed(res, True) for _ in range(2)]
        d_in = [packed(src, False) for _ in range(2)]
        d_out = [packed(res, False) for _ in range(2)]
        h2d = h_inbuf.numel()
        d2h = h_outbuf[0][0].numel()
        io = []
        for j in range(2):
            v = d_in[j][1]
            io.append((v[0], v[1], v[2], v[3] if wl.sinks is not None else None,
                       d_out[j][1][0], d_out[j][1][1]))
        edescs = [[descriptor(i, io[j]) for j in range(2)] for i in range(replicas)]
        erefs = [[ctypes.byref(d) for d in row] for row in edescs]
        # copies, event records and waits go straight to the CUDA runtime, so
        # that the host side of a step costs a few microseconds
        rt = cudart()
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        h_in, h_out = vp(s_in.cuda_stream), vp(s_out.cuda_stream)
        evs = [[torch.cuda.Event() for _ in range(2)] for _ in range(3)]
        for row in evs:   # every buffer starts free (this also creates the events)
            for e in row:
                e.record(stream)
        torch.cuda.synchronize()
        ev_in, ev_k, ev_out = [[vp(e.cuda_event) for e in row] for row in evs]

        def copies(j):
            return ([(vp(d_in[j][0].data_ptr()), vp(h_inbuf.data_ptr()), h2d)],
                    [(vp(h_outbuf[j][0].data_ptr()), vp(d_out[j][0].data_ptr()), d2h)])
        cps = [copies(0), copies(1)]
        H2D, D2H = 1, 2

        def e2e_step(i):   # returns the OR of the runtime's error codes
            j = i % 2
            ins, outs = cps[j]
            err = rt.cudaStreamWaitEvent(h_in, ev_k[j], 0)   # step i - 2 has read these inputs
            for d, h, n in ins:
                err |= rt.cudaMemcpyAsync(d, h, n, H2D, h_in)
            err |= rt.cudaEventRecord(ev_in[j], h_in)
            err |= rt.cudaStreamWaitEvent(sh, ev_in[j], 0)
            err |= rt.cudaStreamWaitEvent(sh, ev_out[j], 0)   # step i - 2's results have left
            st = f_args(erefs[i % replicas][j], ws_ptr, ws_n, sh)
            if st != 0:
                raise RuntimeError(fpd.fp8_paged_decode_status_string(st))
            err |= rt.cudaEventRecord(ev_k[j], sh)
            err |= rt.cudaStreamWaitEvent(h_out, ev_k[j], 0)
            for h, d, n in outs:
                err |= rt.cudaMemcpyAsync(h, d, n, D2H, h_out)
            return err | rt.cudaEventRecord(ev_out[j], h_out)

        def serial_step(i):
            ins, outs = cps[0]
            err = 0
            for d, h, n in ins:
                err |= rt.cudaMemcpyAsync(d, h, n, H2D, sh)
            st = f_args(erefs[i % replicas][0], ws_ptr, ws_n, sh)
            if st != 0:
                raise RuntimeError(fpd.fp8_paged_decode_status_string(st))
            for h, d, n in outs:
                err |= rt.cudaMemcpyAsync(h, d, n, D2H, sh)
            return err

        Ke = K
        for i in range(min(args.warmup, 50)):
            assert e2e_step(i) == 0, "CUDA runtime error in the end-to-end loop"
        torch.cuda.synchronize()
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        s_in.wait_event(s2)
        err = 0
        for i in range(Ke):
            err |= e2e_step(i)
        stream.wait_stream(s_out)
        e2.record(stream)
        torch.cuda.synchronize()
        barrier()
        te = max_over_ranks(s2.elapsed_time(e2), dev)
        assert err == 0, "CUDA runtime error in the end-to-end loop"
        # the last step's result must be what the device computed
        last = (Ke - 1) % 2
        assert torch.equal(h_outbuf[last][0], d_out[last][0].cpu())
        # serial: copies and the call back to back on one stream
        Ks = min(Ke, 2000)
        s3, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s3.record(stream)
        for i in range(Ks):
            err |= serial_step(i)
        e3.record(stream)
        torch.cuda.synchronize()
        barrier()
        ts = max_over_ranks(s3.elapsed_time(e3), dev)
        assert err == 0, "CUDA runtime error in the end-to-end loop"
        e2e = {"value": whole_job_value(ws, kv_bytes, Ke, te), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": te / Ke,
               "serial": {"value": whole_job_value(ws, kv_bytes, Ks, ts),
                          "ms_per_step": ts / Ks},
               "note": "every step: q, block_table, seq_lens (and sinks) in one pinned host "
                       "buffer copied to the device, out and lse read back in one copy; "
                       "double-buffered on two side streams so that a step's copies overlap "
                       "the neighbouring steps' kernels ('serial': all on one stream); the KV "
                       "cache is resident device state"}

    bits = fpd.fp8_paged_decode_check_status(wsp)
    assert bits == 0, f"device status {bits}"

    hbm, peak_src = measured_peaks()
    split_avg_ms = statistics.fmean(split_ms)
    achieved = kv_bytes / (split_avg_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": ncu_traffic(args.config, kv_bytes, plan, wl.q_len,
                                                  wl.kv_format),
                "kernel": f"fpd_split_kernel<{wl.D},{2 if wl.groups > 8 else 1}>",
                "algorithmic_bytes_per_launch": kv_bytes,
                "unit_bytes": f"2*D = {2 * wl.D} B per (attended token, KV head); "
                              f"{kv_bytes // (2 * wl.D)} units per launch",
                "kernel_avg_us": split_avg_ms * 1e3, "peak_source": peak_src,
                "kernel_timing": f"CUDA events around the split kernel on its stream, "
                                 f"{len(split_ms)} calls right after the timed region"}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        dt, kvb, nrows, thr = oracle_sample(wl, args.cpu_seconds)
        cpu = {"value": kvb / dt / 1e9, "unit": UNIT, "cores": thr, "kind": "oracle",
               "sample": f"{nrows} random (sequence, query token, head) rows of the workload, "
                         f"{kvb:.0f} KV bytes (each row's share of its sequence), "
                         f"{dt:.1f} s wall"}

    launches_per_step = 1 + (1 if plan["max_splits"] > 1 else 0)   # split (+ combine)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "dtype_detail": ("E4M3 KV" if not nvfp4 else
                             "NVFP4 KV (E2M1 x E4M3 block scale)") +
                            " converted exactly to f16; mma.sync f16 x f16 -> f32; "
                            "softmax and reductions in f32; bf16 output",
            "data": "synthetic",
            "config": {"workload": W.describe(args.config), "B": wl.B, "q_len": wl.q_len,
                       "kv_format": wl.kv_format,
                       "Hq": wl.Hq,
                       "Hkv": wl.Hkv, "D": wl.D, "block_tokens": wl.block_tokens,
                       "kv_bytes_per_call": kv_bytes, "parallelism": f"replicas x{ws}",
                       "l2": f"inputs larger than L2: {replicas} KV replicas rotated, "
                             f"{replicas * kv_bytes / 2**20:.0f} MiB read per rotation vs "
                             f"{l2 / 2**20:.0f} MiB L2",
                       "plan": plan},
            "us_per_call": ms_per_step * 1e3,
            "us_per_call_p10_p90_evented": [float(np.percentile(call_ms, 10) * 1e3),
                                            float(np.percentile(call_ms, 90) * 1e3)],
            "split_kernel_us": split_avg_ms * 1e3,
            "combine_kernel_us": statistics.fmean(combine_ms) * 1e3,
            "pct_of_peak": 100.0 * value / hbm,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step * K, "clocks": clocks, "parity_guard": guard,
            "graph_replay_cold_l2": graph,
        }
        return line
    return None


def run_cache_write(args):
    """FP8 KV-cache write: GB/s on a large batch, us on a decode-step batch (1 GPU)."""
    import numpy as np
    import torch
    import fp8_paged_decode_b200 as fpd
    from fp8_paged_decode_b200 import workloads as W
    c = W.CONFIGS[args.config]
    Hkv, D, bt = c["Hkv"], c["D"], c["block_tokens"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    hbm, peak_src = measured_peaks()
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    res = {}
    for name, T in (("prefill", args.write_tokens), ("decode_step", c["B"])):
        nb = 2 * ((T + bt - 1) // bt) + 8
        key = torch.randn((T, Hkv, D), generator=gen, device=dev).to(torch.bfloat16)
        value = torch.randn((T, Hkv, D), generator=gen, device=dev).to(torch.bfloat16)
        perm = torch.randperm(nb * bt, generator=gen, device=dev)[:T].to(torch.int64)
        kc = torch.zeros((nb, bt, Hkv, D), dtype=torch.uint8, device=dev)
        vc = torch.zeros_like(kc)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        bytes_per = T * Hkv * D * 6
        f = lambda: fpd.fp8_paged_decode_cache_write(key, value, perm, kc, vc, 0.02, 0.01,
                                                     status=status, stream=stream)
        for _ in range(args.warmup):
            f()
        torch.cuda.synchronize()
        K = max(3, min(args.steps, 2000))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        graph = None
        if name == "decode_step":   # small: replay a graph of 100 calls
            side = torch.cuda.Stream()
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=side):
                    for _ in range(100):
                        fpd.fp8_paged_decode_cache_write(key, value, perm, kc, vc, 0.02, 0.01,
                                                         status=status, stream=side)
            stream.wait_stream(side)
            K = max(1, K // 100)
            graph.replay()
        sampler = ClockSampler(0)
        sampler.start()
        time.sleep(0.25)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(K):
            if graph is not None:
                graph.replay()
            else:
                f()
        e1.record(stream)
        torch.cuda.synchronize()
        clocks = sampler.stop()
        if graph is not None:
            K *= 100
            del graph
        ms = e0.elapsed_time(e1) / K
        assert int(status.item()) == 0
        gbs = bytes_per / (ms / 1e3) / 1e9
        res[name] = {"tokens": T, "us_per_call": ms * 1e3, "bytes_per_call": bytes_per,
                     "GBps": gbs, "frac_of_peak": gbs / hbm, "calls": K, "clocks": clocks,
                     "l2": "bytes per call larger than L2 (126 MiB)" if bytes_per > 126 * 2**20
                           else "bytes per call smaller than L2 (latency case)"}
    line = {"metric": "FP8 KV-cache write HBM GB/s (bf16 K/V in, E4M3 pages out)",
            "value": res["prefill"]["GBps"], "unit": "GB/s", "n_gpus": 1,
            "steps": res["prefill"]["calls"], "warmup": args.warmup,
            "ms_per_step": res["prefill"]["us_per_call"] / 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16->e4m3 (f32 product)",
            "data": "synthetic",
            "config": {"workload": f"cache write, Hkv={Hkv} D={D} block_tokens={bt} "
                                   f"({args.config} shape), shuffled slots", "tokens": args.write_tokens},
            "roofline": {"bound": "hbm", "achieved": res["prefill"]["GBps"], "peak": hbm,
                         "unit": "GB/s", "frac": res["prefill"]["frac_of_peak"], "traffic": None,
                         "kernel": "fpd_cache_write_kernel", "peak_source": peak_src,
                         "unit_bytes": "6 B per element (bf16 K and V read, E4M3 written)"},
            "cases": res, "gpu_launches": res["prefill"]["calls"]}
    print(json.dumps(line))
    if args.json_out:
        with open(args.json_out, "w") as fo:
            json.dump(line, fo, indent=1)
    return 0


def run_cp(args):
    """Context-parallel decode of one workload over R ranks: each rank decodes
    its contiguous page share of every sequence into an f32 partial, the
    partials are all-gathered over NCCL, and each rank merges them.  Under
    torchrun (R = world size) every step runs all three, timed per step on
    each rank, max over ranks.  On one process the step of the rank with the
    most keys of an R-way partition is timed (its decode and the merge of R
    partials computed beforehand) and the exchange is not run.  L2 is evicted
    (a 1 GiB read) before each timed step, outside the timed events."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import fp8_paged_decode_b200 as fpd
    from fp8_paged_decode_b200 import cp
    from fp8_paged_decode_b200 import workloads as W

    ws, rank, local = dist_env()
    assert ws == args.gpus, f"--gpus {args.gpus} but WORLD_SIZE={ws}"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        dist.init_process_group("nccl", init_method="env://", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=120))
    R = ws if ws > 1 else args.cp_ranks
    if args.kv_format != "e4m3" or args.q_len != 1:
        raise SystemExit("--op cp: E4M3 pages and one query per sequence")
    wl = make_wl(args)
    if wl.window_left >= 0:
        raise SystemExit(f"--op cp: {args.config} has a sliding window, which context-parallel "
                         "decode does not take")
    B, Hq, D, bt = wl.B, wl.Hq, wl.D, wl.block_tokens
    q = torch.from_numpy(wl.q.view(np.int16)).view(torch.bfloat16).to(dev)
    kc = torch.from_numpy(wl.k_cache).to(dev)
    vc = torch.from_numpy(wl.v_cache).to(dev)
    sinks = None if wl.sinks is None else torch.from_numpy(wl.sinks).to(dev)
    shards = [cp.cp_shard(wl.block_table, wl.seq_lens, R, r, bt) for r in range(R)]
    keys = [int(l.astype(np.int64).sum()) for _, l in shards]
    me = rank if ws > 1 else int(np.argmax(keys))
    rows = B * Hq
    blk = cp.partial_block_floats(rows, D)
    partial = torch.zeros(blk, dtype=torch.float32, device=dev)
    gathered = torch.zeros((R, blk), dtype=torch.float32, device=dev)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    lib = fpd.load_library()
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    vp = ctypes.c_void_p

    def descriptor(table, lens, buf):
        """The f32 partial decode of one rank's keys into `buf`, as the C ABI's descriptor."""
        a = fpd.fpd_decode_args()
        a.q, a.q_dtype = q.data_ptr(), fpd.FPD_Q_BF16
        a.k_cache, a.v_cache = kc.data_ptr(), vc.data_ptr()
        a.kv_format, a.kv_layout = fpd.FPD_KV_E4M3, fpd.FPD_KV_NHD
        a.block_table, a.seq_lens = table.data_ptr(), lens.data_ptr()
        a.B, a.q_len, a.Hq, a.Hkv, a.D = B, 1, Hq, wl.Hkv, D
        a.num_blocks, a.block_tokens, a.max_blocks = wl.num_blocks, bt, table.shape[1]
        a.k_scale, a.v_scale, a.sm_scale = wl.k_scale, wl.v_scale, wl.sm_scale
        a.window_left, a.sinks = -1, None
        a.out, a.lse = buf.data_ptr(), buf.data_ptr() + rows * D * 4
        a.out_dtype = fpd.FPD_OUT_F32
        a.chunk_pages_override = args.chunk_pages
        return a

    dev_shards = [(torch.from_numpy(t).to(dev), torch.from_numpy(l).to(dev)) for t, l in shards]
    descs = [descriptor(*dev_shards[r], gathered[r]) for r in range(R)]
    mine = descriptor(*dev_shards[me], partial)
    need = max(fpd.fp8_paged_decode_workspace_bytes_args(d) for d in descs)
    assert need > 0
    wsp = torch.zeros(need, dtype=torch.uint8, device=dev)
    ws_ptr, ws_n = vp(wsp.data_ptr()), ctypes.c_size_t(wsp.numel())
    f_dec = lib.fp8_paged_decode_attention_args
    merge_args = (vp(gathered.data_ptr()), R, blk, rows, Hq, D,
                  vp(sinks.data_ptr()) if sinks is not None else None, vp(out.data_ptr()), 0,
                  vp(lse.data_ptr()), sh)
    if ws == 1:   # every rank's partial, once: the merge's input
        for d in descs:
            assert f_dec(ctypes.byref(d), ws_ptr, ws_n, sh) == 0
    mine_ref = ctypes.byref(mine)

    def step():
        st = f_dec(mine_ref, ws_ptr, ws_n, sh)
        if ws > 1:
            cp.cp_exchange(partial, None, gathered)
        st |= lib.fp8_paged_decode_cp_merge(*merge_args)
        assert st == 0

    if args.cp_fused:
        # the exchange fused into the decode: the rank's combine kernel stores
        # its rows into every rank's gather buffer and raises its flag there;
        # the merge waits for the R flags.  One process: the other ranks'
        # slots are filled once, and their flags are raised (a fill, before
        # the timed events) each step.
        ex = cp.CpExchange(B, Hq, D) if ws > 1 else cp.CpExchange.local(R, B, Hq, D)
        fused = []
        for r in range(R if ws == 1 else 1):
            rr = r if ws == 1 else rank
            a = descriptor(*dev_shards[rr], partial)
            a.out, a.lse = None, None
            fused.append(a)
        fstatus = torch.zeros(1, dtype=torch.int32, device=dev)
        fsh = ctypes.c_void_p(stream.cuda_stream)

        def set_fields(a, r):
            (a.cp_gather, a.cp_flags, a.cp_ranks, a.cp_rank, a.cp_epoch,
             a.cp_block_floats) = ex.publish_fields(r)

        # this rank's gather buffer and flags, per epoch parity
        views = {}
        for _ in range(2):
            ex.next_epoch()
            views[ex.epoch & 1] = (ex.gather(me), ex.flags(me))
            for r, a in enumerate(fused):
                set_fields(a, r if ws == 1 else rank)
            if ws == 1:   # every rank's slots of both buffers hold its partial
                for a in fused:
                    assert f_dec(ctypes.byref(a), ws_ptr, ws_n, fsh) == 0
        mine_f = fused[me] if ws == 1 else fused[0]
        mine_f_ref = ctypes.byref(mine_f)
        margs = [None, R, blk, rows, Hq, D,
                 ctypes.c_void_p(sinks.data_ptr()) if sinks is not None else None,
                 ctypes.c_void_p(out.data_ptr()), 0, ctypes.c_void_p(lse.data_ptr()),
                 None, None, ctypes.c_uint64(1_000_000_000), ctypes.c_void_p(fstatus.data_ptr()),
                 fsh]
        f_merge_wait = lib.fp8_paged_decode_cp_merge_wait

        def pre_step():   # untimed: a new epoch; one process: every rank's flag raised
            e = ex.next_epoch()
            set_fields(mine_f, me if ws == 1 else rank)
            g, fl = views[e & 1]
            margs[0], margs[10], margs[11] = (ctypes.c_void_p(g.data_ptr()),
                                              ctypes.c_void_p(fl.data_ptr()), ctypes.c_uint32(e))
            if ws == 1:
                fl.fill_(e)

        def step():
            st = f_dec(mine_f_ref, ws_ptr, ws_n, fsh)
            st |= f_merge_wait(*margs)
            assert st == 0
    else:
        def pre_step():
            pass

    # L2 is evicted by reading a 1 GiB buffer (a reduction), which leaves no
    # dirty lines whose write-back would compete with the timed reads
    flush_buf = torch.ones(1024 * 2 ** 20, dtype=torch.uint8, device=dev)   # the host stays ahead
    flush = lambda: torch.amax(flush_buf)
    K = max(1, min(args.steps, 2000))
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        pre_step()
        step()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.25)
    torch.cuda.synchronize()
    # the timed steps: two events around each step, L2 flushed before it
    pairs = [(ev(), ev()) for _ in range(K)]
    for e0, e1 in pairs:
        flush()
        pre_step()
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    total_ms = float(sum(e0.elapsed_time(e1) for e0, e1 in pairs))
    mx = max_over_ranks(total_ms, dev) if ws > 1 else total_ms
    ms = mx / K
    # breakdown (untimed for the line's value): the rank's decode alone, the merge alone
    dec = [(ev(), ev()) for _ in range(min(K, 200))]
    for e0, e1 in dec:
        flush()
        e0.record(stream)
        assert f_dec(mine_ref, ws_ptr, ws_n, sh) == 0
        e1.record(stream)
    fused_alone = {}
    if args.cp_fused:
        assert int(fstatus.item()) == 0, "a rank's flag did not arrive"
        # the publishing decode alone, then the waiting merge alone (flags set)
        pub = [(ev(), ev()) for _ in range(min(K, 200))]
        for e0, e1 in pub:
            flush()
            pre_step()
            e0.record(stream)
            assert f_dec(mine_f_ref, ws_ptr, ws_n, fsh) == 0
            e1.record(stream)
        mw = [(ev(), ev()) for _ in range(min(K, 200))]
        for e0, e1 in mw:
            flush()
            e0.record(stream)
            assert f_merge_wait(*margs) == 0
            e1.record(stream)
        torch.cuda.synchronize()
        fused_alone = {
            "publishing_decode_median_cold_l2": float(np.median([a.elapsed_time(b) for a, b in pub])) * 1e3,
            "waiting_merge_median_cold_l2": float(np.median([a.elapsed_time(b) for a, b in mw])) * 1e3}
        ex.close()
    # the merge alone: a CUDA graph of 100 launches, replayed 10 times
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    side_args = merge_args[:-1] + (ctypes.c_void_p(side.cuda_stream),)
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for _ in range(100):
                lib.fp8_paged_decode_cp_merge(*side_args)
    stream.wait_stream(side)
    graph.replay()
    m0, m1 = ev(), ev()
    m0.record(stream)
    for _ in range(10):
        graph.replay()
    m1.record(stream)
    torch.cuda.synchronize()
    del graph
    dec_ms = float(np.median([e0.elapsed_time(e1) for e0, e1 in dec]))
    merge_ms = m0.elapsed_time(m1) / 1000
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    row_kv = wl.Hkv * D * 2   # K and V bytes of one token
    all_bytes = int(wl.seq_lens.astype(np.int64).sum()) * row_kv
    my_bytes = keys[me] * row_kv
    gbs = all_bytes / (ms / 1e3) / 1e9
    hbm, peak_src = measured_peaks()
    line = {
        "metric": "context-parallel decode: KV GB/s over all ranks' keys per step; us/step",
        "value": gbs, "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms, "us_per_step": ms * 1e3, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "cp_ranks": R,
        "exchange": (("fused: the combine kernel stores the rows into every rank's gather "
                      "buffer over peer memory and raises a flag; the merge waits for the flags"
                      + ("" if ws > 1 else " (one GPU: the other ranks' slots and flags are "
                         "set outside the timed step)")) if args.cp_fused else
                     "nccl all_gather_into_tensor of the f32 partials" if ws > 1 else
                     "not run: one GPU; the timed step is one rank's decode and merge"),
        "us_alone": {"partial_decode_median_cold_l2": dec_ms * 1e3,
                     "merge_graph_replay": merge_ms * 1e3, **fused_alone},
        "rank_kv_bytes": my_bytes, "all_kv_bytes": all_bytes,
        "partial_decode_frac_of_peak": my_bytes / (dec_ms / 1e3) / 1e9 / hbm,
        "peak_source": peak_src,
        "exchange_bytes_per_rank": blk * 4,
        "config": {"workload": f"{W.describe(args.config)}; keys split into {R} "
                               "contiguous page runs per sequence",
                   "l2": "evicted (a 1 GiB read) before each timed step"},
        "clocks": clocks,
        "gpu_launches": K * 3,   # split, combine and merge kernels per step
    }
    print(json.dumps(line))
    if args.json_out:
        with open(args.json_out, "w") as fo:
            json.dump(line, fo, indent=1)
    return 0


def main():
    args = parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.op == "cache_write":
        return run_cache_write(args)
    if args.op == "cp":
        return run_cp(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
