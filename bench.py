#!/usr/bin/env python
"""Throughput of Jet-Long dynamic bifocal RoPE attention on B200.

One step = the whole hot path on its headline workloads:
  * one prefill of the 128K workload (B=1, Hq=32, Hkv=8, d=128, L=131072,
    w_pretrained=32768 so G=4, w0=4096, rope_theta=1e6, bf16), and
  * one full pass of the decode workload (B=8, Hq=32, Hkv=8, d=128, raw-K/V
    cache of 131136 rows, 64 single-token steps at L = 131041..131104, so G
    goes 4 -> 5 inside the pass).
value = prefill TFLOP/s on computed FLOPs (whole job: all ranks' FLOPs / max
rank time).  The decode figures (GB/s of K/V streamed, tokens/s) ride along in
"decode".  Inputs are larger than L2 (q alone is 1 GiB, the caches 4.3 GB), so
no explicit flush is done between steps.

--impl reference times the fp64 CPU oracle (the only reference this method has
here) on a bounded sample of the same workload.
Multi-GPU: replicas only (each rank runs the same independent workload), weak
scaling, no data-path collective.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from rope_context_extension_jet_b200 import inputs as I  # noqa: E402

METRIC = "bifocal prefill TFLOP/s & % bf16 peak at L=128K; decode HBM GB/s"
BM = BN = 128  # tile shape used to count computed FLOPs
E2E_CHUNKS = 16  # query chunks of the end-to-end host-buffer prefill


def tile_counts(L, w0, bm=BM, bn=BN, P=0):
    """(causal tiles, band tiles) of the (query-block, key-block) grid; query rows
    are positions [P, L) (P = 0: the whole sequence)."""
    nqb = (L - P + bm - 1) // bm
    tiles = band = 0
    for qb in range(nqb):
        i_lo, i_hi = P + qb * bm, min(P + qb * bm + bm - 1, L - 1)
        nkb = i_hi // bn + 1
        tiles += nkb
        for kb in range(nkb):
            j_lo, j_hi = kb * bn, kb * bn + bn - 1
            dmax, dmin = i_hi - j_lo, max(0, i_lo - j_hi)
            if dmin < w0 <= dmax:
                band += 1
    return tiles, band


def prefill_flops(w, P=0):
    """(useful, computed) FLOPs of the query rows [P, L) of workload w."""
    useful = 4.0 * w.d * w.Hq * w.B * (w.L * (w.L + 1) / 2 - P * (P + 1) / 2)
    tiles, band = tile_counts(w.L, min(w.w0, w.L), P=P)
    computed = w.B * w.Hq * (tiles * 4.0 * w.d * BM * BN + band * 2.0 * w.d * BM * BN)
    return useful, computed, tiles, band


def decode_bytes(w, L):
    el = 2 if w.dtype == "bf16" else 4
    kv = 2.0 * w.B * w.Hkv * L * w.d * el
    qo = 2.0 * w.B * w.Hq * w.d * el
    return kv, kv + qo


PREFILL_KERNEL = "prefill_pair_kernel"
# sources the timed prefill kernel is compiled from (its DRAM counters are
# reported only while they hash to the value recorded with the capture)
PREFILL_SOURCES = ("prefill_pair.cu", "prefill_tc_common.cuh", "tc_ptx.cuh", "jl_ptx.cuh", "jl_common.cuh")


DECODE_SOURCES = ("decode.cu", "jl_ptx.cuh", "jl_common.cuh")


def prefill_source_hash(names=PREFILL_SOURCES):
    import hashlib
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "rope_context_extension_jet_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def prefill_traffic():
    """DRAM bytes per 128K prefill launch from the committed ncu capture, or None
    when the kernel sources changed since the counters were taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[PREFILL_KERNEL]
        if prefill_source_hash() != rec["source_sha256"]:
            return None
        return rec["dram_bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        return None


# dense bf16 tensor-core FLOPs per SM per clock (tcgen05: one 128x128x16 MMA
# per 64 cycles per SM = 8192 FLOP/cycle) and the SM count of a B200
TENSOR_FLOP_PER_CLK_SM = 8192
B200_SMS = 148


def _find_mhz(d, want):
    """First numeric value under a key that names an SM clock in MHz and contains
    `want` (the peaks file's layout is the driver's; search it instead of assuming)."""
    if isinstance(d, dict):
        for k, v in d.items():
            kl = str(k).lower()
            if isinstance(v, (int, float)) and "mhz" in kl and "mem" not in kl and want in kl:
                return float(v)
        for v in d.values():
            r = _find_mhz(v, want)
            if r is not None:
                return r
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "bf16_sustained_sm_mhz": _find_mhz(d, "sustain"),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "bf16_sustained_sm_mhz": 1300.0, "source": "fallback"}


def per_clock(tflops, sm_mhz, peaks):
    """Clock-normalised view of a tensor-core rate: TFLOP/s per GHz of SM clock
    beside the same figure for the measured cuBLAS peak, and the fraction of the
    tensor pipe's nominal 8192 FLOP/cycle/SM at the clock the kernel ran at."""
    if not sm_mhz:
        return None
    r = {"sm_mhz": sm_mhz, "tflops_per_ghz": round(tflops / (sm_mhz / 1e3), 2),
         "frac_of_tensor_pipe_at_this_clock": round(
             tflops * 1e12 / (B200_SMS * TENSOR_FLOP_PER_CLK_SM * sm_mhz * 1e6), 4)}
    if peaks.get("bf16_sustained_sm_mhz"):
        pk = peaks["bf16_tflops_sustained"] / (peaks["bf16_sustained_sm_mhz"] / 1e3)
        r["sustained_peak_tflops_per_ghz"] = round(pk, 2)
        r["frac_of_sustained_peak_per_clock"] = round(r["tflops_per_ghz"] / pk, 4)
    return r


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = str(gpu_index)
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def to_dev(a, dev):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(a).to(dev)


def to_pinned(a):
    import torch
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    t = t.pin_memory()
    return t.view(torch.bfloat16) if a.dtype == np.uint16 else t


def oracle_prefill_sample(w, budget_s=20.0, nthreads=0, seed=77, inputs=None):
    """Time the fp64 oracle on seeded random query rows (head, position) of the
    prefill workload: calls of a fixed number of rows (64 per host thread) until
    about budget_s seconds of work.  Both the repo arm's cpu_baseline leg and the
    --impl reference arm sample the oracle through this function, so the two
    report the same quantity."""
    import oracle
    q, k, v = inputs if inputs is not None else I.prefill_inputs(w)
    rng = np.random.default_rng(seed)
    cores = nthreads or os.cpu_count()
    batch = 64 * max(1, cores)
    done_rows = 0
    flops = 0.0
    t_total = 0.0
    while done_rows == 0 or t_total < budget_s:
        h = rng.integers(0, w.Hq, size=batch)
        i = rng.integers(0, w.L, size=batch)
        rows = np.stack([np.zeros(batch, np.int64), h, i], axis=1)
        t0 = time.perf_counter()
        oracle.prefill_rows(q, k, v, rows, w0=w.w0, w_pretrained=w.w_pretrained,
                            rope_theta=w.rope_theta, scale=w.scale, nthreads=nthreads)
        t_total += time.perf_counter() - t0
        done_rows += batch
        flops += float(np.sum(4.0 * w.d * (i + 1)))
    return {"value": flops / t_total / 1e12, "unit": "TFLOP/s", "cores": int(cores),
            "kind": "oracle", "seconds": round(t_total, 2), "rows": done_rows,
            "sample": f"{done_rows} random query rows (head, position) of the 128K prefill in calls "
                      f"of {batch} rows, fp64, useful FLOPs 4*d*(i+1) per row"}


def bench_config(wp, wd, world):
    """The `config` object of the JSON line (identical for both arms)."""
    return {"workload": wp.name, "B": wp.B, "Hq": wp.Hq, "Hkv": wp.Hkv, "d": wp.d, "L": wp.L,
            "w_pretrained": wp.w_pretrained, "G": max(1, -(-wp.L // wp.w_pretrained)),
            "w0": wp.w0, "rope_theta": wp.rope_theta, "decode_workload": wd.name,
            "parallelism": f"replicas x{world}", "l2": "inputs larger than L2 (no flush)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = I.C4
    steps = []
    per = min(20.0, max(2.0, 90.0 / max(1, args.steps + args.warmup)))
    inputs = I.prefill_inputs(w)
    for s in range(args.warmup + args.steps):
        r = oracle_prefill_sample(w, budget_s=per, seed=77 + s, inputs=inputs)
        if s >= args.warmup:
            steps.append(r)
    secs = float(np.sum([r["seconds"] for r in steps]))
    rows = int(np.sum([r["rows"] for r in steps]))
    val = float(np.sum([r["value"] * r["seconds"] for r in steps]) / secs)
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs * 1000.0 / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, I.D, world),
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": steps[0]["cores"],
                         "kind": "oracle",
                         "sample": f"{rows} random query rows (head, position) of the 128K prefill over "
                                   f"{args.steps} timed steps (each: {steps[0]['sample']})"},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def max_across_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank scalar over all ranks (the multi-GPU timing rule: a
    replica job takes as long as its slowest rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput of `world` replicas: all ranks' work / slowest rank's time."""
    return world * work_per_rank / max_seconds


def run_profile(args):
    """One kernel on a reduced workload of the same shape family, for ncu."""
    import torch
    import rope_context_extension_jet_b200 as jl
    jl.load_library()
    torch.cuda.set_device(0)
    if args.profile == "prefill":
        w = I.C4.with_(L=args.L)
        q, k, v = (to_dev(a, "cuda") for a in I.prefill_inputs(w))
        out = torch.empty_like(q)
        for _ in range(args.warmup + args.steps):
            jl.prefill(q, k, v, out, w0=w.w0, w_pretrained=w.w_pretrained,
                       rope_theta=w.rope_theta, scale=w.scale)
    else:
        w = I.D.with_(L0=args.L - 1, Lcap=args.L + 64, steps=1)
        qs, kc, vc = I.decode_inputs(w)
        qd, kcd, vcd = to_dev(np.ascontiguousarray(qs[0]), "cuda"), to_dev(kc, "cuda"), to_dev(vc, "cuda")
        ws = torch.empty(jl.decode_workspace_size(w.B, w.Hq, w.Hkv, w.Lcap, w.d), dtype=torch.uint8,
                         device="cuda")
        for _ in range(args.warmup + args.steps):
            jl.decode(qd, kcd, vcd, w.length_at(0), w0=w.w0, w_pretrained=w.w_pretrained,
                      rope_theta=w.rope_theta, scale=w.scale, workspace=ws)
    jl.device_status()
    print(json.dumps({"profile": args.profile, "L": args.L, "launches": jl.launch_count()}))


# ---------------------------------------------------------------- ncu harness
# Counters read for one kernel launch (a few replay passes; run on the reduced
# --profile workloads only).
NCU_METRICS = (
    "gpu__time_duration.sum",
    "sm__cycles_elapsed.avg.per_second",
    "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active",
    "smsp__issue_active.avg.pct_of_peak_sustained_active",
    "sm__inst_executed_pipe_xu.avg.pct_of_peak_sustained_active",
    "sm__warps_active.avg.pct_of_peak_sustained_active",
    "dram__bytes_read.sum",
    "dram__bytes_write.sum",
    "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed",
    "launch__registers_per_thread",
    "smsp__inst_executed.sum",
)
NCU_KERNELS = {"prefill": "prefill_pair_kernel", "decode": "decode_tc_kernel"}


def parse_ncu_csv(text):
    """Rows of ncu's --csv metric output as dicts {kernel, id, metric, unit, value}."""
    import csv
    import io
    lines = [ln for ln in text.splitlines() if ln.startswith('"')]
    rows = []
    for r in csv.DictReader(io.StringIO("\n".join(lines))):
        try:
            val = float(r["Metric Value"].replace(",", ""))
        except (KeyError, ValueError):
            continue
        rows.append({"kernel": r.get("Kernel Name", ""), "id": int(r.get("ID", 0)),
                     "metric": r["Metric Name"], "unit": r.get("Metric Unit", ""), "value": val})
    return rows


# Counters kept from a --set full capture (the rest of its ~1000 stay in the
# .csv under gpurun_out/)
NCU_FULL_SHOWN = (
    "gpu__time_duration.sum", "sm__cycles_elapsed.avg.per_second", "dram__bytes_read.sum",
    "dram__bytes_write.sum", "dram__cycles_active.avg.pct_of_peak_sustained_elapsed",
    "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed",
    "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active",
    "sm__inst_executed_pipe_xu.avg.pct_of_peak_sustained_active",
    "sm__inst_executed_pipe_fma.avg.pct_of_peak_sustained_active",
    "sm__inst_executed_pipe_alu.avg.pct_of_peak_sustained_active",
    "sm__inst_executed_pipe_lsu.avg.pct_of_peak_sustained_active",
    "smsp__issue_active.avg.pct_of_peak_sustained_active", "sm__warps_active.avg.pct_of_peak_sustained_active",
    "smsp__inst_executed.sum", "launch__registers_per_thread", "launch__grid_size", "launch__cluster_dim_x",
    "smsp__average_warps_issue_stalled_long_scoreboard_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_wait_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_barrier_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_short_scoreboard_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_math_pipe_throttle_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_mio_throttle_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_lg_throttle_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_no_instruction_per_issue_active.ratio",
    "smsp__average_warps_issue_stalled_branch_resolving_per_issue_active.ratio",
    "l1tex__data_pipe_lsu_wavefronts_mem_shared.sum",
)


def parse_ncu_raw_csv(text):
    """ncu --page raw --csv output (one header row of metric names, one row of
    units, one row per kernel) as the same dicts as parse_ncu_csv."""
    import csv
    import io
    lines = [ln for ln in text.splitlines() if ln.startswith('"')]
    recs = list(csv.reader(io.StringIO("\n".join(lines))))
    if len(recs) < 3:
        return []
    head, units = recs[0], recs[1]
    rows = []
    for rec in recs[2:]:
        kname = rec[head.index("Kernel Name")] if "Kernel Name" in head else ""
        for name, unit, val in zip(head, units, rec):
            try:
                v = float(val.replace(",", ""))
            except ValueError:
                continue
            rows.append({"kernel": kname, "id": 0, "metric": name, "unit": unit, "value": v})
    return rows


def launch_summary(rows):
    """Per kernel (name up to its template arguments): launches, total ms, share
    of the summed device time, from gpu__time_duration.sum rows (ns)."""
    per = {}
    for r in rows:
        if r["metric"] != "gpu__time_duration.sum":
            continue
        name = r["kernel"].split("(")[0].strip()
        n, t = per.get(name, (0, 0.0))
        per[name] = (n + 1, t + r["value"] * 1e-6)
    total = sum(t for _, t in per.values()) or 1.0
    return sorted(((k, n, t, t / total) for k, (n, t) in per.items()), key=lambda x: -x[2])


def _ncu_cmd(extra, bench_args, log):
    return (["ncu", "--clock-control", "none", "--print-units", "base", "--csv", "--log-file", log] + extra
            + [sys.executable, os.path.join(ROOT, "bench.py")] + bench_args)


# Every capture profiles/ holds, in the order they run: (mode, L).
NCU_ALL = (("launches", None), ("traffic", 131072), ("prefill", 32768), ("decode", 32768),
           ("prefill-full", 32768), ("decode-full", 32768))


def ncu_summary_name(mode, L):
    """File name (without extension) under profiles/ of the capture `mode` at length L."""
    if mode == "launches":
        return "launches_bench"
    kname = NCU_KERNELS["decode" if mode.startswith("decode") else "prefill"]
    if mode == "traffic":
        return f"{kname}_L{L}_dram"
    if mode.endswith("-full"):
        return f"{kname}_L{L}_full"
    return f"{kname}_L{L}_counters"


def run_ncu_all():
    """Regenerate every summary under profiles/: each capture in its own process
    (each runs its command plainly first, then under ncu); stops at the first
    that fails."""
    for mode, L in NCU_ALL:
        cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--ncu", mode]
        if L is not None:
            cmd += ["--L", str(L)]
        r = subprocess.run(cmd)
        if r.returncode != 0:
            raise SystemExit(f"capture {mode} exited {r.returncode}")


def run_ncu(args):
    """Profiling harness: run the bench command once without ncu (it must exit 0),
    then the same command under ncu, and write the summary under profiles/."""
    out_dir = os.path.join(ROOT, "gpurun_out")
    os.makedirs(out_dir, exist_ok=True)
    peaks = load_peaks()
    if args.ncu == "launches":
        bench_args = ["--steps", str(args.steps), "--warmup", str(args.warmup), "--no-cpu-baseline"]
        extra = ["--metrics", "gpu__time_duration.sum"]
    elif args.ncu in ("prefill-full", "decode-full"):
        which = args.ncu.split("-")[0]
        bench_args = ["--profile", which, "--L", str(args.L), "--steps", "1", "--warmup", "1"]
        extra = ["--set", "full", "--page", "raw", "-k", "regex:" + NCU_KERNELS[which], "-s", "1", "-c", "1"]
    elif args.ncu == "traffic":
        bench_args = ["--profile", "prefill", "--L", str(args.L), "--steps", "1", "--warmup", "1"]
        extra = ["--metrics", "gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum",
                 "-k", "regex:" + NCU_KERNELS["prefill"], "-s", "1", "-c", "1"]
    else:
        bench_args = ["--profile", args.ncu, "--L", str(args.L), "--steps", "1", "--warmup", "1"]
        extra = ["--metrics", ",".join(NCU_METRICS), "-k", "regex:" + NCU_KERNELS[args.ncu], "-s", "1", "-c", "1"]
    plain = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + bench_args,
                           capture_output=True, text=True)
    if plain.returncode != 0:
        print(plain.stdout[-2000:], plain.stderr[-2000:])
        raise SystemExit(f"plain run exited {plain.returncode}; not profiling")
    log = os.path.join(out_dir, f"ncu_{args.ncu}.csv")
    cmd = _ncu_cmd(extra, bench_args, log)
    t0 = time.time()
    r = subprocess.run(cmd, capture_output=True, text=True)
    secs = time.time() - t0
    if r.returncode != 0:
        print(r.stdout[-2000:], r.stderr[-2000:])
        raise SystemExit(f"ncu exited {r.returncode}")
    text = open(log).read()
    rows = parse_ncu_raw_csv(text) if args.ncu.endswith("-full") else parse_ncu_csv(text)
    import shlex
    shown = shlex.join(["python" if c == sys.executable else c for c in cmd]).replace(os.path.join(ROOT, ""), "")
    lines = []
    if args.ncu == "launches":
        summ = launch_summary(rows)
        lines += [f"# Launch list: `python bench.py {' '.join(bench_args)}`", "",
                  "Every launch of the bench command with its device time (ncu, one pass, serialised and",
                  "cold-cache: compare shares, not absolute times).", "", "Command (run after the same bench",
                  "command exited 0 without ncu):", "", "    " + shown, "",
                  "| kernel | launches | total ms | share |", "|---|---|---|---|"]
        lines += [f"| `{k}` | {n} | {t:.3f} | {sh:.1%} |" for k, n, t, sh in summ]
        rec = {"launches": [{"kernel": k, "launches": n, "total_ms": round(t, 4), "share": round(sh, 4)}
                            for k, n, t, sh in summ]}
        name = ncu_summary_name("launches", None)
    else:
        m = {r["metric"]: r["value"] for r in rows}
        if args.ncu.endswith("-full"):
            m = {k: v for k, v in m.items() if any(k.startswith(w) for w in NCU_FULL_SHOWN)}
        dur = m.get("gpu__time_duration.sum", float("nan")) * 1e-9
        dram = m.get("dram__bytes_read.sum", 0.0) + m.get("dram__bytes_write.sum", 0.0)
        rec = {"metrics": m, "seconds": dur, "dram_bytes": dram}
        if args.ncu in ("prefill", "traffic", "prefill-full"):
            w = I.C4.with_(L=args.L)
            useful, computed, _, _ = prefill_flops(w)
            rec.update({"workload": f"prefill bf16 B=1 Hq=32 Hkv=8 d=128 L={args.L} G={max(1, -(-args.L // w.w_pretrained))} "
                                    f"w0={w.w0}", "flops_computed": computed,
                        "tflops": computed / dur / 1e12 if dur > 0 else None})
            rec["frac_of_bf16_burst"] = rec["tflops"] / peaks["bf16_tflops"] if rec["tflops"] else None
            kname = NCU_KERNELS["prefill"]
        else:
            w = I.D.with_(L0=args.L - 1, Lcap=args.L + 64, steps=1)
            kv, allb = decode_bytes(w, args.L)
            rec.update({"workload": f"decode bf16 B=8 Hq=32 Hkv=8 d=128 L={args.L}", "kv_bytes": kv,
                        "gbs_kv": kv / dur / 1e9 if dur > 0 else None})
            rec["frac_of_hbm"] = rec["gbs_kv"] / peaks["hbm_gbs"] if rec["gbs_kv"] else None
            kname = NCU_KERNELS["decode"]
        rec["peaks"] = {k: v for k, v in peaks.items()}
        name = ncu_summary_name(args.ncu, args.L)
        lines += [f"# `{kname}`: {rec['workload']}", "", "One launch after one warm-up launch (ncu, clock control none),",
                  "captured after the same command exited 0 without ncu:", "", "    " + shown, "",
                  "| metric | value |", "|---|---|"]
        lines += [f"| `{k}` | {v:.6g} |" for k, v in m.items()]
        if "tflops" in rec:
            lines += ["", f"Computed FLOPs {rec['flops_computed']:.4e} over {dur * 1e3:.3f} ms = "
                          f"{rec['tflops']:.1f} TFLOP/s, {rec['frac_of_bf16_burst']:.3f} of the {peaks['source']} "
                          f"bf16 burst peak ({peaks['bf16_tflops']} TFLOP/s); DRAM {dram / 1e9:.3f} GB "
                          f"({dram / dur / 1e9:.0f} GB/s)."]
        else:
            lines += ["", f"K/V bytes {rec['kv_bytes']:.4e} over {dur * 1e3:.3f} ms = {rec['gbs_kv']:.0f} GB/s, "
                          f"{rec['frac_of_hbm']:.3f} of the {peaks['source']} HBM copy bandwidth "
                          f"({peaks['hbm_gbs']} GB/s); DRAM counted {dram / 1e9:.3f} GB."]
    srcs = DECODE_SOURCES if args.ncu.startswith("decode") else PREFILL_SOURCES
    if args.ncu == "launches":
        srcs = PREFILL_SOURCES + ("decode.cu", "range_scan.cu", "rope_keys.cu")
    lines += ["", f"Sources: sha256 of {', '.join(srcs)}: {prefill_source_hash(srcs)[:16]}; "
                  f"capture took {secs:.0f} s."]
    prof = os.path.join(ROOT, "profiles")
    with open(os.path.join(prof, name + ".md"), "w") as f:
        f.write("\n".join(lines) + "\n")
    rec["command"] = shown
    rec["sources"] = {"files": list(srcs), "sha256": prefill_source_hash(srcs)}
    with open(os.path.join(prof, name + ".json"), "w") as f:
        json.dump(rec, f, indent=1, sort_keys=True)
    if args.ncu == "traffic" and args.L == I.C4.L:
        tr_path = os.path.join(prof, "traffic.json")
        try:
            tr = json.load(open(tr_path))
        except (OSError, ValueError):
            tr = {}
        tr[PREFILL_KERNEL] = {"dram_bytes_per_launch": dram, "source_sha256": prefill_source_hash(),
                              "workload": rec["workload"], "command": shown}
        with open(tr_path, "w") as f:
            json.dump(tr, f, indent=1)
    print(json.dumps({"ncu": args.ncu, "summary": os.path.join("profiles", name + ".md"),
                      "seconds": round(secs, 1)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--profile", choices=["prefill", "decode"], default=None,
                    help="run only one kernel on a reduced workload (for ncu captures)")
    ap.add_argument("--L", type=int, default=32768, help="sequence / cache length for --profile")
    ap.add_argument("--ncu", choices=["launches", "prefill", "decode", "traffic", "prefill-full", "decode-full",
                                      "all"],
                    default=None,
                    help="profiling harness: the bench command (launches), one kernel of the --profile "
                         "workloads (prefill, decode) or one full-size prefill's DRAM bytes (traffic, "
                         "--L 131072), under ncu; writes the summary (.md) and its figures (.json) under "
                         "profiles/; 'all' runs every capture profiles/ holds, one after the other")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.ncu == "all":
        run_ncu_all()
        return
    if args.ncu:
        run_ncu(args)
        return
    if args.profile:
        run_profile(args)
        return

    import torch
    import torch.distributed as dist
    import rope_context_extension_jet_b200 as jl

    jl.load_library()  # fails loudly without the built library
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return max_across_ranks(x, world, dev)

    peaks = load_peaks()
    wp, wd = I.C4, I.D
    stream = torch.cuda.current_stream(dev)

    # ---------------- inputs (host, seeded), then resident in HBM
    q, k, v = I.prefill_inputs(wp)
    qd, kd, vd = to_dev(q, dev), to_dev(k, dev), to_dev(v, dev)
    outd = torch.empty_like(qd)
    dq, dkc, dvc = I.decode_inputs(wd)
    dqd, dkcd, dvcd = to_dev(dq, dev), to_dev(dkc, dev), to_dev(dvc, dev)
    del dkc, dvc
    dout = torch.empty_like(dqd[0])
    ws = torch.empty(jl.decode_workspace_size(wd.B, wd.Hq, wd.Hkv, wd.Lcap, wd.d),
                     dtype=torch.uint8, device=dev)

    def prefill_call():
        jl.prefill(qd, kd, vd, outd, w0=wp.w0, w_pretrained=wp.w_pretrained,
                   rope_theta=wp.rope_theta, scale=wp.scale, stream=stream)

    def decode_call(t):
        jl.decode(dqd[t], dkcd, dvcd, wd.length_at(t), dout, w0=wd.w0,
                  w_pretrained=wd.w_pretrained, rope_theta=wd.rope_theta, scale=wd.scale,
                  workspace=ws, stream=stream)

    for _ in range(args.warmup):
        prefill_call()
        for t in range(wd.steps):
            decode_call(t)
    jl.device_status(stream)

    # ---------------- timed region (device time, CUDA events on the launching stream)
    sampler = ClockSampler(local)
    ev_p = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    ev_d = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    launches0 = jl.launch_count()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        ev_p[s][0].record(stream)
        prefill_call()
        ev_p[s][1].record(stream)
        ev_d[s][0].record(stream)
        for t in range(wd.steps):
            decode_call(t)
        ev_d[s][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    launches = jl.launch_count() - launches0
    barrier()
    clocks = sampler.stop()
    jl.device_status(stream)

    total_ms = max_over_ranks(t_start.elapsed_time(t_end))
    pre_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ev_p])))
    dec_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ev_d])))

    useful, computed, tiles, band = prefill_flops(wp)
    pre_tflops = whole_job_rate(computed, world, pre_ms * 1e-3) / 1e12
    pre_useful_tflops = whole_job_rate(useful, world, pre_ms * 1e-3) / 1e12
    kv_bytes = sum(decode_bytes(wd, wd.length_at(t))[0] for t in range(wd.steps))
    all_bytes = sum(decode_bytes(wd, wd.length_at(t))[1] for t in range(wd.steps))
    dec_gbs = whole_job_rate(kv_bytes, world, dec_ms * 1e-3) / 1e9
    dec_tok_s = whole_job_rate(wd.B * wd.steps, world, dec_ms * 1e-3)

    # ---------------- the same kernel in plain-RoPE mode (w0 >= L: every pair
    # local, one phase, no band tiles), outside the timed region: the cost of
    # the bifocal routing against plain RoPE attention on the same inputs
    wplain = wp.with_(w0=wp.L)

    def plain_call():
        jl.prefill(qd, kd, vd, outd, w0=wplain.w0, w_pretrained=wplain.w_pretrained,
                   rope_theta=wplain.rope_theta, scale=wplain.scale, stream=stream)

    plain_call()
    pl_ev = []
    for _ in range(2):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        plain_call()
        b.record(stream)
        pl_ev.append((a, b))
    torch.cuda.synchronize(dev)
    jl.device_status(stream)
    plain_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in pl_ev])))
    _, plain_computed, _, _ = prefill_flops(wplain)

    # ---------------- the other configurations (PR1 fp32, C2 G = 1, C3 G = 2 with
    # outlier keys): the same kernels on their shapes, outside the timed region
    other = {}
    for wo in (I.PR1, I.C2, I.C3):
        qo, ko, vo = (to_dev(a, dev) for a in I.prefill_inputs(wo))
        oo = torch.empty_like(qo)

        def other_call():
            jl.prefill(qo, ko, vo, oo, w0=wo.w0, w_pretrained=wo.w_pretrained, rope_theta=wo.rope_theta,
                       scale=wo.scale, stream=stream)

        other_call()
        ev_o = []
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            other_call()
            b.record(stream)
            ev_o.append((a, b))
        torch.cuda.synchronize(dev)
        jl.device_status(stream)
        ms_o = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ev_o])))
        u_o, c_o, _, _ = prefill_flops(wo)
        other[wo.name] = {"ms": round(ms_o, 4), "dtype": wo.dtype,
                          "tflops_computed": round(whole_job_rate(c_o, world, ms_o * 1e-3) / 1e12, 2),
                          "tflops_useful": round(whole_job_rate(u_o, world, ms_o * 1e-3) / 1e12, 2),
                          "tokens_per_s": round(world * wo.B * wo.L / (ms_o * 1e-3), 1)}
        del qo, ko, vo, oo

    # ---------------- the pages' three-pass inclusion-exclusion form of the same
    # prefill (jetlong_prefill_ie), outside the timed region: one pass against three
    ie_ws = torch.empty(int(jl.load_library().jetlong_prefill_ie_workspace_size(wp.B, wp.Hq, wp.L, wp.d, 0)),
                        dtype=torch.uint8, device=dev)

    def ie_call():
        jl.prefill_ie(qd, kd, vd, outd, w0=wp.w0, w_pretrained=wp.w_pretrained, rope_theta=wp.rope_theta,
                      scale=wp.scale, workspace=ie_ws, stream=stream)

    ie_call()
    ie_ev = []
    for _ in range(2):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ie_call()
        b.record(stream)
        ie_ev.append((a, b))
    torch.cuda.synchronize(dev)
    jl.device_status(stream)
    ie_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ie_ev])))
    del ie_ws

    # ---------------- chunked prefill (jetlong_prefill_chunk): the last 8192 rows
    # of the same 128K sequence as one chunk over the resident K/V, outside the
    # timed region
    P_ch = wp.L - 8192
    q_ch = qd[:, :, P_ch:].contiguous()
    out_ch = torch.empty_like(q_ch)

    def chunk_call():
        jl.prefill_chunk(q_ch, kd, vd, P_ch, out_ch, w0=wp.w0, w_pretrained=wp.w_pretrained,
                         rope_theta=wp.rope_theta, scale=wp.scale, stream=stream)

    chunk_call()
    ch_ev = []
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        chunk_call()
        b.record(stream)
        ch_ev.append((a, b))
    torch.cuda.synchronize(dev)
    jl.device_status(stream)
    ch_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ch_ev])))
    _, ch_computed, _, _ = prefill_flops(wp, P=P_ch)
    del q_ch, out_ch

    # ---------------- a serving-shaped variable-length batch (jetlong_prefill_varlen):
    # 64 sequences of seeded lengths in [512, 8192] (Hq=32, Hkv=8, d=128,
    # w_pretrained=2048 so G runs 1..4, w0=1024), one call, against one
    # jetlong_prefill per sequence on the same inputs; outside the timed region
    vl_lens = [int(x) for x in np.random.default_rng(6000).integers(512, 8193, size=64)]
    vl_max = max(vl_lens)
    gen = torch.Generator(device=dev).manual_seed(6001)
    vq = torch.randn((64, 32, vl_max, 128), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    vk = torch.randn((64, 8, vl_max, 128), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    vv = torch.randn((64, 8, vl_max, 128), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    vo = torch.empty_like(vq)
    vl_kw = dict(w0=1024, w_pretrained=2048, rope_theta=1e6, scale=1.0 / math.sqrt(128), stream=stream)

    def varlen_call():
        jl.prefill_varlen(vq, vk, vv, vl_lens, vo, **vl_kw)

    per_seq = [(vq[b:b + 1, :, :n].contiguous(), vk[b:b + 1, :, :n].contiguous(),
                vv[b:b + 1, :, :n].contiguous()) for b, n in enumerate(vl_lens)]

    def per_seq_call():
        for sq_, sk_, sv_ in per_seq:
            jl.prefill(sq_, sk_, sv_, **vl_kw)

    vl_res = {}
    for name, fn in (("one_call", varlen_call), ("one_prefill_per_sequence", per_seq_call)):
        fn()
        l0 = jl.launch_count()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b_.record(stream)
        torch.cuda.synchronize(dev)
        vl_res[name] = (max_over_ranks(a.elapsed_time(b_)), jl.launch_count() - l0)
    jl.device_status(stream)
    vl_flops = sum(prefill_flops(I.C4.with_(B=1, L=n, w_pretrained=2048, w0=1024))[1] for n in vl_lens)
    del vq, vk, vv, vo, per_seq

    # ---------------- decode over a standard RoPE cache (jetlong_decode_rope_cache),
    # one pass of the same 64 steps outside the timed region; the kernel's work
    # does not depend on the cached values, so the resident cache bytes serve
    def decode_rc_call(t):
        jl.decode_rope_cache(dqd[t], dkcd, dvcd, wd.length_at(t), dout, w0=wd.w0,
                             w_pretrained=wd.w_pretrained, rope_theta=wd.rope_theta,
                             scale=wd.scale, workspace=ws, stream=stream)

    for t in range(wd.steps):
        decode_rc_call(t)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for t in range(wd.steps):
        decode_rc_call(t)
    b.record(stream)
    torch.cuda.synchronize(dev)
    jl.device_status(stream)
    rc_ms = max_over_ranks(a.elapsed_time(b))
    rc_gbs = whole_job_rate(kv_bytes, world, rc_ms * 1e-3) / 1e9

    # ---------------- end to end through the public API with host buffers
    qh, kh, vh = to_pinned(q), to_pinned(k), to_pinned(v)
    outh = torch.empty(outd.shape, dtype=outd.dtype).pin_memory()
    e2e_ev = []
    for s in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        # the public host-buffer call: inputs in, prefill, output out, with the
        # transfers of one chunk overlapped with the compute of another
        jl.prefill_streamed(qh, kh, vh, outh, qd, kd, vd, outd, w0=wp.w0, w_pretrained=wp.w_pretrained,
                            rope_theta=wp.rope_theta, scale=wp.scale, nchunks=E2E_CHUNKS, stream=stream)
        b.record(stream)
        if s >= args.warmup:
            e2e_ev.append((a, b))
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in e2e_ev])))
    h2d = sum(x.numel() * x.element_size() for x in (qd, kd, vd))
    d2h = outd.numel() * outd.element_size()

    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = oracle_prefill_sample(wp, budget_s=args.cpu_budget, inputs=(q, k, v))
        frac_s = pre_tflops / world / peaks["bf16_tflops_sustained"]
        frac_b = pre_tflops / world / peaks["bf16_tflops"]
        line = {
            "metric": METRIC, "value": round(pre_tflops, 2), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) q/k/v, bf16)",
            "config": bench_config(wp, wd, world),
            "prefill": {"ms": round(pre_ms, 3), "tflops_computed": round(pre_tflops, 2),
                        "tflops_useful": round(pre_useful_tflops, 2),
                        "flops_computed": computed, "flops_useful": useful,
                        "tiles": tiles, "band_tiles": band,
                        "tokens_per_s": round(world * wp.B * wp.L / (pre_ms * 1e-3), 1),
                        "frac_of_burst_bf16": round(frac_b, 4),
                        "frac_of_sustained_bf16": round(frac_s, 4),
                        "chunk_last_8192_rows": {
                            "P": P_ch, "C": wp.L - P_ch, "ms": round(ch_ms, 3),
                            "tflops_computed": round(whole_job_rate(ch_computed, world, ch_ms * 1e-3) / 1e12, 2)},
                        "inclusion_exclusion_three_pass": {
                            "ms": round(ie_ms, 3), "three_pass_over_one_pass_time": round(ie_ms / pre_ms, 4)},
                        "plain_rope_same_kernel": {
                            "w0": wplain.w0, "ms": round(plain_ms, 3),
                            "tflops_computed": round(whole_job_rate(plain_computed, world, plain_ms * 1e-3) / 1e12, 2),
                            "bifocal_over_plain_time": round(pre_ms / plain_ms, 4)}},
            "other_prefill_configs": other,
            "varlen_batch": {
                "sequences": 64, "lengths": "seeded uniform in [512, 8192]", "tokens": int(sum(vl_lens)),
                "Hq": 32, "Hkv": 8, "d": 128, "w_pretrained": 2048, "w0": 1024,
                "flops_computed": vl_flops,
                "one_call": {"ms": round(vl_res["one_call"][0], 3), "launches": vl_res["one_call"][1],
                             "tflops_computed": round(world * vl_flops / (vl_res["one_call"][0] * 1e-3) / 1e12, 2),
                             "frac_of_burst_bf16": round(vl_flops / (vl_res["one_call"][0] * 1e-3) / 1e12
                                                         / peaks["bf16_tflops"], 4)},
                "one_prefill_per_sequence": {
                    "ms": round(vl_res["one_prefill_per_sequence"][0], 3),
                    "launches": vl_res["one_prefill_per_sequence"][1],
                    "tflops_computed": round(world * vl_flops / (vl_res["one_prefill_per_sequence"][0] * 1e-3) / 1e12,
                                             2)}},
            "decode": {"ms_per_token_step": round(dec_ms / wd.steps, 4),
                       "gbs_kv": round(dec_gbs, 1), "bytes_per_pass_kv": kv_bytes,
                       "bytes_per_pass_all": all_bytes, "tokens_per_s": round(dec_tok_s, 1),
                       "frac_of_hbm": round(dec_gbs / world / peaks["hbm_gbs"], 4),
                       "roofline": {"bound": "hbm", "achieved": round(dec_gbs / world, 1),
                                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                    "frac": round(dec_gbs / world / peaks["hbm_gbs"], 4),
                                    "kernel": "decode_tc_kernel<128, 4>",
                                    "peak_source": f"{peaks['source']} HBM copy"},
                       "rope_cache": {"ms_per_token_step": round(rc_ms / wd.steps, 4),
                                      "gbs_kv": round(rc_gbs, 1),
                                      "frac_of_hbm": round(rc_gbs / world / peaks["hbm_gbs"], 4)},
                       "G": [jl.group_size(wd.length_at(0), wd.w_pretrained),
                             jl.group_size(wd.length_at(wd.steps - 1), wd.w_pretrained)]},
            "roofline": {"bound": "tensor", "achieved": round(pre_tflops / world, 2),
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(frac_b, 4), "traffic": prefill_traffic(),
                         "kernel": PREFILL_KERNEL,
                         "peak_source": f"{peaks['source']} bf16 burst (cuBLAS GEMM timed alone; "
                                        "the prefill is one launch of ~0.15 s)",
                         "frac_of_sustained": round(frac_s, 4),
                         "per_clock": per_clock(pre_tflops / world, clocks.get("sm_mhz"), peaks)},
            "e2e": {"value": round(world * computed / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 3), "call": "prefill_streamed",
                    "chunks": E2E_CHUNKS},
            "gpu_launches": int(launches),
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
