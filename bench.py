#!/usr/bin/env python3
"""Benchmark of paged-KV decode attention (libpagedattn, B200).

One step = one paged_attn_decode call (split-KV decode + merge) over the
workload's whole visible KV cache.  Default workload: speculative verify,
batch 1, 8 causal query tokens after 61440 cached tokens (L = 61448), 32/8
heads, head_dim 128, block_size 16, fp16 cache.  The 200k-context decode
(1 query token, 32/4 heads, L = 196608) is measured the same way and reported
alongside.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 (launched with torch.distributed.run): every rank runs an independent
replica of the workload on its own GPU (weak scaling, no data-path
collective); the time is the max over ranks and the value the sum of all
ranks' KV bytes over that time.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_decode_flash_b200 import inputs as gen  # noqa: E402

METRIC = "µs/call and KV-read HBM GB/s (% of B200 peak) at 61k and 200k context"
NOMINAL_HBM_GBS = 8000.0
PRIMARY = "spec_verify_61k"
SECONDARY = "decode_200k"
WORKLOAD_TEXT = {
    "spec_verify_61k": "speculative verify: B=1, 8 causal query tokens after 61440 cached "
                       "(L=61448), Hq/Hkv=32/8, head_dim 128, block_size 16, fp16 N(0,1), "
                       "seeded random block permutation",
    "decode_200k": "200k-context decode: B=1, 1 query token, Hq/Hkv=32/4, head_dim 128, "
                   "L=196608, block_size 16, fp16 N(0,1) with 1% of keys x8",
}


OTHER_CONFIGS = ("tiny", "sliding_window", "mixed_q8_0")
CONFIG_TEXT = {
    "tiny": "tiny decode: B=1, 1 query token, Hq/Hkv=8/2, L=1024, block_size 16, fp16, "
            "64 of 128 pool blocks (latency-bound: the whole KV is 1 MB)",
    "sliding_window": "sliding-window drafter: B=1, 8 non-causal query tokens, window 2048 "
                      "of L=24576, Hq/Hkv=32/8, fp16; blocks outside the window hold NaN",
    "mixed_q8_0": "mixed batch: B=8, 4 causal query tokens, L_s ~ U[4096, 65536], "
                  "Hq/Hkv=32/8, q8_0 cache (int8 + fp16 scale per 32)",
}


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_sha():
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "paged_kv_decode_flash_b200", "csrc", "*"))):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """Per-launch DRAM bytes of the decode kernel from the committed ncu
    summary, or None if absent or taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    ent = d.get(workload)
    if not ent or ent.get("source_sha") != kernel_source_sha():
        return None
    return float(ent["dram_bytes_per_launch"])


def max_over_ranks(x, dist, device):
    """The largest of the ranks' x (every rank gets it); x itself without a
    process group.  Times of a multi-GPU run are the slowest rank's."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(kv_bytes_per_rank, world, seconds_per_step):
    """Whole-job KV-read rate: every rank reads its own replica's bytes each
    step (weak scaling), over the slowest rank's time per step."""
    return world * kv_bytes_per_rank / seconds_per_step / 1e9


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def bench_ours(args, rank, world, dist):
    import torch
    from paged_kv_decode_flash_b200 import binding as B

    dev_index = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(dev_index)
    device = torch.device("cuda", dev_index)
    l2_bytes = torch.cuda.get_device_properties(device).L2_cache_size

    def measure(name, steps, warmup, with_e2e):
        case = gen.CONFIGS[name](seed=rank)
        kv_bytes = gen.visible_kv_bytes(case)
        pool_bytes = case.k_cache.nbytes + case.v_cache.nbytes
        copies = max(2, math.ceil(3 * l2_bytes / pool_bytes))
        base = B.case_to_device(case, device)
        pools = [(base["k_cache"], base["v_cache"])]
        for _ in range(copies - 1):
            pools.append((base["k_cache"].clone(), base["v_cache"].clone()))
        dec = B.PagedDecode.for_case(case, device=device)
        out = torch.empty_like(base["q"])
        kw = dict(causal=case.causal, window=case.window, scale=case.scale,
                  kv_dtype=case.kv_dtype)
        stream = torch.cuda.current_stream(device)

        def step(i, o=out):
            k, v = pools[i % copies]
            dec(base["q"], k, v, base["block_table"], base["context_lens"], out=o,
                stream=stream, **kw)

        for i in range(warmup):
            step(i)
        torch.cuda.synchronize()
        if dec.get_error() != 0:
            raise RuntimeError("device reported a data error during warm-up")

        # The calls are replayed from a CUDA graph (a decode step runs inside
        # captured graphs; the call allocates nothing and never waits on the
        # host): a graph of G calls, G dividing `steps`, rotating the pools.
        G = max(d for d in range(1, min(steps, 500) + 1) if steps % d == 0)
        gstream = torch.cuda.Stream(device)
        gstream.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gstream):
            for i in range(G):
                k, v = pools[i % copies]
                dec(base["q"], k, v, base["block_table"], base["context_lens"], out=out,
                    stream=gstream, **kw)
        with torch.cuda.stream(gstream):
            graph.replay()
        torch.cuda.synchronize()

        # Timed region: exactly `steps` calls back to back between two events
        # on the launching stream (barrier + synchronize on both sides).
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev_index) as clk:
            if dist:
                dist.barrier()
            torch.cuda.synchronize()
            with torch.cuda.stream(gstream):  # replay() launches on the current stream
                t0.record(gstream)
                for _ in range(steps // G):
                    graph.replay()
                t1.record(gstream)
            torch.cuda.synchronize()
            if dist:
                dist.barrier()
        total_ms = t0.elapsed_time(t1)
        if dec.get_error(gstream) != 0:
            raise RuntimeError("device reported a data error in the timed region")
        # The same calls launched one by one from Python (reported beside).
        n_eager = min(steps, 500)
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        ea.record(stream)
        for i in range(n_eager):
            step(i)
        eb.record(stream)
        torch.cuda.synchronize()
        eager_us = ea.elapsed_time(eb) * 1e3 / n_eager
        del graph
        total_ms = max_over_ranks(total_ms, dist, device)
        # Per-call spread (outside the timed region): events around each call.
        n_ev = min(steps, 300)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_ev)]
        for i in range(n_ev):
            ev[i][0].record(stream)
            step(i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        per_call = sorted(a.elapsed_time(b) * 1e3 for a, b in ev)  # us
        res = {
            "case": case, "kv_bytes": kv_bytes, "copies": copies, "pool_bytes": pool_bytes,
            "ms_per_step": total_ms / steps, "eager_us": eager_us, "graph_calls": G,
            "us_median": per_call[len(per_call) // 2], "us_min": per_call[0],
            "us_p90": per_call[min(len(per_call) - 1, int(0.9 * len(per_call)))],
            "clocks": clk.summary(), "splits": dec.num_splits(case.kv_dtype),
            "launches": dec.launches_per_call(case.kv_dtype),
        }
        if with_e2e:
            res["e2e"] = e2e(case, dec, base, pools[0], steps=min(steps, 500))
        del pools, base
        torch.cuda.empty_cache()
        return res

    def e2e(case, dec, base, pool, steps):
        """Per step: pinned host -> device copy of the step's inputs (q,
        block_table, context_lens), the C-ABI decode, device -> pinned host
        copy of the output, synchronise.  The KV cache is the persistent
        cache state and stays resident."""
        hq = torch.from_numpy(case.q).pin_memory()
        hbt = torch.from_numpy(case.block_table).pin_memory()
        hcl = torch.from_numpy(case.context_lens).pin_memory()
        hout = torch.empty(hq.shape, dtype=torch.float16).pin_memory()
        dq, dbt, dcl = (torch.empty_like(x, device=device) for x in (hq, hbt, hcl))
        dout = torch.empty_like(dq)
        kw = dict(causal=case.causal, window=case.window, scale=case.scale,
                  kv_dtype=case.kv_dtype)

        def one():
            dq.copy_(hq, non_blocking=True)
            dbt.copy_(hbt, non_blocking=True)
            dcl.copy_(hcl, non_blocking=True)
            dec(dq, pool[0], pool[1], dbt, dcl, out=dout, **kw)
            hout.copy_(dout, non_blocking=True)
            torch.cuda.current_stream().synchronize()

        for _ in range(5):
            one()
        if dist:
            dist.barrier()
        t = time.perf_counter()
        for _ in range(steps):
            one()
        dt = (time.perf_counter() - t) / steps
        dt = max_over_ranks(dt, dist, device)
        h2d = hq.nbytes + hbt.nbytes + hcl.nbytes
        return {"s_per_step": dt, "h2d": h2d, "d2h": hout.nbytes}

    primary = args.workload
    if primary not in WORKLOAD_TEXT and not args.primary_only:
        raise SystemExit("--workload " + primary + " is timed alone: add --primary-only")
    secondary = SECONDARY if primary == PRIMARY else PRIMARY
    prim = measure(primary, args.steps, args.warmup, with_e2e=True)
    sec = measure(secondary, max(1, args.steps // 2), args.warmup, with_e2e=False) \
        if not args.primary_only else None
    # The parity-test configurations, timed the same way (reported, not the
    # headline): tiny decode, sliding window, mixed batch over a q8_0 cache.
    others = {}
    if not args.primary_only:
        for name in OTHER_CONFIGS:
            r = measure(name, max(3, min(args.steps // 10, 200)), args.warmup, with_e2e=False)
            others[name] = r

    peak, peak_kind = measured_peaks()
    kv = prim["kv_bytes"]
    value = job_gbs(kv, world, prim["ms_per_step"] * 1e-3)
    achieved = kv / (prim["ms_per_step"] * 1e-3) / 1e9  # per launch pair, timed region
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(prim["ms_per_step"], 5),
        "us_per_call": round(prim["ms_per_step"] * 1e3, 2),
        "pct_of_8TBps": round(100 * kv / (prim["ms_per_step"] * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded N(0,1) fp16 KV, random block permutation)",
        "impl": "ours",
        "config": {
            "workload": WORKLOAD_TEXT.get(primary) or CONFIG_TEXT[primary],
            "kv_bytes_per_step": kv,
            "num_splits": prim["splits"],
            "l2": f"inputs larger than L2: {prim['copies']} KV pools of "
                  f"{prim['pool_bytes'] / 1e6:.0f} MB rotated per step (L2 {l2_bytes / 1e6:.0f} MB)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "per_call_us": {"median": round(prim["us_median"], 2), "min": round(prim["us_min"], 2),
                        "p90": round(prim["us_p90"], 2),
                        "what": "events around single eager calls (includes launch gaps)"},
        "eager_us_per_call": round(prim["eager_us"], 2),
        "timing": f"CUDA graph of {prim['graph_calls']} calls replayed {args.steps // prim['graph_calls']}x "
                  "inside the timed region; eager_us_per_call = the same calls launched one by one",
        "roofline": {
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
            "traffic": recorded_traffic(primary),
            "kernel": "one paged_attn_decode call: one launch of the split-KV decode kernel "
                      "(cooperative when its grid fits on the device at once), whose CTAs "
                      "also merge the split partials; time = timed region / steps",
        },
        "clocks": prim["clocks"],
        "gpu_launches": prim["launches"] * args.steps,
    }
    e = prim["e2e"]
    line["e2e"] = {"value": round(job_gbs(kv, world, e["s_per_step"]), 1), "unit": "GB/s",
                   "us_per_call": round(e["s_per_step"] * 1e6, 2),
                   "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"]}
    if sec is not None:
        kv2 = sec["kv_bytes"]
        line["also"] = {
            "workload": WORKLOAD_TEXT[secondary],
            "us_per_call": round(sec["ms_per_step"] * 1e3, 2),
            "eager_us_per_call": round(sec["eager_us"], 2),
            "value": round(job_gbs(kv2, world, sec["ms_per_step"] * 1e-3), 1), "unit": "GB/s",
            "pct_of_8TBps": round(100 * kv2 / (sec["ms_per_step"] * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 1),
            "roofline_frac": round(kv2 / (sec["ms_per_step"] * 1e-3) / 1e9 / peak, 4),
            "per_call_us": {"median": round(sec["us_median"], 2), "min": round(sec["us_min"], 2),
                            "p90": round(sec["us_p90"], 2)},
            "kv_bytes_per_step": kv2, "num_splits": sec["splits"],
            "traffic": recorded_traffic(secondary),
        }
    if others:
        line["configs"] = {}
        for name, r in others.items():
            kvb = r["kv_bytes"]
            gbs = kvb / (r["ms_per_step"] * 1e-3) / 1e9
            line["configs"][name] = {
                "workload": CONFIG_TEXT[name], "kv_bytes_per_step": kvb,
                "us_per_call": round(r["ms_per_step"] * 1e3, 2), "GB/s": round(gbs, 1),
                "eager_us_per_call": round(r["eager_us"], 2),
                "roofline_frac": round(gbs / peak, 4), "num_splits": r["splits"],
                "launches_per_call": r["launches"],
                "per_call_us": {"median": round(r["us_median"], 2), "min": round(r["us_min"], 2)},
                "l2": f"{r['copies']} KV pool copies rotated",
            }
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(prim["case"], budget_s=args.cpu_seconds)
    return line


# ---------------------------------------------------------------------------
# the fp64 oracle on the host cores (baseline, never the product path)
# ---------------------------------------------------------------------------
def cpu_baseline(case, budget_s=15.0):
    import oracle
    orc = oracle.load()
    threads = orc.num_threads()
    rows = np.random.default_rng(0).permutation(case.rows)
    done, t_total = 0, 0.0
    batch = max(1, threads)
    while done < rows.size and t_total < budget_s:
        ids = rows[done: done + batch]
        t = time.perf_counter()
        orc.attend_rows(case, ids)
        t_total += time.perf_counter() - t
        done += ids.size
    per_call = t_total / done * case.rows
    kv = gen.visible_kv_bytes(case)
    return {"value": round(kv / per_call / 1e9, 4), "unit": "GB/s",
            "us_per_call": round(per_call * 1e6, 1), "cores": threads, "kind": "oracle",
            "sample": f"{done} of {case.rows} query rows of one call, "
                      f"{t_total:.1f} s of fp64 C with OpenMP, extrapolated to the full call"}


def bench_reference(args, rank, world):
    """The oracle, as it stands, on this host's cores: each step is a bounded
    sample of the workload's rows, timed and extrapolated to a full call."""
    if rank != 0:
        return None
    case = gen.CONFIGS[PRIMARY](seed=0)
    budget = max(1.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(case, budget_s=budget)
    samples = [cpu_baseline(case, budget_s=budget) for _ in range(args.steps)]
    us = statistics.median(s["us_per_call"] for s in samples)
    kv = gen.visible_kv_bytes(case)
    value = kv / (us * 1e-6) / 1e9
    cb = dict(samples[-1])
    cb["value"] = round(value, 4)
    return {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1e3, 3),
        "us_per_call": round(us, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD_TEXT[PRIMARY], "kv_bytes_per_step": kv,
                   "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": cb,
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--primary-only", action="store_true")
    ap.add_argument("--workload", choices=[PRIMARY, SECONDARY, *OTHER_CONFIGS], default=PRIMARY,
                    help="workload of the headline line (the other of the two headline "
                         "workloads is reported under 'also'; the other configurations only "
                         "with --primary-only, e.g. for a profiler run)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = env_int("WORLD_SIZE", 1)
    rank = env_int("RANK", 0)
    if args.impl == "reference":
        line = bench_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(env_int("LOCAL_RANK", 0))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        line = bench_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
