#!/usr/bin/env python3
"""Benchmark of paged-KV decode attention (libpagedattn, B200).

One step = one paged_attn_decode call (split-KV decode with its merge) over
the workload's whole visible KV cache.  Default workload: speculative verify,
batch 1, 8 causal query tokens after 61440 cached tokens (L = 61448), 32/8
heads, head_dim 128, block_size 16, fp16 cache.  The 200k-context decode
(1 query token, 32/4 heads, L = 196608) is measured the same way and reported
alongside under "also"; the other configurations under "configs".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--split replicas|context]

N > 1 (launched with torch.distributed.run): --split replicas (default) runs
an independent replica of the workload on every rank (weak scaling, no
data-path collective); --split context cuts one long sequence's KV blocks
across the ranks, each rank computes fp32 partials (O, lse) of its share,
one all-gather exchanges them and every rank merges (paged_attn_merge).  The
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import platform
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
DRIFT_LIMIT_PCT = 1.5
WORKLOAD_TEXT = {
    "spec_verify_61k": "speculative verify: B=1, 8 causal query tokens after 61440 cached "
                       "(L=61448), Hq/Hkv=32/8, head_dim 128, block_size 16, fp16 N(0,1), "
                       "seeded random block permutation",
    "decode_200k": "200k-context decode: B=1, 1 query token, Hq/Hkv=32/4, head_dim 128, "
                   "L=196608, block_size 16, fp16 N(0,1) with 1% of keys x8",
    "tiny": "tiny decode: B=1, 1 query token, Hq/Hkv=8/2, L=1024, block_size 16, fp16, "
            "64 of 128 pool blocks (latency-bound: the whole KV is 1 MB)",
    "sliding_window": "sliding-window drafter: B=1, 8 non-causal query tokens, window 2048 "
                      "of L=24576, Hq/Hkv=32/8, fp16; blocks outside the window hold NaN",
    "mixed_q8_0": "mixed batch: B=8, 4 causal query tokens, L_s ~ U[4096, 65536], "
                  "Hq/Hkv=32/8, q8_0 cache (int8 + fp16 scale per 32)",
    "mtp_q8_0_61k": "MTP verify over an int8 cache (the pages' decode shape): B=1, 4 causal "
                    "query tokens x 6 query heads per KV head (24 rows), Hq/Hkv=24/4, "
                    "L=61448, q8_0 cache",
    "mtp_int8_row_61k": "the same shape over an int8 cache with fp32 row scales",
    "verify_64rows_61k": "8-token verify at GQA 8 (64 rows per KV head): B=1, Hq/Hkv=64/8, "
                         "L=61448, fp16",
    "prefill_chunk_16k": "a chunk of 64 new tokens appended to a 16320-token cache (L=16384, "
                         "causal): B=1, Hq/Hkv=32/8 (256 rows per KV head, eight row parts "
                         "of 32), fp16",
}
OTHER_CONFIGS = ("tiny", "sliding_window", "mixed_q8_0", "mtp_q8_0_61k", "mtp_int8_row_61k",
                 "verify_64rows_61k", "prefill_chunk_16k")


def make_workload(name, seed=0):
    if name in gen.CONFIGS:
        return gen.CONFIGS[name](seed)
    if name in ("mtp_q8_0_61k", "mtp_int8_row_61k"):
        dt = gen.KV_Q8_0 if name == "mtp_q8_0_61k" else gen.KV_INT8_ROW
        return gen.make_case(name=name, seed=seed, context_lens=(61448,), n_query=4,
                             num_q_heads=24, num_kv_heads=4, causal=1, kv_dtype=dt)
    if name == "verify_64rows_61k":
        return gen.make_case(name=name, seed=seed, context_lens=(61448,), n_query=8,
                             num_q_heads=64, num_kv_heads=8, causal=1)
    if name == "prefill_chunk_16k":
        return gen.make_case(name=name, seed=seed, context_lens=(16384,), n_query=64,
                             num_q_heads=32, num_kv_heads=8, causal=1)
    raise KeyError(name)


def config_dict(name, world, split="replicas"):
    """The workload description, the same for both arms."""
    case = make_workload(name)
    return {"workload": WORKLOAD_TEXT[name], "kv_bytes_per_step": gen.visible_kv_bytes(case),
            "parallelism": (f"{split} x{world}" if world > 1 else "single GPU")}


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


def spread(values):
    """median, min, max and (max - min) / median in percent of a list."""
    med = statistics.median(values)
    return {"median": med, "min": min(values), "max": max(values),
            "spread_pct": 100.0 * (max(values) - min(values)) / med if med > 0 else 0.0}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


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
        time.sleep(0.5)  # nvidia-smi's start-up (driver queries) is over before timing
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
def read_peak(device, torch, B):
    """Read-only HBM ceiling of the decode kernel's access pattern: the
    library's streaming probe (4 KB bulk copies into 32 KB shared-memory
    slots, one CTA per SM) over 4 GiB, best of 5 (CUDA events)."""
    import ctypes
    L = B.lib()
    f = L.paged_attn_stream_read
    f.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    f.restype = ctypes.c_int
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    nbytes = 4 << 30
    buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
    buf.fill_(1)
    sink = torch.empty(sms, dtype=torch.int32, device=device)
    st = torch.cuda.current_stream(device)
    best = 0.0
    for it in range(6):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        rc = f(buf.data_ptr(), nbytes, sink.data_ptr(), sms, st.cuda_stream)
        b.record(st)
        torch.cuda.synchronize()
        if rc != 0 or bool((sink == -559038737).any()):  # 0xdeadbeef: a wait timed out
            return None
        if it > 0:
            best = max(best, (nbytes // 32768 * 32768) / (a.elapsed_time(b) * 1e-3) / 1e9)
    del buf
    torch.cuda.empty_cache()
    return {"value": round(best, 1), "unit": "GB/s", "what": "read-only streaming probe "
            "(paged_attn_stream_read: 4 KB bulk copies into 6 x 32 KB smem slots per SM, "
            f"{sms} CTAs, 4 GiB, best of 5)"}


def bench_ours(args, rank, world, dist):
    import torch
    from paged_kv_decode_flash_b200 import binding as B

    dev_index = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(dev_index)
    device = torch.device("cuda", dev_index)
    l2_bytes = torch.cuda.get_device_properties(device).L2_cache_size

    def measure(name, steps, warmup, reps, with_e2e):
        case = make_workload(name, seed=rank)
        kv_bytes = gen.visible_kv_bytes(case)
        pool_bytes = case.k_cache.nbytes + case.v_cache.nbytes
        # Inputs larger than L2: at least four copies of the pool, and enough
        # that the VISIBLE bytes the rotated calls read add up to 3x L2 (at
        # most 48 GB of copies).  With two copies of a 252 MB pool, lines of
        # the call before last measurably survived in L2 (0.5 us at 61k, 2.8
        # us with every cache line marked evict-first); with four, none do.
        copies = max(4, math.ceil(3 * l2_bytes / kv_bytes))
        copies = max(2, min(copies, int(48e9 // pool_bytes)))
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

        # Timed regions: exactly `steps` calls back to back between two events
        # on the launching stream (barrier + synchronize on both sides); the
        # first is the reported one, all `reps` give the spread.
        times = []
        with ClockSampler(dev_index) as clk:
            with torch.cuda.stream(gstream):  # one more untimed replay, under the sampler
                graph.replay()
            torch.cuda.synchronize()
            for _ in range(reps):
                t0 = torch.cuda.Event(enable_timing=True)
                t1 = torch.cuda.Event(enable_timing=True)
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
                times.append(max_over_ranks(t0.elapsed_time(t1), dist, device))
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
        rep_us = [t * 1e3 / steps for t in times]
        res = {
            "case": case, "kv_bytes": kv_bytes, "copies": copies, "pool_bytes": pool_bytes,
            "ms_per_step": times[0] / steps, "rep_us": rep_us, "eager_us": eager_us,
            "graph_calls": G, "us_median": per_call[len(per_call) // 2], "us_min": per_call[0],
            "us_p90": per_call[min(len(per_call) - 1, int(0.9 * len(per_call)))],
            "clocks": clk.summary(), "splits": dec.num_splits(case.kv_dtype),
            "launches": dec.launches_per_call(case.kv_dtype),
        }
        if with_e2e:
            res["e2e"] = e2e(case, dec, pools[0], steps=min(steps, 500))
        del pools, base
        torch.cuda.empty_cache()
        return res

    def e2e(case, dec, pool, steps):
        """Per step, through the library's public call: ONE pinned host ->
        device copy of the step's inputs (q, block_table and context_lens
        packed in one buffer), the C-ABI decode, a device -> pinned host copy
        of the output, synchronise.  The KV cache is the persistent cache
        state and stays resident."""
        parts = [("q", case.q), ("block_table", case.block_table),
                 ("context_lens", case.context_lens)]
        offs, off = {}, 0
        for n, a in parts:
            offs[n] = off
            off = (off + a.nbytes + 255) // 256 * 256
        host = torch.empty(off, dtype=torch.uint8).pin_memory()
        for n, a in parts:
            host[offs[n]: offs[n] + a.nbytes].copy_(torch.from_numpy(np.ascontiguousarray(a).view(np.uint8).reshape(-1)))
        dbuf = torch.empty(off, dtype=torch.uint8, device=device)

        def view(n, a, dt):
            return dbuf[offs[n]: offs[n] + a.nbytes].view(dt).view(a.shape)

        dq = view("q", case.q, torch.float16)
        dbt = view("block_table", case.block_table, torch.int32)
        dcl = view("context_lens", case.context_lens, torch.int32)
        hout = torch.empty(case.q.shape, dtype=torch.float16).pin_memory()
        dout = torch.empty_like(dq)
        kw = dict(causal=case.causal, window=case.window, scale=case.scale,
                  kv_dtype=case.kv_dtype)

        def one():
            dbuf.copy_(host, non_blocking=True)
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
        return {"s_per_step": dt, "h2d": host.numel(), "d2h": hout.nbytes}

    primary = args.workload
    if primary not in (PRIMARY, SECONDARY) and not args.primary_only:
        raise SystemExit("--workload " + primary + " is timed alone: add --primary-only")
    secondary = SECONDARY if primary == PRIMARY else PRIMARY
    reps = max(3, args.reps)
    prim = measure(primary, args.steps, args.warmup, reps, with_e2e=True)
    sec = measure(secondary, args.steps, args.warmup, reps, with_e2e=False) \
        if not args.primary_only else None
    # The other configurations, timed the same way with the full step count
    # (reported, not the headline).
    others = {}
    if not args.primary_only:
        for name in OTHER_CONFIGS:
            others[name] = measure(name, args.steps, args.warmup, reps, with_e2e=False)
    probe = read_peak(device, torch, B) if not args.no_probe else None

    peak, peak_kind = measured_peaks()
    kv = prim["kv_bytes"]
    value = job_gbs(kv, world, prim["ms_per_step"] * 1e-3)
    achieved = kv / (prim["ms_per_step"] * 1e-3) / 1e9
    rs = spread(prim["rep_us"])
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(prim["ms_per_step"], 5),
        "us_per_call": round(prim["ms_per_step"] * 1e3, 2),
        "pct_of_8TBps": round(100 * achieved / NOMINAL_HBM_GBS, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded N(0,1) fp16 KV, random block permutation)",
        "impl": "ours",
        "config": config_dict(primary, world),
        "setup": {"num_splits": prim["splits"],
                  "l2": f"inputs larger than L2: {prim['copies']} KV pools of "
                        f"{prim['pool_bytes'] / 1e6:.0f} MB rotated per step "
                        f"({prim['copies'] * kv / 1e6:.0f} MB of visible KV; L2 {l2_bytes / 1e6:.0f} MB)"},
        "repeats": {"n": reps, "us_per_call": [round(x, 2) for x in prim["rep_us"]],
                    "median_us": round(rs["median"], 2), "min_us": round(rs["min"], 2),
                    "spread_pct": round(rs["spread_pct"], 2),
                    "drift_flag": rs["spread_pct"] > DRIFT_LIMIT_PCT,
                    "what": f"{reps} timed regions of `steps` calls each; the first is the "
                            f"reported value; drift_flag when (max - min) / median > {DRIFT_LIMIT_PCT}%"},
        "per_call_us": {"median": round(prim["us_median"], 2), "min": round(prim["us_min"], 2),
                        "p90": round(prim["us_p90"], 2),
                        "what": "events around single eager calls (includes launch gaps)"},
        "eager_us_per_call": round(prim["eager_us"], 2),
        "timing": f"CUDA graph of {prim['graph_calls']} calls replayed {args.steps // prim['graph_calls']}x "
                  "inside each timed region; eager_us_per_call = the same calls launched one by one",
        "roofline": {
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
            "traffic": recorded_traffic(primary),
            "read_peak": probe,
            "frac_of_read_peak": round(achieved / probe["value"], 4) if probe else None,
            "kernel": "one paged_attn_decode call: one launch of the split-KV decode kernel "
                      "(cooperative), whose CTAs also merge the split partials; "
                      "time = timed region / steps",
        },
        "clocks": prim["clocks"],
        "gpu_launches": prim["launches"] * args.steps,
    }
    e = prim["e2e"]
    line["e2e"] = {"value": round(job_gbs(kv, world, e["s_per_step"]), 1), "unit": "GB/s",
                   "us_per_call": round(e["s_per_step"] * 1e6, 2),
                   "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                   "what": "one pinned H2D copy of the packed q / block_table / context_lens, "
                           "the C-ABI call, a pinned D2H copy of the output, synchronise"}
    if sec is not None:
        kv2 = sec["kv_bytes"]
        rs2 = spread(sec["rep_us"])
        line["also"] = {
            "workload": WORKLOAD_TEXT[secondary],
            "us_per_call": round(sec["ms_per_step"] * 1e3, 2),
            "eager_us_per_call": round(sec["eager_us"], 2),
            "value": round(job_gbs(kv2, world, sec["ms_per_step"] * 1e-3), 1), "unit": "GB/s",
            "pct_of_8TBps": round(100 * kv2 / (sec["ms_per_step"] * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 1),
            "roofline_frac": round(kv2 / (sec["ms_per_step"] * 1e-3) / 1e9 / peak, 4),
            "repeats_us": [round(x, 2) for x in sec["rep_us"]],
            "spread_pct": round(rs2["spread_pct"], 2),
            "drift_flag": rs2["spread_pct"] > DRIFT_LIMIT_PCT,
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
            rsn = spread(r["rep_us"])
            line["configs"][name] = {
                "workload": WORKLOAD_TEXT[name], "kv_bytes_per_step": kvb,
                "us_per_call": round(r["ms_per_step"] * 1e3, 2), "GB/s": round(gbs, 1),
                "repeats_us": [round(x, 2) for x in r["rep_us"]],
                "spread_pct": round(rsn["spread_pct"], 2),
                "drift_flag": rsn["spread_pct"] > DRIFT_LIMIT_PCT,
                "eager_us_per_call": round(r["eager_us"], 2),
                "roofline_frac": round(gbs / peak, 4), "num_splits": r["splits"],
                "launches_per_call": r["launches"],
                "per_call_us": {"median": round(r["us_median"], 2), "min": round(r["us_min"], 2)},
                "l2": f"{r['copies']} KV pool copies rotated "
                      f"({r['copies'] * kvb / 1e6:.0f} MB of visible KV)",
                "traffic": recorded_traffic(name),
            }
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(prim["case"], budget_s=args.cpu_seconds)
    return line


# ---------------------------------------------------------------------------
# the fp64 oracle on the host cores (baseline, never the product path)
# ---------------------------------------------------------------------------
def oracle_sample(orc, case, rows, threads):
    """Wall time of the oracle on the given query rows with `threads` threads."""
    orc.set_num_threads(threads)
    t = time.perf_counter()
    orc.attend_rows(case, rows)
    return time.perf_counter() - t


def cpu_baseline(case, budget_s=10.0):
    import oracle
    orc = oracle.load()
    cores = os.cpu_count() or 1
    rows = np.random.default_rng(0).permutation(case.rows)
    done, t_total = 0, 0.0
    while done < rows.size and t_total < budget_s:
        ids = rows[done: done + cores]
        t_total += oracle_sample(orc, case, ids, cores)
        done += ids.size
    per_call = t_total / done * case.rows
    # one thread, a smaller sample
    n1 = max(1, min(4, case.rows))
    t1 = oracle_sample(orc, case, rows[:n1], 1) / n1 * case.rows
    orc.set_num_threads(cores)
    kv = gen.visible_kv_bytes(case)
    return {"value": round(kv / per_call / 1e9, 4), "unit": "GB/s",
            "us_per_call": round(per_call * 1e6, 1), "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{done} of {case.rows} query rows of one call, {t_total:.1f} s of fp64 C "
                      f"with OpenMP on {cores} threads, scaled to the full call",
            "single_thread": {"us_per_call": round(t1 * 1e6, 1),
                              "value": round(kv / t1 / 1e9, 5), "unit": "GB/s",
                              "sample": f"{n1} query rows on 1 thread, scaled to the full call"}}


def bench_reference(args, rank, world):
    """The oracle, as it stands, on this host's cores.  Each step is one
    bounded sample of the workload's query rows (the same sample every step),
    timed in full: ms_per_step is that sample's time, and value the sample's
    share of the algorithmic KV bytes over it."""
    if rank != 0:
        return None
    import oracle
    orc = oracle.load()
    case = make_workload(PRIMARY, seed=0)
    cores = os.cpu_count() or 1
    orc.set_num_threads(cores)
    n_rows = min(case.rows, max(cores, 32))
    rows = np.random.default_rng(0).permutation(case.rows)[:n_rows]
    for _ in range(args.warmup):
        orc.attend_rows(case, rows)
    ts = []
    for _ in range(args.steps):
        t = time.perf_counter()
        orc.attend_rows(case, rows)
        ts.append(time.perf_counter() - t)
    sec = statistics.mean(ts)
    kv = gen.visible_kv_bytes(case) * n_rows / case.rows
    value = kv / sec / 1e9
    return {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec * 1e3, 3),
        "us_per_call": round(sec * 1e6 * case.rows / n_rows, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": config_dict(PRIMARY, world),
        "setup": {"step": f"{n_rows} of {case.rows} query rows of one call per step "
                          f"(the fp64 oracle, OpenMP on {cores} threads); us_per_call scales "
                          "that to the full call"},
        "cpu_baseline": {"kind": "oracle", "cores": cores, "cpu_model": cpu_model(),
                         "value": round(value, 4), "unit": "GB/s",
                         "sample": f"{n_rows} query rows per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--split", choices=["replicas", "context"], default="replicas")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-probe", action="store_true")
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
        if args.split == "context" and world > 1:
            from paged_kv_decode_flash_b200 import context_parallel
            line = context_parallel.bench(args, rank, world, dist)
        else:
            line = bench_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
