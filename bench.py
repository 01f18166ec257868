#!/usr/bin/env python3
"""Benchmark of MoE token dispatch + combine on B200 (libepx, sm_100a).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl epx|reference]

A step is one pass of the hot path over one batch: routing layout ->
dispatch/expand -> combine reduce (the stand-in expert output that combine
reads is produced once before timing; the stand-in is not part of the
metric).  Prints ONE JSON line on rank 0.

N > 1 (launched by torch.distributed.run): every rank runs an independent
replica on its own GPU with its own seeded batch (weak scaling, no
collective on the data path); a barrier brackets the timed region and the
elapsed time is the max over ranks.

--impl reference times the CPU oracle (single-threaded C) on the host on a
bounded sample of the same workload, for the same metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dispatch+combine tokens/s at 7168×top8; achieved HBM GB/s vs B200 roofline"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024

DESCRIBE = {
    "tiny": "tiny T=128 H=256 E=16 R=4 top-4 uniform",
    "decode": "decode T=128 H=7168 E=256 R=16 top-8 uniform",
    "prefill": "prefill-skew T=4096 H=7168 E=256 R=16 top-8 zipf(1.2)",
    "lowbatch1": "low-batch T=1 H=3584 E=896 R=32 top-16 (1 real row)",
    "lowbatch2": "low-batch T=2 H=3584 E=896 R=32 top-16 (1 real row)",
    "lowbatch4": "low-batch T=4 H=3584 E=896 R=32 top-16 (1 real row)",
    "lowbatch8": "low-batch T=8 H=3584 E=896 R=32 top-16 (1 real row)",
    "dp_compact": "dp-batch [120,1x7] compact 127 rows H=7168 E=256 R=16 top-8",
    "dp_padded": "dp-batch [120,1x7] padded to 960 rows H=7168 E=256 R=16 top-8",
}

# sources whose hash keys the committed ncu DRAM traffic figure
KERNEL_SOURCES = {
    "layout_dispatch_expand": ["combine_ep_layout_07_b200/csrc/fused.cu",
                               "combine_ep_layout_07_b200/csrc/epx_internal.cuh"],
    "dispatch_expand": ["combine_ep_layout_07_b200/csrc/dispatch.cu",
                        "combine_ep_layout_07_b200/csrc/epx_internal.cuh"],
    "combine_reduce": ["combine_ep_layout_07_b200/csrc/combine.cu",
                       "combine_ep_layout_07_b200/csrc/epx_internal.cuh"],
    "layout": ["combine_ep_layout_07_b200/csrc/layout.cu",
               "combine_ep_layout_07_b200/csrc/epx_internal.cuh"],
    "dispatch": ["combine_ep_layout_07_b200/csrc/dispatch.cu",
                 "combine_ep_layout_07_b200/csrc/epx_internal.cuh"],
    "expand_index": ["combine_ep_layout_07_b200/csrc/gather.cu",
                     "combine_ep_layout_07_b200/csrc/epx_internal.cuh"],
    "combine_local": ["combine_ep_layout_07_b200/csrc/combine_two_stage.cu",
                      "combine_ep_layout_07_b200/csrc/epx_internal.cuh"],
    "combine_epilogue": ["combine_ep_layout_07_b200/csrc/combine_two_stage.cu",
                         "combine_ep_layout_07_b200/csrc/epx_internal.cuh"],
}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")


# ------------------------------------------------------------------ helpers

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["epx", "reference"], default="epx")
    ap.add_argument("--workload", choices=sorted(DESCRIBE), default="prefill")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--layout-variant", type=int, default=0,
                    help="0 automatic, 1 warp chunks, 2 count matrix")
    ap.add_argument("--dispatch-variant", type=int, default=0)
    ap.add_argument("--combine-variant", type=int, default=0)
    ap.add_argument("--idx-bits", type=int, choices=[32, 64], default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--flush", choices=["auto", "always", "never"], default="auto")
    ap.add_argument("--eager", action="store_true",
                    help="launch the three calls from Python each step instead of replaying "
                         "one captured CUDA graph per step")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-expand", action="store_true",
                    help="dispatch writes recv rows only plus a gather index (the expert "
                         "consumer reads recv through it); also times that consumer "
                         "against the one reading the expanded copy")
    ap.add_argument("--step-calls", choices=["auto", "separate", "fused", "paired"],
                    default="auto",
                    help="layout and dispatch/expand as one kernel (fused), as one call of two "
                         "kernels whose dispatch reads x early (paired), as two calls "
                         "(separate), or automatic (see step_mode)")
    ap.add_argument("--small-steps", type=int, default=1500,
                    help="steps of each small-batch workload measured beside the headline "
                         "(0 skips them)")
    ap.add_argument("--two-stage", choices=["fp32", "bf16"], default=None,
                    help="combine as a per-(token, rank) local reduce with fp32 or bf16 "
                         "partials followed by the epilogue, instead of the fused reduce")
    return ap.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def alg_bytes(T, T_real, N_recv, N_route, H, k, R, idx_bytes, part_bytes=None,
              no_expand=False, fused=False):
    # fused: False / "separate" (layout and dispatch_expand apart), True /
    # "one_launch" (one kernel), "paired" (one call of the two kernels)
    """Algorithmic HBM bytes per step of each kernel (each byte the definition
    must move once; no re-reads).  With part_bytes (4 or 2) the combine is the
    two-stage form: local reduce + epilogue through N_recv partial rows.  With
    no_expand the dispatch writes recv rows only, plus the gather index.  With
    fused the layout and dispatch/expand are one kernel (their bytes add; the
    layout's own pos / recv_pos stores replace the dispatch's loads of them)."""
    row = H * 2
    layout = T * k * idx_bytes + T * k * 4 + T * R * 4
    if fused is True or fused == "one_launch":
        out = dict(layout_dispatch_expand=layout + T_real * row + (N_recv + N_route) * row)
    elif fused == "paired":
        out = dict(layout_dispatch_expand=layout + T_real * row + (N_recv + N_route) * row
                   + T * k * 4 + T * R * 4)
    elif no_expand:
        out = dict(layout=layout,
                   dispatch=T_real * row + N_recv * row + T * R * 4,
                   expand_index=T * k * 4 + T * R * 4 + N_route * 4)
    else:
        out = dict(layout=layout,
                   dispatch_expand=T_real * row + (N_recv + N_route) * row + T * k * 4 + T * R * 4)
    if part_bytes is None:
        out["combine_reduce"] = N_route * row + T * row + T * k * (4 + 4)
    else:
        out["combine_local"] = N_route * row + N_recv * H * part_bytes + T * k * 8 + T * R * 4
        out["combine_epilogue"] = N_recv * H * part_bytes + T * row + T * R * 4
    out["total"] = sum(out.values())
    return out


def step_alg_bytes(T, tot, H, k, R, args, part_bytes, mode):
    """alg_bytes of one step of the bench's own workload: the same options
    (index width, two-stage partials, no-expand) in whichever form the calls
    take (`mode`: one_launch, paired or separate)."""
    return alg_bytes(T, tot["T_real"], tot["N_recv"], tot["N_route"], H, k, R,
                     args.idx_bits // 8, part_bytes, args.no_expand, fused=mode)


def sources_hash(kernel):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def layout_auto_engine(T, k):
    """The layout schedule the automatic choice takes for T tokens x top-k
    (label for the traffic lookup only): the warp-chunk cluster while a
    cluster of up to 16 CTAs covers the batch in at most four passes of 32
    warps of floor(32/k)-token chunks, else the grid schedule.  The
    shared-memory limit of the warp-chunk table is not mirrored here."""
    csize = max(1, min(16, (T * k + 2047) // 2048))
    tpc = -(-T // csize)
    tpw = max(1, 32 // k)
    return "warp_chunks" if -(-tpc // tpw) <= 4 * 32 else "grid"


def committed_traffic(kernel, workload, engine=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (and copy engine); otherwise None."""
    try:
        lines = open(TRAFFIC_FILE).read().splitlines()
    except OSError:
        return None
    if kernel not in KERNEL_SOURCES:
        return None
    want = sources_hash(kernel)
    for ln in lines:
        if ln.startswith("#") or not ln.strip():
            continue
        kv = dict(x.split("=", 1) for x in ln.split() if "=" in x)
        if (kv.get("kernel") == kernel and kv.get("workload") == workload
                and kv.get("source") == want and kv.get("engine") in (None, engine)):
            return float(kv["dram_bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None
        self.error = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", self.gpu_id],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception as e:  # nvidia-smi missing
            self.error = str(e)
            return
        t0 = time.time()
        while time.time() - t0 < 5 and os.path.getsize(self.path) == 0:
            time.sleep(0.05)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t_lo, t_hi):
        if self.error or not self.path:
            return {"error": self.error or "not started"}
        rows = []
        for ln in open(self.path).read().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                rows.append(dict(ts=ts, sm=float(parts[2]), smax=float(parts[3]),
                                 power=parts[4], active=parts[5], hw=parts[6],
                                 hwt=parts[7], swt=parts[8], pcap=parts[9]))
            except (ValueError, IndexError):
                continue
        os.unlink(self.path)
        inwin = [r for r in rows if t_lo - 0.25 <= r["ts"] <= t_hi + 0.25]
        window = "timed"
        if len(inwin) < 3:
            inwin, window = rows, "whole run (timed region shorter than the sampling period)"
        if not inwin:
            return {"error": "no samples"}
        reasons = set()
        for r in inwin:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in inwin),
                "sm_max_mhz": max(r["smax"] for r in inwin),
                "reasons": sorted(reasons), "samples": len(inwin), "window": window}


def gpu_uuid(torch, dev):
    try:
        u = torch.cuda.get_device_properties(dev).uuid
        s = str(u)
        return s if s.startswith("GPU-") else "GPU-" + s
    except Exception:
        return str(dev)


# --------------------------------------------------------------- CPU oracle

def oracle_pass(oracle, wl, y_bits, idx):
    """One oracle pass of the timed path (layout, dispatch/expand, combine)."""
    lay = oracle.layout(idx, wl["E"], wl["R"])
    oracle.dispatch_expand(wl["x"], lay)
    return oracle.combine(y_bits, wl["topk_weights"], lay), lay


def slice_workload(wl, n):
    out = dict(wl)
    for key in ("x", "topk_idx", "topk_weights"):
        out[key] = np.ascontiguousarray(wl[key][:n])
    out["T"] = n
    return out


def host_cpu():
    """CPU model and logical core count of this host (for the oracle's timing)."""
    model = platform.processor() or ""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "nproc": os.cpu_count()}


def step_stats(step_ms):
    """Median and 10th / 90th percentiles of the per-step times, in µs."""
    a = np.sort(np.asarray(step_ms, dtype=np.float64)) * 1e3
    pick = lambda q: float(a[min(len(a) - 1, int(round(q * (len(a) - 1))))])
    return {"median": pick(0.5), "p10": pick(0.1), "p90": pick(0.9)}


class PinnedToOneCore:
    """Runs the enclosed code on one host core (the oracle is single-threaded;
    pinning keeps its timing from migrating between cores).  Restores the
    previous affinity; a no-op where affinity cannot be set."""

    def __enter__(self):
        self.prev = None
        try:
            self.prev = os.sched_getaffinity(0)
            self.core = min(self.prev)
            os.sched_setaffinity(0, {self.core})
        except (AttributeError, OSError):
            self.core = None
        return self

    def __exit__(self, *exc):
        if self.prev is not None:
            try:
                os.sched_setaffinity(0, self.prev)
            except OSError:
                pass
        return False


def cpu_baseline(wl, budget_s, idx_bits):
    """Oracle, as it stands, over the full workload repeated for ~budget_s,
    pinned to one host core."""
    import oracle
    oracle.build()
    idx = wl["topk_idx"].astype(np.int64 if idx_bits == 64 else np.int32)
    lay = oracle.layout(idx, wl["E"], wl["R"])
    _, expanded = oracle.dispatch_expand(wl["x"], lay)
    y = oracle.standin(expanded, lay)
    out = None
    with PinnedToOneCore() as pin:
        passes, t0 = 0, time.perf_counter()
        while True:
            out, _ = oracle_pass(oracle, wl, y, idx)
            passes += 1
            el = time.perf_counter() - t0
            if el >= budget_s:
                break
    value = lay["T_real"] * passes / el
    return dict(value=value, unit=UNIT, cores=1, kind="oracle", host=host_cpu(),
                pinned_core=pin.core,
                sample=f"{passes} full pass(es) of the {wl['name']} workload "
                       f"({lay['T_real']} effective tokens each) in {el:.1f} s, "
                       f"single-threaded C, layout+dispatch/expand+combine"), \
        dict(layout=lay, expanded=expanded, y=y, out=out)


# ---------------------------------------------------------- reference arm

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0            # rank 0 alone runs the CPU oracle
    import oracle
    from combine_ep_layout_07_b200 import workloads as wlmod
    oracle.build()
    wl = wlmod.make(args.workload, seed=args.seed)
    idx_full = wl["topk_idx"].astype(np.int64 if args.idx_bits == 64 else np.int32)
    # calibrate the per-token oracle cost, then size the sample so the whole
    # run (warm-up + timed) takes about two minutes at most
    n_cal = min(wl["T"], 64)
    sub = slice_workload(wl, n_cal)
    sidx = idx_full[:n_cal]
    slay = oracle.layout(sidx, wl["E"], wl["R"])
    _, sex = oracle.dispatch_expand(sub["x"], slay)
    sy = oracle.standin(sex, slay)
    t0 = time.perf_counter()
    oracle_pass(oracle, sub, sy, sidx)
    per_tok = (time.perf_counter() - t0) / n_cal
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(wl["T"], budget / max(per_tok, 1e-9))))
    sub = slice_workload(wl, n)
    sidx = np.ascontiguousarray(idx_full[:n])
    slay = oracle.layout(sidx, wl["E"], wl["R"])
    _, sex = oracle.dispatch_expand(sub["x"], slay)
    sy = oracle.standin(sex, slay)
    with PinnedToOneCore() as pin:
        for _ in range(args.warmup):
            oracle_pass(oracle, sub, sy, sidx)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle_pass(oracle, sub, sy, sidx)
        el = time.perf_counter() - t0
    units = slay["T_real"] * args.steps
    value = units / el
    sample = (f"first {n} of {wl['T']} rows of the {wl['name']} workload "
              f"({slay['T_real']} effective tokens) per step, single-threaded C oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 accumulate / bf16 data",
        "data": "synthetic", "config": dict(workload_config(wl, args, slay),
                                            launch="host CPU, single thread"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample, "host": host_cpu(), "pinned_core": pin.core},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def step_mode(args, T, k):
    """How the step runs layout and dispatch/expand: "one_launch" (one kernel,
    ep_layout_dispatch_expand variant 1), "paired" (ep_layout_dispatch_expand
    variant 2: the layout and a dispatch that reads x before its wait, one
    call), or "separate" (ep_layout, then ep_dispatch_expand).  Automatic: the
    library's choice, i.e. what ep_layout_dispatch_expand does with variant 0
    (one launch from EPX_FUSED_AUTO_MIN_ROUTES to EPX_FUSED_AUTO_MAX_ROUTES
    routes, paired elsewhere)."""
    if getattr(args, "no_expand", False) or args.step_calls == "separate":
        return "separate"
    if args.step_calls == "fused":
        return "one_launch"
    if args.step_calls == "paired":
        return "paired"
    from combine_ep_layout_07_b200 import epx
    if epx.FUSED_AUTO_MIN_ROUTES <= T * k <= epx.FUSED_AUTO_MAX_ROUTES:
        return "one_launch"
    return "paired"


def workload_config(wl, args, lay_totals, flush_desc=None, mode="separate"):
    cfg = {"workload": DESCRIBE[args.workload], "T": wl["T"], "H": wl["H"], "E": wl["E"],
           "R": wl["R"], "k": wl["k"], "seed": args.seed, "idx_bits": args.idx_bits,
           "T_real": int(lay_totals["T_real"]), "N_recv": int(lay_totals["N_recv"]),
           "N_route": int(lay_totals["N_route"]),
           "timed": ({"one_launch": "layout_dispatch_expand (one launch) + ",
                      "paired": "layout_dispatch_expand (layout + dispatch_expand in one call) + "
                      }.get(mode) or "layout + " + (
               "dispatch (recv only) + expand_index + " if getattr(args, "no_expand", False)
               else "dispatch_expand + ")) + (
               "combine_reduce" if not getattr(args, "two_stage", None) else
               "combine_local_reduce (%s partials) + combine_epilogue" % args.two_stage),
           "parallelism": f"replicas x{dist_env()[1]}"}
    if flush_desc:
        cfg["l2"] = flush_desc
    cfg["launch"] = ("eager, events between kernels" if getattr(args, "eager", True) else
                     "one CUDA graph per step, kernels chained by programmatic dependent "
                     "launch; per-kernel split from a second run of the same steps with "
                     "events between kernels")
    return cfg


class Step:
    """Device buffers and the calls of one step of the path on one workload."""

    def __init__(self, torch, epx, wl, args, dev, mode, two_stage=None, no_expand=False):
        self.torch, self.epx, self.wl = torch, epx, wl
        T, H, E, R, k = wl["T"], wl["H"], wl["E"], wl["R"], wl["k"]
        itype = torch.int64 if args.idx_bits == 64 else torch.int32
        self.x = x = torch.from_numpy(wl["x"].view(np.int16)).view(torch.bfloat16).to(dev)
        self.idx = idx = torch.from_numpy(wl["topk_idx"]).to(itype).to(dev)
        self.w = w = torch.from_numpy(wl["topk_weights"]).to(dev)
        self.lay = lay = epx.Layout(T, k, E, R, args.idx_bits, device=dev)
        self.recv = recv = torch.empty((lay.recv_cap, H), dtype=torch.bfloat16, device=dev)
        self.expanded = expanded = torch.empty((lay.exp_cap, H), dtype=torch.bfloat16,
                                               device=dev)
        self.y = y = torch.empty_like(expanded)
        self.out = out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.part = part = None
        if two_stage:
            self.part = part = torch.empty(
                (lay.recv_cap, H), device=dev,
                dtype=torch.float32 if two_stage == "fp32" else torch.bfloat16)
        self.src = src = (torch.empty((lay.exp_cap,), dtype=torch.int32, device=dev)
                          if no_expand else None)
        self.mode, self.no_expand = mode, no_expand
        self.args = args
        self.calls = self.calls_for(mode)
        self.names = [n for n, _ in self.calls]
        # kernels per step: the paired call launches the layout and the dispatch
        self.n_kernels = len(self.calls) + (1 if mode == "paired" else 0)

    def calls_for(self, mode):
        """The step's calls in `mode` on this step's buffers."""
        epx, args, wl = self.epx, self.args, self.wl
        E, R = wl["E"], wl["R"]
        idx, x, w, lay = self.idx, self.x, self.w, self.lay
        recv, expanded, y, out, part, src = (self.recv, self.expanded, self.y, self.out,
                                             self.part, self.src)
        calls = []
        if mode in ("one_launch", "paired"):
            v = 1 if mode == "one_launch" else 2
            calls.append(("layout_dispatch_expand", lambda st: epx.layout_dispatch_expand(
                idx, x, E, R, out=lay, recv=recv, expanded=expanded, variant=v, stream=st)))
        else:
            calls.append(("layout", lambda st: epx.layout(
                idx, E, R, out=lay, variant=args.layout_variant, stream=st)))
            if self.no_expand:
                calls.append(("dispatch", lambda st: epx.dispatch(x, lay, recv=recv, stream=st)))
                calls.append(("expand_index", lambda st: epx.expand_index(lay, src=src,
                                                                          stream=st)))
            else:
                calls.append(("dispatch_expand", lambda st: epx.dispatch_expand(
                    x, lay, recv=recv, expanded=expanded, variant=args.dispatch_variant,
                    stream=st)))
        if part is None:
            calls.append(("combine_reduce", lambda st: epx.combine_reduce(
                y, w, lay, out=out, variant=args.combine_variant, stream=st)))
        else:
            calls.append(("combine_local", lambda st: epx.combine_local_reduce(
                y, w, lay, partial=part, stream=st)))
            calls.append(("combine_epilogue", lambda st: epx.combine_epilogue(
                part, lay, out=out, stream=st)))
        return calls

    def prepare(self, stream):
        """The stand-in expert's output that combine reads (made once,
        outside the timed steps) and the layout totals."""
        torch, epx = self.torch, self.epx
        with torch.cuda.stream(stream):
            epx.layout(self.idx, self.wl["E"], self.wl["R"], out=self.lay, stream=stream)
            epx.dispatch_expand(self.x, self.lay, recv=self.recv, expanded=self.expanded,
                                stream=stream)
            epx.standin_expert(self.expanded, self.lay, y=self.y, stream=stream)
        self.tot = epx.read_totals(self.lay, stream=stream)
        return self.tot

    def launch(self, st, events=None, calls=None):
        calls = self.calls if calls is None else calls
        for i, (_, fn) in enumerate(calls):
            if events is not None:
                events[i].record(st)
            fn(st)
        if events is not None:
            events[len(calls)].record(st)


class L2Flush:
    """Evicts L2 between steps by READING a buffer of twice its size (outside
    the timed events): lines the previous step left dirty are written back
    during the flush, and the step starts with its inputs in DRAM and no
    dirty lines of anyone else's to write back.  The buffer is float32 and
    is summed in float32 into a preallocated scalar: no conversion copy (an
    integer buffer summed into int64 is first converted, i.e. written, by
    torch), one reduction kernel that only reads."""

    def __init__(self, torch, dev):
        self.buf = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)
        self.torch = torch

    def __call__(self):
        self.torch.sum(self.buf, dim=0, out=self.sink)

    DESC = "L2 flushed between steps (256 MiB float32 read, outside the timed events)"


def time_step(torch, launch, n_calls, stream, dev, steps, warmup, flush=None, eager=False,
              split=True, pg=None):
    """Times `steps` steps of `launch(st, events=None)` with CUDA events on
    `stream`.  Graph mode (default): the step is captured once with events at
    its ends only (programmatic-launch overlaps kept) and, when split, once
    more with events between its calls for the per-call split.  Returns
    (per-step ms, per-step cumulative split ms or None, wall-clock window)."""
    graph = graph_k = None
    if not eager:
        with torch.cuda.stream(stream):
            launch(stream)          # launchers set their function attributes here
        torch.cuda.synchronize(dev)
        gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            cs = torch.cuda.current_stream()
            gev[0].record(cs)
            launch(cs)
            gev[1].record(cs)
        if split:
            gks = [torch.cuda.Event(enable_timing=True, external=True)
                   for _ in range(n_calls + 1)]
            graph_k = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_k, stream=stream):
                launch(torch.cuda.current_stream(), gks)
        torch.cuda.synchronize(dev)

    def one(rec=None, use_split=False):
        if flush is not None:
            flush()
        if graph is not None:
            (graph_k if use_split else graph).replay()
            if rec is not None:
                torch.cuda.current_stream().synchronize()
                if use_split:
                    rec.append([gks[0].elapsed_time(gks[j]) for j in range(1, len(gks))])
                else:
                    rec.append(gev[0].elapsed_time(gev[1]))
        else:
            if rec is not None:
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_calls + 1)]
                launch(torch.cuda.current_stream(), ev)
                rec.append(ev)
            else:
                launch(torch.cuda.current_stream())

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            one()
            if graph_k is not None:
                one(use_split=True)
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    rec, rec_k = [], []
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    t_lo = time.time()
    with torch.cuda.stream(stream):
        for _ in range(steps):
            one(rec)
    torch.cuda.synchronize(dev)
    t_hi = time.time()
    if pg:
        pg.barrier()
    if graph_k is not None:
        with torch.cuda.stream(stream):
            for _ in range(steps):
                one(rec_k, use_split=True)
        torch.cuda.synchronize(dev)
    if graph is None:   # cumulative times from each step's first event
        rec_k = [[e[0].elapsed_time(e[j]) for j in range(1, len(e))] for e in rec]
        step_ms = [r[-1] for r in rec_k]
    else:
        step_ms = rec
    del graph, graph_k
    return step_ms, (rec_k if (split or eager) else None), (t_lo, t_hi)


def time_amortized(torch, launch, stream, dev, flush, reps=50, rounds=40, warmup=2):
    """Per-step time of `launch` with L2 flushed by a read before every step,
    amortised over `reps` steps between two events: one CUDA graph of reps x
    [flush, step] against one of reps x [flush], replayed alternately;
    per round, step = (A - B) / reps.  The events' timestamp granularity
    (a few µs after a long kernel such as the flush) divides by reps, and
    each step is charged the write-back of the lines it left dirty (which
    the next flush has to write back).  Returns step_stats of the rounds,
    plus their mean."""
    with torch.cuda.stream(stream):
        launch(stream)          # launchers set their function attributes here
        flush()
    torch.cuda.synchronize(dev)
    graphs, evs = [], []
    for with_step in (True, False):
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            cs = torch.cuda.current_stream()
            ev[0].record(cs)
            for _ in range(reps):
                flush()
                if with_step:
                    launch(cs)
            ev[1].record(cs)
        graphs.append(g)
        evs.append(ev)
    torch.cuda.synchronize(dev)
    per = []
    with torch.cuda.stream(stream):
        for r in range(warmup + rounds):
            t = []
            for g, ev in zip(graphs, evs):
                g.replay()
                torch.cuda.current_stream().synchronize()
                t.append(ev[0].elapsed_time(ev[1]))
            if r >= warmup:
                per.append((t[0] - t[1]) / reps)
    del graphs
    st = step_stats(per)
    st["mean"] = statistics.fmean(per) * 1e3
    st["method"] = (f"graph of {reps} x [L2 read-flush, step] minus graph of {reps} x "
                    f"[L2 read-flush], {rounds} rounds")
    return st


def time_floor(torch, epx, stream, dev, n_kernels, steps, warmup, flush):
    """ep_latency_floor chain of n_kernels, timed exactly like a step (per
    step, and amortised)."""
    buf = torch.zeros(64 * (2 * n_kernels + 2), dtype=torch.int32, device=dev)
    fn = lambda st, ev=None: epx.latency_floor(buf, n_kernels, stream=st)  # noqa: E731
    ms, _, _ = time_step(torch, fn, 1, stream, dev, steps, warmup, flush=flush, split=False)
    out = step_stats(ms)
    out["amortized"] = time_amortized(torch, fn, stream, dev, flush)
    return out


SMALL_WORKLOADS = ("decode", "dp_compact", "dp_padded", "lowbatch1")


def measure_small(torch, epx, wlmod, args, dev, stream, peak, flush, floors):
    """Step time of each small-batch workload in the same run (graph mode, L2
    flushed by a read between steps, automatic layout/dispatch choice)."""
    res = {}
    for name in SMALL_WORKLOADS:
        if name == args.workload:
            continue
        wl = wlmod.make(name, seed=args.seed)
        mode = step_mode(args, wl["T"], wl["k"])
        st = Step(torch, epx, wl, args, dev, mode)
        tot = st.prepare(stream)
        ms, rec_k, _ = time_step(torch, st.launch, len(st.calls), stream, dev, args.small_steps,
                                 max(3, args.warmup), flush=flush)
        stats = step_stats(ms)
        am = time_amortized(torch, st.launch, stream, dev, flush)
        b = alg_bytes(wl["T"], tot["T_real"], tot["N_recv"], tot["N_route"], wl["H"], wl["k"],
                      wl["R"], args.idx_bits // 8, fused=mode)
        kern = {n: statistics.median([r[i] - (r[i - 1] if i else 0.0) for r in rec_k]) * 1e3
                for i, n in enumerate(st.names)}
        floor = floors.get(st.n_kernels)
        res[name] = {
            "workload": DESCRIBE[name], "T_real": int(tot["T_real"]),
            "step_us_amortized": am, "step_us": stats,
            "tokens_per_s": tot["T_real"] / (am["median"] / 1e6),
            "alg_bytes": b["total"],
            "hbm_frac": b["total"] / (am["median"] / 1e6) / 1e9 / peak,
            "launches": st.n_kernels, "calls": st.names,
            "kernel_us_median_split": kern,
            "x_floor": (am["median"] / floor["amortized"]["median"]) if floor else None,
        }
    return res


# ---------------------------------------------------------------- epx arm

def run_epx(args):
    import torch
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl epx needs a CUDA GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    from combine_ep_layout_07_b200 import epx
    from combine_ep_layout_07_b200 import workloads as wlmod

    wl = wlmod.make(args.workload, seed=args.seed + rank)
    T, H, E, R, k = wl["T"], wl["H"], wl["E"], wl["R"], wl["k"]
    stream = torch.cuda.Stream(device=dev)
    mode = step_mode(args, T, k)
    step = Step(torch, epx, wl, args, dev, mode, two_stage=args.two_stage,
                no_expand=args.no_expand)
    tot = step.prepare(stream)
    lay, recv, expanded, y, out = step.lay, step.recv, step.expanded, step.y, step.out
    consumer = None
    if args.no_expand:
        consumer = time_consumers(torch, epx, lay, recv, expanded, y, stream, dev, tot, H,
                                  max(10, min(args.steps, 200)))

    part_bytes = None if step.part is None else step.part.element_size()
    bytes_ = step_alg_bytes(T, tot, H, k, R, args, part_bytes, mode)
    working = bytes_["total"]
    do_flush = args.flush == "always" or (args.flush == "auto" and working < 2 * L2_BYTES)
    l2flush = L2Flush(torch, dev)
    if do_flush:
        flush_desc = L2Flush.DESC
    elif working >= 2 * L2_BYTES:
        flush_desc = f"inputs larger than L2 ({working / 1e6:.0f} MB moved per step, no flush)"
    else:
        flush_desc = (f"hot L2: no flush between steps ({working / 1e6:.0f} MB moved per step, "
                      f"below 2x L2)")

    sampler = ClockSampler(gpu_uuid(torch, local)) if rank == 0 else None
    if sampler:
        sampler.start()
    step_ms, rec_k, (t_lo, t_hi) = time_step(
        torch, step.launch, len(step.calls), stream, dev, args.steps, args.warmup,
        flush=l2flush if do_flush else None, eager=args.eager, split=True, pg=pg)
    if sampler:
        sampler.stop()
    amortized = None
    if do_flush and not args.eager:
        amortized = time_amortized(torch, step.launch, stream, dev, l2flush)
    # the paired call's two kernels cannot be split by events without
    # undoing their overlap: the per-kernel times of the roofline come from a
    # split pass of the same step as separate calls (layout, dispatch_expand)
    sep_ms = sep_bytes = None
    if mode == "paired" and not args.eager:
        sep_calls = step.calls_for("separate")
        _, rec_sep, _ = time_step(
            torch, lambda st, ev=None: step.launch(st, ev, sep_calls), len(sep_calls), stream,
            dev, args.steps, args.warmup, flush=l2flush if do_flush else None, split=True,
            pg=pg)
        sep_ms = {n: [r[i] - (r[i - 1] if i else 0.0) for r in rec_sep]
                  for i, (n, _) in enumerate(sep_calls)}
        sep_bytes = step_alg_bytes(T, tot, H, k, R, args, part_bytes, "separate")
    names = step.names
    k_ms = {n: [r[i] - (r[i - 1] if i else 0.0) for r in rec_k] for i, n in enumerate(names)}
    total_ms = reduce_max(pg, sum(step_ms), dev)
    value = whole_job_value(tot["T_real"] * args.steps, world, total_ms)

    # ---- e2e through the host-buffer C-ABI call
    e2e = None if args.no_e2e else run_e2e(torch, epx, wl, args, dev, stream, pg, world,
                                           tot["T_real"])

    peak, peak_kind = load_peaks()
    # ---- latency floor and the small-batch workloads, same run, same protocol
    floors, small, small_clocks = {}, None, None
    if args.small_steps > 0 and rank == 0:
        # clocks sampled over this phase too: a latency-bound step follows the
        # SM clock, which may differ from the headline's timed region
        sampler2 = ClockSampler(gpu_uuid(torch, local))
        sampler2.start()
        s_lo = time.time()
        n_floor = max(3, min(args.small_steps, 1000))
        for n in (2, 3):
            floors[n] = time_floor(torch, epx, stream, dev, n, n_floor, max(3, args.warmup),
                                   l2flush)
        small = measure_small(torch, epx, wlmod, args, dev, stream, peak, l2flush, floors)
        s_hi = time.time()
        sampler2.stop()
        small_clocks = sampler2.summary(s_lo, s_hi)

    if rank != 0:
        finish(pg)
        return 0

    def kernel_stats(ms_by_name, nbytes):
        out = {}
        for name, ms in ms_by_name.items():
            avg_s = statistics.fmean(ms) / 1e3
            gbs = nbytes[name] / avg_s / 1e9
            out[name] = {"us": avg_s * 1e6, "us_median": statistics.median(ms) * 1e3,
                         "alg_bytes": nbytes[name], "gbs": gbs, "frac": gbs / peak}
        return out

    kernels = kernel_stats(k_ms, bytes_)
    kernels_sep = kernel_stats(sep_ms, sep_bytes) if sep_ms else None
    roof_k = kernels_sep or kernels
    dom = max(roof_k, key=lambda n: roof_k[n]["us"])
    engine = {"dispatch": "recv_only", "expand_index": "gather_index",
              "combine_local": "two_stage_" + str(args.two_stage),
              "combine_epilogue": "two_stage_" + str(args.two_stage),
              "layout_dispatch_expand": mode,
              "dispatch_expand": "bulk" if args.dispatch_variant == 2 or
              (args.dispatch_variant == 0 and T >= 1024) else "vec",
              "combine_reduce": "warp_per_token" if args.combine_variant == 1 else "split",
              "layout": {1: "warp_chunks", 2: "count_matrix", 3: "grid"}.get(
                  args.layout_variant, layout_auto_engine(T, k))}
    traffic = committed_traffic(dom, args.workload, engine.get(dom))
    roofline = {"bound": "hbm", "kernel": dom, "achieved": roof_k[dom]["gbs"], "peak": peak,
                "unit": "GB/s", "frac": roof_k[dom]["gbs"] / peak,
                "timed_in": ("split pass of the step as separate calls (the paired call's "
                             "kernels are not split by events)") if kernels_sep else
                "split pass of the step's calls",
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind ==
                "measured" else "fallback 6.65 TB/s",
                "traffic": traffic}
    step_gbs = bytes_["total"] / (total_ms / args.steps / 1e3) / 1e9

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, args, tot, flush_desc, mode),
        "roofline": roofline,
        "step_hbm": {"alg_bytes": bytes_["total"], "gbs": step_gbs, "frac": step_gbs / peak},
        "step_us": step_stats(step_ms),
        **({"step_us_amortized": amortized} if amortized else {}),
        "kernels": kernels,
        **({"kernels_separate_calls": kernels_sep} if kernels_sep else {}),
        "gpu_launches": step.n_kernels * args.steps,
        **({"consumer": consumer} if consumer else {}),
        "e2e": e2e,
    }
    if floors:
        line["floor_us"] = {
            str(n): dict(v, what=f"{n} chained one-warp launches (programmatic dependent launch),"
                                 " one global load each after its wait, graph-timed like the "
                                 "step, L2 flushed by a read")
            for n, v in floors.items()}
    if small:
        line["small_batch"] = small
        line["small_batch_clocks"] = small_clocks
    if sampler:
        line["clocks"] = sampler.summary(t_lo, t_hi)
    if world == 1 and not args.no_cpu_baseline:
        cb, ores = cpu_baseline(wl, args.cpu_budget, args.idx_bits)
        line["cpu_baseline"] = cb
        line["parity"] = parity_summary(torch, lay, expanded, out, ores)
    print(json.dumps(line), flush=True)
    finish(pg)
    return 0


def time_consumers(torch, epx, lay, recv, expanded, y, stream, dev, tot, H, n):
    """The stand-in expert reading the expanded copy vs reading recv through
    the gather index (CUDA events, eager, n calls each)."""
    src = epx.expand_index(lay, stream=stream)
    res = {}
    for name, fn in (("from_expanded", lambda: epx.standin_expert(expanded, lay, y=y,
                                                                     stream=stream)),
                     ("gather_from_recv", lambda: epx.standin_expert_gather(
                         recv, lay, src, y=y, stream=stream))):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = {"us": e0.elapsed_time(e1) * 1e3 / n}
    row = H * 2
    res["from_expanded"]["alg_bytes"] = 2 * tot["N_route"] * row
    res["gather_from_recv"]["alg_bytes"] = tot["N_recv"] * row + tot["N_route"] * (row + 4)
    res["expanded_bytes_not_written"] = tot["N_route"] * row
    return res


def parity_summary(torch, lay, expanded, out, ores):
    """Whole-output comparison with the oracle on the benchmarked workload."""
    from combine_ep_layout_07_b200 import workloads as wlmod
    o = ores["layout"]
    pos_ok = bool(np.array_equal(lay.pos.cpu().numpy(), o["pos"]))
    ne = o["N_route"]
    ex = expanded[:ne].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    ex_ok = bool(np.array_equal(ex, ores["expanded"]))
    g = wlmod.bf16_bits_to_f32(out.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))
    r = wlmod.bf16_bits_to_f32(ores["out"])
    ok = bool(np.all(np.abs(g - r) <= 2.0 ** -7 * np.abs(r) + 1e-3))
    return {"layout_pos_bit_exact": pos_ok, "expanded_bit_exact": ex_ok,
            "combine_within_tol": ok}


E2E_STREAMS = 3


def run_e2e(torch, epx, wl, args, dev, stream, pg, world, T_real):
    """The metric through ep_roundtrip_host with pinned host buffers: every
    step copies its inputs host -> device, runs layout, dispatch/expand, the
    stand-in expert and combine, and copies the output back.  Steps rotate
    over E2E_STREAMS streams with their own device scratch and output buffer,
    so one step's upload overlaps the others' compute and download (the link
    is full duplex; with three streams an upload is always queued while a
    stream's own download runs) -- what a caller pipelining the public call
    gets."""
    T, H, E, R, k = wl["T"], wl["H"], wl["E"], wl["R"], wl["k"]
    itype = torch.int64 if args.idx_bits == 64 else torch.int32
    x_h = torch.from_numpy(wl["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    i_h = torch.from_numpy(wl["topk_idx"]).to(itype).pin_memory()
    w_h = torch.from_numpy(wl["topk_weights"]).pin_memory()
    nbytes = epx.roundtrip_device_bytes(T, H, k, E, R, args.idx_bits)
    streams = [stream] + [torch.cuda.Stream(device=dev) for _ in range(E2E_STREAMS - 1)]
    dmem = [torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in streams]
    out_h = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in streams]
    n = max(1, args.e2e_steps)
    ns = len(streams)
    for i in range(2 * ns):
        epx.roundtrip_host(x_h, i_h, w_h, E, R, dmem[i % ns], out_h[i % ns],
                           stream=streams[i % ns])
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    ends = [torch.cuda.Event(enable_timing=True) for _ in streams]
    e0.record(streams[0])
    for st in streams[1:]:
        st.wait_event(e0)
    for i in range(n):
        s = i % ns
        epx.roundtrip_host(x_h, i_h, w_h, E, R, dmem[s], out_h[s], stream=streams[s])
    for s, ev in zip(streams, ends):
        ev.record(s)
    torch.cuda.synchronize(dev)
    ms = reduce_max(pg, max(e0.elapsed_time(ev) for ev in ends), dev)
    h2d = x_h.numel() * 2 + i_h.numel() * i_h.element_size() + w_h.numel() * 4
    d2h = out_h[0].numel() * 2
    return {"value": whole_job_value(T_real * n, world, ms), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "path": "ep_roundtrip_host per step (pinned host -> device, layout, "
                    "dispatch/expand, stand-in expert, combine, device -> host), steps "
                    f"rotating over {ns} streams"}


def reduce_max(pg, value: float, device) -> float:
    """Max of a per-rank float over all ranks (identity without a group)."""
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: units every rank processed over the slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


def finish(pg):
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_epx(args)


if __name__ == "__main__":
    sys.exit(main())
