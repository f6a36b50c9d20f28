#!/usr/bin/env python
"""Throughput benchmark: weights quantized per second through the whole hot
path on B200 -- imatrix -> group-scale search with fused RTN + pack ->
dequant -> imatrix-weighted proxy error -- one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config c1] [--impl tq|reference]

A step is one pass of every row of the path over one batch of synthetic input
(the workload named by --config; default: the dense int4-g128 4096 x 4096
workload).  `value` is device-timed with inputs resident in HBM (CUDA events,
barrier + synchronize on both sides, max over ranks); `e2e` repeats the step
through the public API starting from pinned host buffers, with the host->device
copies of the inputs and the device->host read of the results inside the
timed region.  `roofline` reports the dominant kernel (the search) against the
FP32 CUDA-core issue peak.  Under torchrun every rank quantizes its own
independent copy of the workload (weak scaling; no collective on the data
path).  --impl reference times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "weights quantized/sec (search+pack) on 1 B200; % of FP32 / HBM roofline"
L2_BYTES = 126 * 2 ** 20
# FP32 lane-instructions per weight of the search (the dominant kernel):
# candidate-element evaluations per weight x instructions per evaluation
# (sym int3: 96 x 7; asym int4: 1024 x 5; NVFP4: 16 x 10).
SEARCH_INSTR_PER_W = {"int3_g64_sym": 96 * 7, "int4_g128_asym": 1024 * 5, "nvfp4_g16": 16 * 10}
SEARCH_CEE_PER_W = {"int3_g64_sym": 96, "int4_g128_asym": 1024, "nvfp4_g16": 16}
# our kernels per call: imatrix 2 (partial + final), search 1 (NVFP4: amax +
# global + search = 3), dequant 1, proxy 1
KERNELS = {"imatrix": 2, "search": {"int3_g64_sym": 1, "int4_g128_asym": 1, "nvfp4_g16": 3},
           "dequant": 1, "proxy": 1}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "bf16_tflops": 1590.0, "source": "fallback"}
    f = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(f):
        d = json.load(open(f))
        p = {"hbm_gbs": d.get("hbm_gbs", 6650.0), "sm_max_mhz": d.get("sm_max_mhz", 1965.0),
             "bf16_tflops": d.get("bf16_tflops", 1590.0), "source": "measured"}
    return p


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        self.rows = []
        self.proc = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
            if not self.uuid.startswith("GPU-"):
                self.uuid = "GPU-" + self.uuid
        except Exception:
            self.uuid = None

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm = [float(r[0]) for r in self.rows if len(r) >= 7 and r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if len(r) >= 7 and r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows if len(r) >= 7 for i in range(4)
                          if r[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sm)}


# ------------------------------------------------------------------ the step

class Step:
    """One pass of the whole path over one input set, on the current stream."""

    def __init__(self, tq, wl, sets):
        self.tq = tq
        self.wl = wl
        self.sets = sets            # list of (sites dict name->X, units list of W)
        self.fmts = [tq.FORMATS[u.fmt] for u in wl.units if u.timed]
        self.units = [u for u in wl.units if u.timed]
        dev = self.units[0].W.device
        # preallocated outputs and workspaces (the timed region allocates nothing)
        self.m = {}
        self.ws_im = {}
        for name, site in wl.sites.items():
            if not any(u.site == name for u in self.units):
                continue
            X = site.X
            self.m[name] = torch.zeros((X.shape[0], X.shape[2]), dtype=torch.float32, device=dev)
            self.ws_im[name] = torch.empty(max(16, tq.imatrix_workspace_bytes(X)), dtype=torch.uint8, device=dev)
        self.res, self.dq, self.px, self.ws_px = [], [], [], []
        for u, fmt in zip(self.units, self.fmts):
            E, O, I = u.W.shape
            m = self._m_for(u)
            self.res.append(tq.tq_search_groups(u.W, m, fmt))
            self.dq.append(torch.empty((E, O, I), dtype=torch.bfloat16, device=dev))
            self.px.append((torch.empty(E, dtype=torch.float64, device=dev),
                            torch.empty(E, dtype=torch.float64, device=dev)))
            self.ws_px.append(torch.empty(max(16, tq.proxy_workspace_bytes(u.W, fmt)), dtype=torch.uint8,
                                          device=dev))
        self.search_events = []
        self.row_events = []

    def _m_for(self, u):
        m = self.m[u.site]
        return m if u.W.shape[0] > 1 else m[0]

    def kernels_per_step(self):
        n = KERNELS["imatrix"] * len(self.m)
        for u in self.units:
            n += KERNELS["search"][u.fmt] + KERNELS["dequant"] + KERNELS["proxy"]
        return n

    def __call__(self, k: int, time_search: bool = False):
        tq = self.tq
        sites, Ws = self.sets[k % len(self.sets)]

        def mark():
            if not time_search:
                return None
            ev = torch.cuda.Event(enable_timing=True)
            ev.record()
            return ev

        for name in self.m:
            X = sites[name]
            a = mark()
            tq.tq_imatrix(X, m=self.m[name], alpha=1.0 / X.shape[1], workspace=self.ws_im[name])
            if time_search:
                self.row_events.append(("imatrix", X.numel() * X.element_size(), a, mark()))
        for i, (u, fmt) in enumerate(zip(self.units, self.fmts)):
            W = Ws[i]
            m = self._m_for(u)
            E, O, I = W.shape
            a = mark()
            r = tq.tq_search_groups(W, m, fmt, out=self.res[i])
            if time_search:
                b = mark()
                self.search_events.append((u.fmt, W.numel(), a, b))
            tq.tq_dequant(r.packed, fmt, r.scales, r.zeros, r.global_scale, E, O, I, out=self.dq[i])
            if time_search:
                c = mark()
                self.row_events.append(("dequant", r.packed.numel() + self.dq[i].numel() * 2
                                        + r.scales.numel() * r.scales.element_size()
                                        + (0 if r.zeros is None else r.zeros.numel()), b, c))
            tq.tq_proxy_error(W, r.packed, fmt, r.scales, r.zeros, r.global_scale, m, out=self.px[i],
                              workspace=self.ws_px[i])
            if time_search:
                self.row_events.append(("proxy", W.numel() * W.element_size() + r.packed.numel()
                                        + r.scales.numel() * r.scales.element_size()
                                        + (0 if r.zeros is None else r.zeros.numel()), c, mark()))


def make_sets(wl, n_sets):
    """Input sets rotated through HBM so that no step finds its inputs in L2
    (set 0 is the workload itself, the others are copies)."""
    units = [u for u in wl.units if u.timed]
    sets = [({k: v.X for k, v in wl.sites.items()}, [u.W for u in units])]
    for _ in range(1, n_sets):
        sets.append(({k: v.X.clone() for k, v in wl.sites.items()}, [u.W.clone() for u in units]))
    return sets


def input_bytes(wl):
    b = sum(u.W.numel() * u.W.element_size() for u in wl.units if u.timed)
    b += sum(s.X.numel() * s.X.element_size() for s in wl.sites.values())
    return b


# ------------------------------------------------------------------ CPU oracle baseline

def oracle_sample(wl, budget_s: float = 12.0):
    """Times the oracle (as it stands) on a bounded sample of the workload:
    for each unit, the imatrix of its site (first matrix) and search + pack +
    dequant + proxy error over the first rows of its first matrix, the row
    count sized to about `budget_s` seconds.  Returns (weights/s, cores,
    description, seconds)."""
    import oracle
    oracle.build()
    units = [u for u in wl.units if u.timed]
    # size the sample: rows per unit so that the search takes ~budget_s in total
    probe_rows = 8
    t0 = time.perf_counter()
    for u in units[:1]:
        _oracle_unit(oracle, wl, u, probe_rows)
    per_row = (time.perf_counter() - t0) / probe_rows
    rows = max(8, min(units[0].W.shape[1], int(budget_s / max(per_row, 1e-6))))
    t0 = time.perf_counter()
    n = 0
    for u in units:
        r = min(rows, u.W.shape[1])
        _oracle_unit(oracle, wl, u, r)
        n += r * u.W.shape[2]
    dt = time.perf_counter() - t0
    desc = (f"oracle (C, fp64, OpenMP) on {rows} rows of the first matrix of each of {len(units)} unit(s) "
            f"= {n} weights: imatrix of the site's columns over all tokens, search+pack, dequant, proxy")
    return n / dt, oracle.num_threads(), desc, dt


def oracle_one_thread(config: str, frac: float = 0.01):
    """The same oracle on one host thread (OMP_NUM_THREADS=1 in a child
    process, so the parent's thread pool is untouched) over a fixed `frac` of
    the first unit's rows: the scaling reference for the multi-core figure.
    Returns (weights/s, description) or None if the child fails."""
    import subprocess
    code = (f"import json, time, synth, bench, oracle; oracle.build(); wl = synth.make({config!r}, 'cpu'); "
            f"u = [x for x in wl.units if x.timed][0]; rows = max(8, int(u.W.shape[1] * {frac!r})); "
            f"t0 = time.perf_counter(); bench._oracle_unit(oracle, wl, u, rows); dt = time.perf_counter() - t0; "
            f"print(json.dumps([rows * u.W.shape[2] / dt, rows, u.W.shape[2], oracle.num_threads(), dt]))")
    env = dict(os.environ, OMP_NUM_THREADS="1")
    try:
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300, env=env,
                           cwd=os.path.dirname(os.path.abspath(__file__)))
        v, rows, cols, threads, dt = json.loads(r.stdout.strip().splitlines()[-1])
    except Exception:   # noqa: BLE001 -- the figure is optional context
        return None
    return v, (f"{rows} rows x {cols} of the first unit ({frac:.0%}), {threads} thread, imatrix of the site "
               f"+ search+pack + dequant + proxy, {dt:.1f} s")


def _oracle_unit(oracle, wl, u, rows):
    X = wl.sites[u.site].X[0].float().cpu().numpy()
    m = oracle.imatrix(X).astype(np.float32)
    W = u.W[0, :rows].float().cpu().numpy()[None]
    if u.fmt == "int3_g64_sym":
        s, i, L, v = oracle.search_sym_int3(W, m)
        oracle.pack_int3(v[0])
        What = oracle.dequant_int3(v[0], s[0])
    elif u.fmt == "int4_g128_asym":
        s, z, i, L, q = oracle.search_asym_int4(W, m)
        oracle.pack_nibbles(q[0], 128, z[0])
        What = oracle.dequant_int4(q[0], s[0], z[0])
    else:
        g = oracle.nvfp4_global(u.W[0].float().cpu().numpy())
        g, sc, i, L, c = oracle.search_nvfp4(W, m, gscale=g)
        oracle.pack_nibbles(c[0], 16)
        What = oracle.dequant_nvfp4(c, sc, g)[0]
    oracle.proxy_error(W[0], What, m)


def read_traffic(path, workload):
    """DRAM bytes per launch of the dominant kernel from the profiles table."""
    try:
        for line in open(path):
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) >= 3 and cells[0] == workload and cells[2].isdigit():
                return int(cells[2])
    except OSError:
        pass
    return None


# ------------------------------------------------------------------ main

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="c1", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--scale", type=float, default=1.0,
                    help="shrink the workload (profiling and tests only; the reported line is for scale 1)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--traffic-table", default=os.path.join(ROOT, "profiles", "traffic.md"),
                    help="ncu DRAM bytes per launch of the dominant kernel, by workload")
    ap.add_argument("--jsonl", default=None,
                    help="also append the result line, with a UTC time stamp and the git revision, to this file")
    return ap.parse_args()


def append_jsonl(path, line):
    """Run log: the JSON result line plus when and from which revision."""
    rec = dict(line)
    rec["time_utc"] = datetime.datetime.now(datetime.timezone.utc).isoformat(timespec="seconds")
    try:
        rec["git"] = subprocess.run(["git", "rev-parse", "--short", "HEAD"], cwd=ROOT, capture_output=True,
                                    text=True, timeout=10).stdout.strip() or None
    except Exception:   # noqa: BLE001 -- a copy without git history still logs
        rec["git"] = None
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def reference_arm(args, world, rank):
    if rank != 0:
        return 0
    wl = synth.make(args.config, "cpu", seed=0)
    nw = wl.n_weights
    vals = []
    for _ in range(args.warmup):
        oracle_sample(wl, budget_s=2.0)
    desc = cores = None
    for _ in range(args.steps):
        v, cores, desc, dt = oracle_sample(wl, budget_s=4.0)
        vals.append(v)
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "weights/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": nw / v * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": f"{args.config}: {synth.DESCRIPTIONS[args.config]}", "weights": nw},
            "cpu_baseline": {"value": v, "unit": "weights/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": v, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if args.jsonl:
        append_jsonl(args.jsonl, line)
    return 0


def main():
    args = parse()
    assert args.warmup >= 3 or args.impl == "reference", "at least 3 warm-up steps"
    if args.impl == "reference":   # rank 0 alone times the oracle; no process group
        return reference_arm(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))

    import group_scale_search_b200 as tq
    from group_scale_search_b200.dist import init_from_env, max_over_ranks
    world, rank, local = init_from_env("nccl", timeout_s=120.0)
    if world == 1:
        torch.cuda.set_device(0)
    tq.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = synth.make(args.config, dev, seed=rank, scale=args.scale)
    nbytes = input_bytes(wl)
    n_sets = max(1, min(64, math.ceil(2 * L2_BYTES / nbytes)))
    sets = make_sets(wl, n_sets)
    step = Step(tq, wl, sets)
    nw = sum(u.W.numel() for u in step.units)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        ev0.record(stream)
        for k in range(args.steps):
            step(k, time_search=True)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    ms_step = ms / args.steps
    value = world * nw / (ms_step * 1e-3)

    # dominant kernel: the search (CUDA events on the launching stream)
    by_fmt = {}
    for fmt, n, a, b in step.search_events:
        d = by_fmt.setdefault(fmt, [0.0, 0])
        d[0] += a.elapsed_time(b)
        d[1] += n
    fmt_main = max(by_fmt, key=lambda f: by_fmt[f][0])
    search_ms = by_fmt[fmt_main][0] / args.steps
    w_per_launch = by_fmt[fmt_main][1] / args.steps
    pk = peaks()
    props = torch.cuda.get_device_properties(dev)
    sms = props.multi_processor_count
    peak_tinst = sms * 128 * pk["sm_max_mhz"] * 1e6 / 1e12
    achieved = SEARCH_INSTR_PER_W[fmt_main] * w_per_launch / (search_ms * 1e-3) / 1e12
    traffic = read_traffic(args.traffic_table, args.config)
    clocks = clk.summary()
    roofline = {"bound": "alu", "achieved": achieved, "peak": peak_tinst, "unit": "Tinst/s",
                "frac": achieved / peak_tinst, "traffic": traffic,
                "kernel": f"search {fmt_main}", "kernel_ms": search_ms,
                "per_unit": f"{SEARCH_INSTR_PER_W[fmt_main]} FP32 lane-instr/weight "
                            f"({SEARCH_CEE_PER_W[fmt_main]} candidate-element evaluations)",
                "peak_basis": f"{sms} SMs x 128 FP32 lanes x {pk['sm_max_mhz']:.0f} MHz ({pk['source']} max clock)",
                "frac_at_observed_clock": (achieved / (sms * 128 * clocks["sm_mhz"] * 1e6 / 1e12))
                if clocks.get("sm_mhz") else None,
                "cee_per_s": SEARCH_CEE_PER_W[fmt_main] * w_per_launch / (search_ms * 1e-3)}

    # every HBM-bound row of the step: algorithmic bytes / CUDA-event time vs the HBM peak
    rows = {}
    for name, nbytes, a, b in step.row_events:
        d = rows.setdefault(name, [0.0, 0])
        d[0] += a.elapsed_time(b)
        d[1] += nbytes
    hbm_rows = {}
    for name, (t_ms, nbytes) in rows.items():
        gbs = nbytes / (t_ms * 1e-3) / 1e9
        hbm_rows[name] = {"ms": t_ms / args.steps, "bytes": nbytes // args.steps, "GB/s": gbs,
                          "frac": gbs / pk["hbm_gbs"]}
    hbm_rows["pack"] = time_pack(tq, step, pk)
    next_rows = {"dequant_gemv": {f"B={B}": time_gemv(tq, step, pk, B) for B in (1, 8)}}
    if step.units[0].fmt == "int4_g128_asym":
        next_rows["asym_ladder_256_64"] = time_ladder(tq, step, peak_tinst)
        next_rows["int4_g64"] = time_int4_g64(tq, step, pk, peak_tinst)
    next_rows["hessian"] = time_hessian(tq, step, pk)
    next_rows["proxy_full_hessian"] = time_proxy_full(tq, step, pk)
    next_rows["gptq_sweep"] = time_gptq(tq, step, peak_tinst)
    next_rows["fp8_tensor"] = time_fp8(tq, step, pk, peak_tinst)
    next_rows["lloyd_max_2bit"] = time_lloyd(tq, step, pk)

    # end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(tq, wl, step, args, world, barrier, dev)

    line = {"metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"{args.config}: {synth.DESCRIPTIONS[args.config]}"
                                   + ("" if args.scale == 1.0 else f" (scaled x{args.scale})"),
                       "weights_per_gpu": nw,
                       "groups_per_gpu": sum(tq.tq_num_groups(tq.FORMATS[u.fmt], u.W.shape[0] * u.W.shape[1],
                                                              u.W.shape[2]) for u in step.units),
                       "step": "imatrix + search with fused RTN/pack + dequant(bf16) + proxy error",
                       "l2": (f"{n_sets} rotating input sets, {n_sets * nbytes / 2**20:.0f} MiB > 126 MiB L2"
                              if n_sets * nbytes > L2_BYTES else
                              f"{n_sets} input sets ({n_sets * nbytes / 2**20:.1f} MiB) fit in L2"),
                       "parallelism": f"weak x{world}: independent workload per GPU"},
            "groups_per_s": value / tq.tq_group_size(tq.FORMATS[fmt_main]),
            "roofline": roofline, "hbm_rows": hbm_rows, "next_rows": next_rows, "clocks": clocks, "e2e": e2e,
            "gpu_launches": step.kernels_per_step() * args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, desc, dt = oracle_sample(wl)
        line["cpu_baseline"] = {"value": v, "unit": "weights/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": dt}
        one = oracle_one_thread(args.config)
        if one is not None:
            line["cpu_baseline"]["one_thread"] = {"value": one[0], "unit": "weights/s", "sample": one[1]}
    if rank == 0:
        print(json.dumps(line), flush=True)
        if args.jsonl:
            append_jsonl(args.jsonl, line)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def time_pack(tq, step, pk, reps=12):
    """tq_pack (RTN + pack with given scales, the stand-alone form of the fused
    pack) on the first unit, outside the step, rotating through the input
    sets: bytes = weights read + packed records written + scales (+ zeros) read."""
    u, r = step.units[0], step.res[0]
    fmt = tq.FORMATS[u.fmt]
    out = torch.empty_like(r.packed)
    Ws = [s[1][0] for s in step.sets]
    nbytes = (u.W.numel() * u.W.element_size() + out.numel() + r.scales.numel() * r.scales.element_size()
              + (0 if r.zeros is None else r.zeros.numel()))
    for k in range(3):
        tq.tq_pack(Ws[k % len(Ws)], fmt, r.scales, r.zeros, r.global_scale, out=out)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for k in range(reps):
        tq.tq_pack(Ws[k % len(Ws)], fmt, r.scales, r.zeros, r.global_scale, out=out)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms": ms, "bytes": nbytes, "GB/s": gbs, "frac": gbs / pk["hbm_gbs"],
            "note": f"first unit, back-to-back launches over {len(Ws)} rotating weight copies"}


def time_ladder(tq, step, peak_tinst, reps=3):
    """The int4 search on the "256/64" grid (256 scales x 64 zero-points: 16
    distinct zero-points, 4096 candidate-element evaluations per weight, 4x
    the default grid's) on the first unit, rotating weight copies; the same
    per-evaluation instruction figure as the default grid's roofline."""
    u = step.units[0]
    m = step._m_for(u)
    p = tq.SearchParams(asym_n_scale=256, asym_n_zero=64)
    Ws = [s[1][0] for s in step.sets]
    res = tq.tq_search_groups(Ws[0], m, tq.INT4_G128_ASYM, params=p)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for k in range(reps):
        tq.tq_search_groups(Ws[k % len(Ws)], m, tq.INT4_G128_ASYM, params=p, out=res)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    nw = u.W.numel()
    cee = 256 * 16
    achieved = cee * 5 * nw / (ms * 1e-3) / 1e12
    return {"ms": ms, "weights_per_s": nw / (ms * 1e-3), "cee_per_s": cee * nw / (ms * 1e-3),
            "achieved_tinst": achieved, "frac": achieved / peak_tinst,
            "note": f"first unit, {reps} launches, 4096 candidate-element evaluations x 5 instr per weight"}


def time_int4_g64(tq, step, pk, peak_tinst, reps=5):
    """The int4-g64 format on the first unit: the joint search with fused RTN
    and pack (1024 candidate-element evaluations per weight, as for g128)
    against the FP32 issue roofline, and the bf16 dequantization against HBM
    (records 0.5 B + scale and zero 5/64 B read, 2 B written per weight)."""
    u = step.units[0]
    m = step._m_for(u)
    fmt = tq.INT4_G64_ASYM
    Ws = [s[1][0] for s in step.sets]
    E, O, I = u.W.shape
    res = tq.tq_search_groups(Ws[0], m, fmt)
    dq = torch.empty((E, O, I), dtype=torch.bfloat16, device=u.W.device)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record()
    for k in range(reps):
        tq.tq_search_groups(Ws[k % len(Ws)], m, fmt, out=res)
    ev[1].record()
    for k in range(reps):
        tq.tq_dequant(res.packed, fmt, res.scales, res.zeros, None, E, O, I, out=dq)
    ev[2].record()
    torch.cuda.synchronize()
    ms_s = ev[0].elapsed_time(ev[1]) / reps
    ms_d = ev[1].elapsed_time(ev[2]) / reps
    nw = u.W.numel()
    ach = 1024 * 5 * nw / (ms_s * 1e-3) / 1e12
    dbytes = res.packed.numel() + res.scales.numel() * 4 + res.zeros.numel() + dq.numel() * 2
    return {"search_ms": ms_s, "search_frac": ach / peak_tinst, "search_weights_per_s": nw / (ms_s * 1e-3),
            "dequant_ms": ms_d, "dequant_frac": dbytes / (ms_d * 1e-3) / 1e9 / pk["hbm_gbs"],
            "note": f"first unit, {reps} launches each; search: 1024 evaluations x 5 instr per weight vs the "
                    "FP32 issue peak; dequant: bytes vs measured HBM (the records are L2-resident when small)"}


# FP32-issue work of one FP8 candidate-element evaluation in k_fp8_loss
# (ncu instruction count of the kernel per evaluation, rounded).
FP8_INSTR_PER_CEE = 14


def time_fp8(tq, step, pk, peak_tinst, reps=3):
    """FP8 (E4M3) per-tensor scale search on the first unit (amax, 64
    candidate losses per weight in fp64, the pick, the fused pack of the
    codes), rotating weight copies; CEE/s and the fraction of the FP32 issue
    peak at FP8_INSTR_PER_CEE instructions per evaluation."""
    u = step.units[0]
    m = step._m_for(u)
    Ws = [s[1][0] for s in step.sets]
    res = tq.tq_search_fp8(Ws[0], m)
    ws = torch.empty(max(16, tq.lib().tq_fp8_workspace_bytes(ctypes.byref(tq._mat(Ws[0], "W")))),
                     dtype=torch.uint8, device=u.W.device)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for k in range(reps):
        tq.tq_search_fp8(Ws[k % len(Ws)], m, out=res, workspace=ws)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    nw = u.W.numel()
    cee = 64 * nw / (ms * 1e-3)
    return {"ms": ms, "weights_per_s": nw / (ms * 1e-3), "cee_per_s": cee,
            "frac": cee * FP8_INSTR_PER_CEE / 1e12 / peak_tinst,
            "note": f"first unit, {reps} launches of the whole call (amax + losses + pick + pack); "
                    f"{FP8_INSTR_PER_CEE} FP32-issue instructions per candidate-element evaluation"}


def time_lloyd(tq, step, pk, n_iter=16, reps=3):
    """Lloyd-Max 2-bit codebook (16 iterations) and codes on the first unit:
    one HBM pass over W (+ the imatrix, L2-resident) per iteration, one for
    the scales and one for the codes; bytes = (n_iter + 3) x W + scales +
    packed codes."""
    u = step.units[0]
    m = step._m_for(u)
    Ws = [s[1][0] for s in step.sets]
    r = tq.tq_lloyd_max_g32(Ws[0], m, n_iter=n_iter)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for k in range(reps):
        tq.tq_lloyd_max_g32(Ws[k % len(Ws)], m, n_iter=n_iter)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    wb = u.W.numel() * u.W.element_size()
    nbytes = (n_iter + 3) * wb + r.scales.numel() * 4 * (n_iter + 3) + r.packed.numel()
    return {"ms": ms, "iterations": n_iter, "bytes": nbytes, "GB/s": nbytes / (ms * 1e-3) / 1e9,
            "frac": nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            "note": f"first unit, {reps} calls (binding allocations included); {n_iter} iterations, one pass each"}


def time_hessian(tq, step, pk):
    """tq_hessian (H = X^T X on the tensor cores) on the first unit's
    calibration activations (one matrix: the first expert of a MoE site),
    rotating through the input sets.  Algorithmic work: the distinct entries
    of the symmetric H, T I (I + 1) flops; peak: the measured dense bf16
    figure."""
    u = step.units[0]
    Xs = [s[0][u.site][0] for s in step.sets]
    T, I = Xs[0].shape
    H = torch.empty((I, I), dtype=torch.float32, device=Xs[0].device)
    flops = T * I * (I + 1)
    tq.tq_hessian(Xs[0], out=H)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    tq.tq_hessian(Xs[0], out=H)
    b.record()
    torch.cuda.synchronize()
    reps = max(3, min(50, int(0.03 / max(a.elapsed_time(b) * 1e-3, 1e-6))))
    a.record()
    for k in range(reps):
        tq.tq_hessian(Xs[k % len(Xs)], out=H)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    tf = flops / (ms * 1e-3) / 1e12
    peak = pk["bf16_tflops"]
    # roofline: the slower of the tensor work and the HBM traffic (X read once, H written)
    nbytes = T * I * 2 + I * I * 4
    t_min = max(flops / (peak * 1e12), nbytes / (pk["hbm_gbs"] * 1e9))
    return {"ms": ms, "T": T, "I": I, "flops": flops, "TFLOP/s": tf, "peak": peak, "frac_tensor": tf / peak,
            "bytes": nbytes, "bound": "tensor" if flops / (peak * 1e12) >= nbytes / (pk["hbm_gbs"] * 1e9) else "hbm",
            "frac": t_min / (ms * 1e-3),
            "note": f"first unit's activations [{T}, {I}] bf16, {reps} launches over {len(Xs)} input sets; "
                    "H fp32 both triangles; frac = roofline time (slower of flops / measured dense bf16 "
                    "burst and bytes / measured HBM) / measured time"}


def time_proxy_full(tq, step, pk):
    """tq_proxy_error_full (tr(E H E^T), tr(W H W^T) with H = X^T X, never
    formed) on the first unit's search output and calibration activations,
    rotating through the input sets.  Algorithmic work: the two products
    X E^T and X W^T, 4 T O I flops per matrix (the kernel issues 6 T O I:
    E enters as two bf16 pieces); peak: the measured dense bf16 figure."""
    u, r = step.units[0], step.res[0]
    fmt = tq.FORMATS[u.fmt]
    sets = [(s[0][u.site], s[1][0]) for s in step.sets]
    X0, W0 = sets[0]
    if W0.dtype != torch.bfloat16 or X0.dtype != torch.bfloat16:
        return {"skipped": "the tensor-core path takes bf16 weights and activations"}
    E, O, I = W0.shape
    T = X0.shape[-2]
    flops = 4 * E * T * O * I
    ws = torch.empty(tq.proxy_full_workspace_bytes(X0, W0), dtype=torch.uint8, device=W0.device)
    out = (torch.empty(E, dtype=torch.float64, device=W0.device), torch.empty(E, dtype=torch.float64, device=W0.device))

    def call(k):
        X, W = sets[k % len(sets)]
        tq.tq_proxy_error_full(X, W, r.packed, fmt, r.scales, r.zeros, r.global_scale, out=out, workspace=ws)

    call(0)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    call(0)
    b.record()
    torch.cuda.synchronize()
    reps = max(3, min(50, int(0.03 / max(a.elapsed_time(b) * 1e-3, 1e-6))))
    a.record()
    for k in range(reps):
        call(k)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    tf = flops / (ms * 1e-3) / 1e12
    peak = pk["bf16_tflops"]
    del ws
    return {"ms": ms, "T": T, "O": O, "I": I, "n_mat": E, "flops": flops, "TFLOP/s": tf, "peak": peak,
            "bound": "tensor", "frac": tf / peak, "num/den": (out[0].sum() / out[1].sum()).item(),
            "note": f"first unit, activations [{T}, {I}] bf16, {reps} calls over {len(sets)} input sets "
                    "(E pieces + one fused two-product GEMM + reduce per call); flops = 4 T O I per matrix, "
                    "frac of measured dense bf16 burst"}


def time_gptq(tq, step, peak_tinst, reps=3):
    """tq_gptq_sweep (GPTQ/LDLQ column sweep with the search's scales held
    fixed) on the first unit, with the factor U (H^-1 = U^T U) of its first
    matrix's calibration Hessian, damped by 1 % of the mean diagonal (fp64
    Cholesky and inverse by the library, before the timed calls; one factor
    for every matrix of a batch).  Algorithmic work: the propagation's fused
    multiply-adds, I (I - 1) / 2 per row, against the FP32 issue peak."""
    u, r = step.units[0], step.res[0]
    fmt = tq.FORMATS[u.fmt]
    if fmt == tq.NVFP4_G16:
        return {"skipped": "the sweep is built for the integer formats"}
    X = step.sets[0][0][u.site][0]
    W = step.sets[0][1][0]
    E, O, I = W.shape
    H = X.double().T @ X.double()
    H += 0.01 * H.diagonal().mean() * torch.eye(I, device=H.device, dtype=torch.float64)
    U = torch.linalg.cholesky(torch.cholesky_inverse(torch.linalg.cholesky(H)), upper=True).float().contiguous()
    del H
    ws = torch.empty(tq.gptq_workspace_bytes(W), dtype=torch.uint8, device=W.device)
    out = (torch.empty((E, O, I), dtype=torch.int8, device=W.device),
           torch.empty((E, O), dtype=torch.float64, device=W.device))
    Ws = [s[1][0] for s in step.sets]
    tq.tq_gptq_sweep(W, fmt, r.scales, r.zeros, U, out=out, workspace=ws)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for k in range(reps):
        tq.tq_gptq_sweep(Ws[k % len(Ws)], fmt, r.scales, r.zeros, U, out=out, workspace=ws)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    fma = E * O * I * (I - 1) / 2
    achieved = fma / (ms * 1e-3) / 1e12
    del ws, out, U
    return {"ms": ms, "n_mat": E, "O": O, "I": I, "fma": fma, "achieved_tinst": achieved,
            "frac": achieved / peak_tinst, "weights_per_s": E * O * I / (ms * 1e-3),
            "note": f"first unit, {reps} calls over rotating weight copies; fused multiply-adds of the "
                    "propagation (I (I-1)/2 per row) vs the FP32 issue peak; the serial rounding is not counted"}


def time_gemv(tq, step, pk, B, reps=20):
    """tq_dequant_gemv (y = What x straight from the records, B token vectors)
    on the first unit's search output, outside the step, over rotating copies
    of the records larger than L2 (x is per matrix for a batch of matrices,
    shared for one): bytes = records + scales (+ zeros) read + x read + y
    written."""
    u, r = step.units[0], step.res[0]
    fmt = tq.FORMATS[u.fmt]
    E, O, I = u.W.shape
    dev = r.packed.device
    q_bytes = (r.packed.numel() + r.scales.numel() * r.scales.element_size()
               + (0 if r.zeros is None else r.zeros.numel()))
    n = max(1, min(64, math.ceil(2 * L2_BYTES / q_bytes)))
    copies = [(r.packed.clone(), r.scales.clone(), None if r.zeros is None else r.zeros.clone()) for _ in range(n)]
    gen = torch.Generator(device=dev).manual_seed(B)
    x = torch.randn((E, B, I) if E > 1 else (B, I), generator=gen, device=dev).bfloat16()
    y = torch.empty((E, B, O), dtype=torch.float32, device=dev)
    nbytes = q_bytes + x.numel() * 2 + y.numel() * 4
    def run():
        for k in range(reps):
            p, sc, z = copies[k % n]
            tq.tq_dequant_gemv(p, fmt, sc, z, r.global_scale, E, O, I, x, out=y)

    run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()     # decode-time launches are replayed from a graph, not issued one by one
    with torch.cuda.graph(graph):
        run()
    graph.replay()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    graph.replay()
    b.record()
    torch.cuda.synchronize()
    del graph, copies
    ms = a.elapsed_time(b) / reps
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms": ms, "bytes": nbytes, "GB/s": gbs, "frac": gbs / pk["hbm_gbs"],
            "weights_per_s": E * O * I / (ms * 1e-3),
            "note": f"first unit, bf16 x, {reps} launches replayed from a CUDA graph over {n} rotating copies "
                    f"of the records ({n * q_bytes / 2**20:.0f} MiB)"}


def _empty_like_result(tq, r):
    e = lambda t: None if t is None else torch.empty_like(t)  # noqa: E731
    return tq.SearchResult(fmt=r.fmt, scales=e(r.scales), zeros=e(r.zeros), global_scale=e(r.global_scale),
                           cand_idx=e(r.cand_idx), loss=e(r.loss), packed=e(r.packed))


def run_e2e(tq, wl, step, args, world, barrier, dev):
    """Same step from pinned host inputs: every step copies its inputs host ->
    device, runs the path and copies the quantized weights (packed codes +
    scales + zeros/global scales) and the proxy-error sums device -> host,
    all inside the timed region.  Copies and compute are pipelined the way a
    quantization service would run them: three streams (copy-in, compute,
    copy-out) and double-buffered device inputs and outputs, so step i+1's
    inputs travel while step i computes."""
    names = [k for k in wl.sites if k in step.m]
    host_sites = {k: wl.sites[k].X.cpu().pin_memory() for k in names}
    host_W = [u.W.cpu().pin_memory() for u in step.units]
    bufs = []
    for b in range(2):
        dsites = {k: torch.empty_like(wl.sites[k].X) for k in names}
        dW = [torch.empty_like(u.W) for u in step.units]
        st = Step.__new__(Step)
        st.__dict__.update(step.__dict__)
        st.sets = [(dsites, dW)]
        st.search_events = []
        # own outputs, so copy-out of step i never races compute of step i+1
        st.res = [_empty_like_result(tq, r) for r in step.res]
        st.dq = [torch.empty_like(d) for d in step.dq]
        st.px = [(torch.empty_like(a), torch.empty_like(c)) for a, c in step.px]
        st.m = {k: torch.empty_like(v) for k, v in step.m.items()}
        outs = []
        for r, (a, c) in zip(st.res, st.px):
            ts = [r.packed, r.scales] + ([r.zeros] if r.zeros is not None else []) + \
                 ([r.global_scale] if r.global_scale is not None else []) + [a, c]
            outs.append([(t, torch.empty(t.shape, dtype=t.dtype, pin_memory=True)) for t in ts])
        bufs.append((st, dsites, dW, outs))
    h2d = sum(t.numel() * t.element_size() for t in list(host_sites.values()) + host_W)
    d2h = sum(h.numel() * h.element_size() for o in bufs[0][3] for _, h in o)
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()

    def run(nsteps):
        comp_done, out_done = [], []
        first = torch.cuda.Event(enable_timing=True)
        last = torch.cuda.Event(enable_timing=True)
        first.record(s_in)
        for i in range(nsteps):
            st, dsites, dW, outs = bufs[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])
                for k in names:
                    dsites[k].copy_(host_sites[k], non_blocking=True)
                for d, h in zip(dW, host_W):
                    d.copy_(h, non_blocking=True)
                copied = torch.cuda.Event()
                copied.record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(copied)
                if i >= 2:
                    s_comp.wait_event(out_done[i - 2])
                st(0)
                ev = torch.cuda.Event()
                ev.record(s_comp)
                comp_done.append(ev)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev)
                for o in outs:
                    for d, h in o:
                        h.copy_(d, non_blocking=True)
                ev2 = torch.cuda.Event()
                ev2.record(s_out)
                out_done.append(ev2)
        s_in.wait_event(out_done[-1])
        last.record(s_in)
        return first, last

    run(max(3, args.warmup // 2))
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    steps = max(4, args.steps // 2)
    a, b = run(steps)
    torch.cuda.synchronize()
    barrier()
    from group_scale_search_b200.dist import max_over_ranks
    ms = max_over_ranks(a.elapsed_time(b), dev)
    nw = sum(u.W.numel() for u in step.units)
    return {"value": world * nw / (ms / steps * 1e-3), "unit": "weights/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms / steps,
            "pipeline": "3 streams (copy-in, compute, copy-out), double-buffered inputs and outputs"}


if __name__ == "__main__":
    sys.exit(main())
