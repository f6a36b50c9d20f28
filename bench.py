#!/usr/bin/env python
"""Throughput benchmark: weights quantized per second through the whole hot
path on B200 -- imatrix -> group-scale search with fused RTN + pack ->
dequant -> imatrix-weighted proxy error -- one JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config c2] [--impl tq|reference]
                  [--workloads all|none|c0,c1,...] [--scaling strong|weak]

A step is one pass of every row of the path over one batch of synthetic input.
The headline workload (--config, default c2: the int3-g64 MoE stack of 64
experts of 2048 x 7168, the largest workload that is one job on one GPU)
carries the line's `value`, `roofline`, `e2e` and `cpu_baseline`; every other
workload gets a row of the same figures under `per_workload`.  `value` is
device-timed with inputs resident in HBM (CUDA events, barrier + synchronize
on both sides, max over ranks); `e2e` repeats the step through the public API
from pinned host buffers, with the host->device copies of the inputs and the
device->host read of the results inside the timed region.  `roofline` reports
the dominant kernel (the search) against the FP32 CUDA-core issue peak;
`hbm_rows` the streaming kernels against the HBM peak.

--gpus N > 1 without a launcher re-executes this script under
torch.distributed.run with N ranks (one per GPU, NCCL).  With --scaling strong
(the default) the ranks split one workload the way the method partitions: the
experts of a MoE stack (no exchange), or the rows of every dense matrix with
the calibration tokens split too (an all-reduce of the per-column sums of x^2
and of the per-matrix (num, den) pairs).  --scaling weak gives every rank its
own independent copy of the workload.  --impl reference times the CPU oracle
on bounded samples of the same workload instead (rank 0 alone).
"""
from __future__ import annotations

import argparse
import ctypes
import dataclasses
import datetime
import json
import math
import os
import socket
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
WORKLOAD_ORDER = ["c0", "c1", "c2", "c3", "c4"]
# FP32 lane-instructions per weight of the search (the dominant kernel):
# candidate-element evaluations per weight x instructions per evaluation
# (sym int3: 96 x 7; asym int4: 1024 x 5; NVFP4: 16 x 10).  An algorithmic
# model of the work, not a count of what the kernels issue.
SEARCH_INSTR_PER_W = {"int3_g64_sym": 96 * 7, "int4_g128_asym": 1024 * 5, "nvfp4_g16": 16 * 10}
SEARCH_CEE_PER_W = {"int3_g64_sym": 96, "int4_g128_asym": 1024, "nvfp4_g16": 16}
# our kernels per call: imatrix 2 (partial + final), search 1 (NVFP4: amax +
# global + search = 3), dequant 1, proxy 1
KERNELS = {"imatrix": 1, "search": {"int3_g64_sym": 1, "int4_g128_asym": 1, "nvfp4_g16": 3},
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


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


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
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
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


# ------------------------------------------------------------------ sharding over ranks

@dataclasses.dataclass
class Shard:
    """This rank's part of a workload split over `world` ranks.

    pieces[k] = (axis, start, end, extent) for timed unit k of the whole
    workload: "experts" (a range of the matrices of a MoE stack) or "rows" (a
    range of the rows of a dense matrix).  site_tokens maps a calibration
    site whose tokens are split to its total token count (its imatrix is the
    all-reduced sum of x^2 over every rank's tokens divided by that count)."""
    world: int
    rank: int
    pieces: list
    site_tokens: dict
    row_units: list      # indices (into this rank's units) of row-split matrices: their (num, den) are all-reduced


def shard_plan(layout, world: int, rank: int):
    """The partition of the method's independent units over ranks: experts of
    a MoE stack split in contiguous ranges (no exchange); a dense matrix
    split by rows, its calibration site by tokens (sizes differ by at most
    one).  Returns [(axis, start, end, extent)] per timed unit and the token
    ranges {site: (t0, t1, T)}."""
    from group_scale_search_b200.dist import shard_range
    pieces, tokens = [], {}
    for name, fmt, (E, O, I), site, timed in layout["units"]:
        if not timed:
            continue
        if E > 1:
            e0, e1 = shard_range(E, rank, world)
            pieces.append(("experts", e0, e1, E))
        else:
            o0, o1 = shard_range(O, rank, world)
            pieces.append(("rows", o0, o1, O))
            if site not in tokens:
                T = layout["sites"][site][1]
                tokens[site] = shard_range(T, rank, world) + (T,)
    return pieces, tokens


def shard_workload(wl, world: int, rank: int):
    """This rank's own copy of its part of `wl` (units and sites cloned, so
    the whole workload can be freed) and its Shard description."""
    units_all = [u for u in wl.units if u.timed]
    lay = {"units": [(u.name, u.fmt, tuple(u.W.shape), u.site, True) for u in units_all],
           "sites": {k: tuple(s.X.shape) + (str(s.X.dtype),) for k, s in wl.sites.items()}}
    pieces, tokens = shard_plan(lay, world, rank)
    units, sites, row_units = [], {}, []
    for u, (axis, a, b, n) in zip(units_all, pieces):
        if b <= a:
            continue
        X = wl.sites[u.site].X
        if axis == "experts":
            W = u.W[a:b].clone()
            sites[u.site] = synth.Site(u.site, X[a:b].clone())
        else:
            W = u.W[:, a:b].clone()
            if u.site not in sites:
                t0, t1, T = tokens[u.site]
                sites[u.site] = synth.Site(u.site, X[:, t0:t1].clone())
            row_units.append(len(units))
        units.append(synth.Unit(u.name, u.fmt, W, u.site))
    site_tokens = {k: v[2] for k, v in tokens.items() if k in sites}
    return synth.Workload(wl.name, units, sites), Shard(world, rank, pieces, site_tokens, row_units)


# ------------------------------------------------------------------ the step

class Step:
    """One pass of the whole path over one input set, on the current stream."""

    def __init__(self, tq, wl, sets, shard=None):
        self.tq = tq
        self.wl = wl
        self.sets = sets            # list of (sites dict name->X, units list of W)
        self.shard = shard
        self.fmts = [tq.FORMATS[u.fmt] for u in wl.units if u.timed]
        self.units = [u for u in wl.units if u.timed]
        dev = self.units[0].W.device
        # preallocated outputs and workspaces (the timed region allocates
        # nothing); the search writes what the metric needs -- scales,
        # zeros, global scales and the packed records -- and no per-group
        # candidate index or loss
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
            self.res.append(tq.search_result_empty(u.W, fmt, want_idx=False, want_loss=False))
            self.dq.append(torch.empty((E, O, I), dtype=torch.bfloat16, device=dev))
            self.px.append((torch.empty(E, dtype=torch.float64, device=dev),
                            torch.empty(E, dtype=torch.float64, device=dev)))
            self.ws_px.append(torch.empty(max(16, tq.proxy_workspace_bytes(u.W, fmt)), dtype=torch.uint8,
                                          device=dev))
        # several units of one format (a dense model's projections): their
        # dequant and proxy run as one grouped launch each
        self.grouped = len(self.units) > 1 and len(set(self.fmts)) == 1 and hasattr(tq, "tq_dequant_batch")
        if self.grouped:
            self.ws_px_batch = torch.empty(max(16, tq.proxy_batch_workspace_bytes([u.W for u in self.units],
                                                                                  self.fmts[0])),
                                           dtype=torch.uint8, device=dev)
        self.search_events = []
        self.row_events = []

    def _m_for(self, u):
        m = self.m[u.site]
        return m if u.W.shape[0] > 1 else m[0]

    def kernels_per_step(self):
        n = KERNELS["imatrix"] * len(self.m)
        for u in self.units:
            n += KERNELS["search"][u.fmt]
            if not self.grouped:
                n += KERNELS["dequant"] + KERNELS["proxy"]
        if self.grouped:
            n += KERNELS["dequant"] + KERNELS["proxy"]
        return n

    def __call__(self, k: int, time_search: bool = False):
        tq = self.tq
        sites, Ws = self.sets[k % len(self.sets)]
        split_tokens = self.shard.site_tokens if self.shard is not None else {}

        def mark():
            if not time_search:
                return None
            ev = torch.cuda.Event(enable_timing=True)
            ev.record()
            return ev

        for name in self.m:
            X = sites[name]
            a = mark()
            if name in split_tokens:      # this rank's tokens: sums of x^2, then the sum over ranks / T
                from group_scale_search_b200.dist import allreduce_imatrix
                tq.tq_imatrix(X, m=self.m[name], alpha=1.0, workspace=self.ws_im[name])
                b = mark()
                self.m[name].copy_(allreduce_imatrix(self.m[name], split_tokens[name]))
            else:
                tq.tq_imatrix(X, m=self.m[name], alpha=1.0 / X.shape[1], workspace=self.ws_im[name])
                b = mark()
            if time_search:
                self.row_events.append(("imatrix", X.numel() * X.element_size(), a, b))
        if self.grouped:
            self._grouped(Ws, mark, time_search)
            return
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
                self.row_events.append(("dequant", self._dq_bytes(i), b, c))
            tq.tq_proxy_error(W, r.packed, fmt, r.scales, r.zeros, r.global_scale, m, out=self.px[i],
                              workspace=self.ws_px[i])
            if time_search:
                self.row_events.append(("proxy", self._px_bytes(W, i), c, mark()))
            self._exchange_proxy(i)

    def _dq_bytes(self, i):
        r = self.res[i]
        return (r.packed.numel() + self.dq[i].numel() * 2 + r.scales.numel() * r.scales.element_size()
                + (0 if r.zeros is None else r.zeros.numel()))

    def _px_bytes(self, W, i):
        r = self.res[i]
        return (W.numel() * W.element_size() + r.packed.numel() + r.scales.numel() * r.scales.element_size()
                + (0 if r.zeros is None else r.zeros.numel()))

    def _exchange_proxy(self, i):
        if self.shard is not None and i in self.shard.row_units:   # whole-matrix (num, den)
            from group_scale_search_b200.dist import allreduce_proxy
            num, den = allreduce_proxy(*self.px[i])
            self.px[i][0].copy_(num)
            self.px[i][1].copy_(den)

    def _grouped(self, Ws, mark, time_search):
        """Every unit's search, then one grouped dequant and one grouped proxy
        launch over all units."""
        tq = self.tq
        fmt = self.fmts[0]
        for i, u in enumerate(self.units):
            a = mark()
            tq.tq_search_groups(Ws[i], self._m_for(u), fmt, out=self.res[i])
            if time_search:
                self.search_events.append((u.fmt, Ws[i].numel(), a, mark()))
        res = self.res
        zeros = [r.zeros for r in res] if res[0].zeros is not None else None
        gsc = [r.global_scale for r in res] if res[0].global_scale is not None else None
        scales = [r.scales for r in res]
        packed = [r.packed for r in res]
        b = mark()
        tq.tq_dequant_batch(packed, fmt, scales, zeros, gsc, [tuple(W.shape) for W in Ws], out=self.dq)
        c = mark()
        tq.tq_proxy_error_batch(Ws, packed, fmt, scales, zeros, gsc, [self._m_for(u) for u in self.units],
                                out=self.px, workspace=self.ws_px_batch)
        d = mark()
        if time_search:
            self.row_events.append(("dequant", sum(self._dq_bytes(i) for i in range(len(Ws))), b, c))
            self.row_events.append(("proxy", sum(self._px_bytes(W, i) for i, W in enumerate(Ws)), c, d))
        for i in range(len(Ws)):
            self._exchange_proxy(i)

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


# ------------------------------------------------------------------ configuration (shared by both arms)

_GROUP = {"int3_g64_sym": 64, "int4_g128_asym": 128, "nvfp4_g16": 16}


def workload_weights(name: str, scale: float = 1.0) -> int:
    lay = synth.layout(name, scale)
    return sum(E * O * I for _, _, (E, O, I), _, timed in lay["units"] if timed)


def config_dict(name: str, scale: float, world: int, scaling: str) -> dict:
    """The workload and how the job runs it, from shapes alone (both arms
    print the same dictionary)."""
    lay = synth.layout(name, scale)
    units = [u for u in lay["units"] if u[4]]
    nw = sum(E * O * I for _, _, (E, O, I), _, _ in units)
    groups = sum(E * O * (-(-I // _GROUP[fmt])) for _, fmt, (E, O, I), _, _ in units)
    nbytes = sum(E * O * I * (4 if name == "c0" else 2) for _, _, (E, O, I), _, _ in units)
    nbytes += sum(E * T * I * (4 if dt == "f32" else 2) for s, (E, T, I, dt) in lay["sites"].items()
                  if any(u[3] == s for u in units))
    per_rank = nbytes / world if scaling == "strong" else nbytes
    n_sets = max(1, min(64, math.ceil(2 * L2_BYTES / per_rank)))
    job = nw * (world if scaling == "weak" else 1)
    if world == 1:
        par = "one GPU"
    elif scaling == "strong":
        par = (f"strong x{world}: " + ("experts split over ranks, no exchange" if units[0][2][0] > 1 else
                                       "rows of every matrix and calibration tokens split over ranks; "
                                       "all-reduce of sum x^2 per column and of (num, den) per matrix"))
    else:
        par = f"weak x{world}: an independent copy of the workload per GPU"
    return {"workload": f"{name}: {synth.DESCRIPTIONS[name]}" + ("" if scale == 1.0 else f" (scaled x{scale})"),
            "weights": job, "groups": groups * (world if scaling == "weak" else 1),
            "step": "imatrix + search with fused RTN/pack + dequant(bf16) + proxy error",
            "l2": (f"{n_sets} rotating input sets per GPU, {n_sets * per_rank / 2**20:.0f} MiB > 126 MiB L2"
                   if n_sets * per_rank > L2_BYTES else
                   f"{n_sets} input sets per GPU ({n_sets * per_rank / 2**20:.1f} MiB) fit in L2"),
            "parallelism": par}


# ------------------------------------------------------------------ CPU oracle baseline

def oracle_rows(wl, budget_s: float):
    """(rows per unit, passes) for an oracle sample of about `budget_s`
    seconds: the first rows of every unit's first matrix, repeated in whole
    passes when that matrix is too small to fill the budget."""
    import oracle
    oracle.build()
    units = [u for u in wl.units if u.timed]
    probe_rows = 8
    t0 = time.perf_counter()
    _oracle_unit(oracle, wl, units[0], probe_rows)
    per_row = max((time.perf_counter() - t0) / probe_rows, 1e-6)
    rows = max(8, min(units[0].W.shape[1], int(budget_s / per_row / len(units))))
    passes = max(1, int(round(budget_s / (per_row * rows * len(units)))))
    return rows, passes


def oracle_sample(wl, rows: int, passes: int = 1):
    """Times the oracle (as it stands) on a bounded sample of the workload:
    for each unit, the imatrix of its site (first matrix) and search + pack +
    dequant + proxy error over the first `rows` rows of its first matrix,
    `passes` times.  Returns (weights/s, cores, description, seconds, weights)."""
    import oracle
    oracle.build()
    units = [u for u in wl.units if u.timed]
    t0 = time.perf_counter()
    n = 0
    for _ in range(passes):
        for u in units:
            r = min(rows, u.W.shape[1])
            _oracle_unit(oracle, wl, u, r)
            n += r * u.W.shape[2]
    dt = time.perf_counter() - t0
    desc = (f"oracle (C, fp64, OpenMP) on {rows} rows of the first matrix of each of {len(units)} unit(s), "
            f"{passes} pass(es) = {n} weights: imatrix of the site's first matrix over all its tokens, "
            f"search+pack, dequant, proxy; host CPU {cpu_model()}")
    return n / dt, oracle.num_threads(), desc, dt, n


def oracle_one_thread(config: str, frac: float = 0.01):
    """The same oracle on one host thread (OMP_NUM_THREADS=1 in a child
    process, so the parent's thread pool is untouched) over a fixed `frac` of
    the first unit's rows: the scaling reference for the multi-core figure.
    Returns (weights/s, description) or None if the child fails."""
    code = (f"import json, time, synth, bench, oracle; oracle.build(); wl = synth.make({config!r}, 'cpu', max_mats=1); "
            f"u = [x for x in wl.units if x.timed][0]; rows = max(8, int(u.W.shape[1] * {frac!r})); "
            f"t0 = time.perf_counter(); bench._oracle_unit(oracle, wl, u, rows); dt = time.perf_counter() - t0; "
            f"print(json.dumps([rows * u.W.shape[2] / dt, rows, u.W.shape[2], oracle.num_threads(), dt]))")
    env = dict(os.environ, OMP_NUM_THREADS="1")
    try:
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300, env=env,
                           cwd=ROOT)
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


def read_profile(path, workload, kernel):
    """The ncu figures of `kernel` on `workload` from the profiles table:
    launches per step, DRAM bytes (read + write) and duration summed over
    them, and the FP32-pipe share of its peak; None where the table has no
    entry."""
    out = {"launches": None, "traffic": None, "ms": None, "fp32_pipe_frac": None, "source": None}
    try:
        for line in open(path):
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) >= 7 and cells[0] == workload and cells[1] == kernel and cells[2].isdigit():
                out["launches"] = int(cells[2])
                out["traffic"] = int(cells[3]) if cells[3].isdigit() else None
                for key, cell in (("ms", cells[4]), ("fp32_pipe_frac", cells[5])):
                    try:
                        out[key] = float(cell)
                    except ValueError:
                        pass
                out["source"] = cells[6]
    except OSError:
        pass
    return out


# ------------------------------------------------------------------ arguments and launch

def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="c2", choices=WORKLOAD_ORDER,
                    help="the headline workload (default c2, the largest one-GPU workload)")
    ap.add_argument("--workloads", default="all",
                    help="workloads timed beside the headline, each as a per_workload row: "
                         "'all', 'none' or a comma list")
    ap.add_argument("--scaling", default="strong", choices=["strong", "weak"],
                    help="N > 1: split one workload over the ranks (strong) or give each its own (weak)")
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--scale", type=float, default=1.0,
                    help="shrink the workload (profiling and tests only; the reported line is for scale 1)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true", help="skip the rows beyond the step")
    ap.add_argument("--plan-only", action="store_true",
                    help="print how the ranks split the workload (CPU and gloo without a GPU) and exit")
    ap.add_argument("--profile-table", default=os.path.join(ROOT, "profiles", "traffic.md"),
                    help="ncu DRAM bytes per launch and FP32-pipe share by workload and kernel")
    ap.add_argument("--jsonl", default=None,
                    help="also append the result line, with a UTC time stamp and the git revision, to this file")
    return ap.parse_args(argv)


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def spawn_ranks(args) -> int:
    """--gpus N with no launcher: run this script under torch.distributed.run
    with N local ranks (rank 0 prints the line) and return its exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", f"--master-port={_free_port()}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd, cwd=ROOT)


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


# ------------------------------------------------------------------ the reference arm (the oracle)

def reference_arm(args, world, rank):
    """The oracle as it stands on the host cores: every step is the same
    bounded sample of the headline workload (the first rows of the first
    matrix of every unit, sized once to about 2 s), timed on its own."""
    if rank != 0:
        return 0
    wl = synth.make(args.config, "cpu", seed=0, scale=args.scale, max_mats=1)
    rows, passes = oracle_rows(wl, budget_s=2.0)
    for _ in range(args.warmup):
        oracle_sample(wl, max(8, rows // 4))
    vals, secs = [], []
    desc = cores = n = None
    for _ in range(args.steps):
        v, cores, desc, dt, n = oracle_sample(wl, rows, passes)
        vals.append(v)
        secs.append(dt)
    dt = statistics.median(secs)
    v = n / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "weights/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": args.scaling if args.gpus > 1 else "weak", "vs_baseline": None,
            "dtype": "f64",
            "data": "synthetic", "config": config_dict(args.config, args.scale, args.gpus, args.scaling),
            "step_definition": f"one bounded sample of the workload per step ({n} weights), host cores only",
            "cpu_baseline": {"value": v, "unit": "weights/s", "cores": cores, "kind": "oracle",
                             "sample": desc, "cpu": cpu_model(), "seconds_per_step": dt},
            "e2e": {"value": v, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if args.jsonl:
        append_jsonl(args.jsonl, line)
    return 0


# ------------------------------------------------------------------ the tq arm

def plan_only(args, world, rank):
    """How the ranks split each workload: every rank builds the (scaled)
    workload's shapes, takes its part, and rank 0 gathers and checks that
    every expert / row / token is covered exactly once."""
    import torch.distributed as dist
    names = [args.config] + [w for w in _other_workloads(args) if w != args.config]
    out = {}
    for name in names:
        lay = synth.layout(name, args.scale)
        pieces, tokens = shard_plan(lay, world, rank)
        mine = {"rank": rank, "pieces": pieces, "tokens": {k: list(v) for k, v in tokens.items()}}
        got = [None] * world
        if world > 1:
            dist.all_gather_object(got, mine)
        else:
            got = [mine]
        units = [u for u in lay["units"] if u[4]]
        ok = True
        for k, u in enumerate(units):
            axis = got[0]["pieces"][k][0]
            extent = got[0]["pieces"][k][3]
            cover = np.zeros(extent, np.int64)
            for g in got:
                _, a, b, _ = g["pieces"][k]
                cover[a:b] += 1
            ok &= bool((cover == 1).all())
        for site in got[0]["tokens"]:
            T = got[0]["tokens"][site][2]
            cover = np.zeros(T, np.int64)
            for g in got:
                a, b, _ = g["tokens"][site]
                cover[a:b] += 1
            ok &= bool((cover == 1).all())
        out[name] = {"ranks": got, "covered_once": ok}
    if rank == 0:
        print(json.dumps({"plan": out, "world": world}), flush=True)
    return 0


def _other_workloads(args):
    if args.workloads == "none":
        return []
    if args.workloads == "all":
        return [w for w in WORKLOAD_ORDER if w != args.config]
    return [w.strip() for w in args.workloads.split(",") if w.strip() and w.strip() != args.config]


def main(argv=None):
    args = parse(argv)
    assert args.warmup >= 3 or args.impl == "reference", "at least 3 warm-up steps"
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        return spawn_ranks(args)
    if env_world is not None and int(env_world) != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {env_world} ranks")
    if args.impl == "reference":   # rank 0 alone times the oracle; no process group
        return reference_arm(args, int(env_world or "1"), int(os.environ.get("RANK", "0")))

    from group_scale_search_b200.dist import init_from_env
    backend = "nccl" if torch.cuda.is_available() and not args.plan_only else "gloo"
    world, rank, local = init_from_env(backend, timeout_s=120.0)
    if args.plan_only:
        rc = plan_only(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        return rc

    import group_scale_search_b200 as tq
    if world == 1:
        torch.cuda.set_device(0)
    tq.lib()
    dev = torch.device("cuda", torch.cuda.current_device())

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    pk = peaks()
    headline, wl_head = run_workload(tq, args.config, args, world, rank, dev, barrier, pk, keep_wl=True)
    per = {}
    for name in _other_workloads(args):
        row, _ = run_workload(tq, name, args, world, rank, dev, barrier, pk)
        per[name] = row

    line = {"metric": METRIC, "value": headline["value"], "unit": "weights/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": headline["ms_per_step"],
            "higher_is_better": True, "scaling": args.scaling if world > 1 else "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_dict(args.config, args.scale, world, args.scaling),
            "groups_per_s": headline["groups_per_s"],
            "roofline": headline["roofline"], "hbm_rows": headline["hbm_rows"],
            "next_rows": headline.get("next_rows"), "clocks": headline["clocks"], "e2e": headline.get("e2e"),
            "gpu_launches": headline["gpu_launches"],
            "per_workload": per}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows, passes = oracle_rows(wl_head, budget_s=12.0)
        v, cores, desc, dt, _ = oracle_sample(wl_head, rows, passes)
        line["cpu_baseline"] = {"value": v, "unit": "weights/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": dt, "cpu": cpu_model()}
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


def run_workload(tq, name, args, world, rank, dev, barrier, pk, keep_wl=False):
    """Times `steps` steps of workload `name` (this rank's part of it) and
    the rows around the step; returns the row's figures (and the workload
    when `keep_wl`, for the CPU baseline)."""
    from group_scale_search_b200.dist import max_over_ranks
    strong = world > 1 and args.scaling == "strong"
    wl = synth.make(name, dev, seed=0 if strong else rank, scale=args.scale)
    shard = None
    if strong:
        wl, shard = shard_workload(wl, world, rank)
        torch.cuda.empty_cache()
    nbytes = input_bytes(wl)
    n_sets = max(1, min(64, math.ceil(2 * L2_BYTES / nbytes)))
    sets = make_sets(wl, n_sets)
    step = Step(tq, wl, sets, shard)
    nw_rank = sum(u.W.numel() for u in step.units)
    nw_job = workload_weights(name, args.scale) * (1 if strong else world)
    stream = torch.cuda.current_stream()

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
    value = nw_job / (ms_step * 1e-3)

    # dominant kernel: the search (CUDA events on the launching stream)
    by_fmt = {}
    for fmt, n, a, b in step.search_events:
        d = by_fmt.setdefault(fmt, [0.0, 0])
        d[0] += a.elapsed_time(b)
        d[1] += n
    fmt_main = max(by_fmt, key=lambda f: by_fmt[f][0])
    search_ms = by_fmt[fmt_main][0] / args.steps
    w_per_launch = by_fmt[fmt_main][1] / args.steps / max(1, sum(1 for u in step.units if u.fmt == fmt_main))
    n_launch = sum(1 for u in step.units if u.fmt == fmt_main)
    props = torch.cuda.get_device_properties(dev)
    sms = props.multi_processor_count
    peak_tinst = sms * 128 * pk["sm_max_mhz"] * 1e6 / 1e12
    achieved = SEARCH_INSTR_PER_W[fmt_main] * by_fmt[fmt_main][1] / args.steps / (search_ms * 1e-3) / 1e12
    clocks = clk.summary()
    prof = read_profile(args.profile_table, name, f"search {fmt_main}")
    per_launch_traffic = (prof["traffic"] // prof["launches"]) if prof["traffic"] and prof["launches"] else None
    roofline = {"bound": "alu", "achieved": achieved, "peak": peak_tinst, "unit": "Tinst/s",
                "frac": achieved / peak_tinst, "traffic": per_launch_traffic if args.scale == 1.0 else None,
                "kernel": f"search {fmt_main}", "kernel_ms": search_ms / n_launch, "launches_per_step": n_launch,
                "weights_per_launch": w_per_launch,
                "per_unit": f"{SEARCH_INSTR_PER_W[fmt_main]} FP32 lane-instr/weight "
                            f"({SEARCH_CEE_PER_W[fmt_main]} candidate-element evaluations): an algorithmic "
                            f"model of the work",
                "peak_basis": f"{sms} SMs x 128 FP32 lanes x {pk['sm_max_mhz']:.0f} MHz ({pk['source']} max clock)",
                "frac_at_observed_clock": (achieved / (sms * 128 * clocks["sm_mhz"] * 1e6 / 1e12))
                if clocks.get("sm_mhz") else None,
                "cee_per_s": SEARCH_CEE_PER_W[fmt_main] * by_fmt[fmt_main][1] / args.steps / (search_ms * 1e-3),
                "ncu_fp32_pipe_frac": prof["fp32_pipe_frac"], "ncu_source": prof["source"]}

    # every HBM-bound row of the step: algorithmic bytes / CUDA-event time vs the HBM peak
    rows = {}
    for rname, nbytes_row, a, b in step.row_events:
        d = rows.setdefault(rname, [0.0, 0, 0])
        d[0] += a.elapsed_time(b)
        d[1] += nbytes_row
        d[2] += 1
    hbm_rows = {}
    kname = {"imatrix": "k_imatrix_partial", "dequant": "k_dequant", "proxy": "k_proxy"}
    if step.grouped:   # one grouped launch per row for all units
        kname.update(dequant="k_dequant_batch", proxy="k_proxy_batch")
    elif fmt_main == "int3_g64_sym":   # the int3 proxy runs the grouped kernel for one unit too
        kname.update(proxy="k_proxy_batch")
    for rname, (t_ms, nb, cnt) in rows.items():
        gbs = nb / (t_ms * 1e-3) / 1e9
        p = read_profile(args.profile_table, name, kname[rname])
        ok = args.scale == 1.0 and p["traffic"] is not None
        hbm_rows[rname] = {"ms": t_ms / args.steps, "bytes": nb // args.steps, "launches_per_step": cnt // args.steps,
                           "GB/s": gbs, "frac": gbs / pk["hbm_gbs"],
                           "ncu_traffic": p["traffic"] if ok else None, "ncu_ms": p["ms"] if ok else None,
                           "ncu_frac": (nb / args.steps / (p["ms"] * 1e-3) / 1e9 / pk["hbm_gbs"])
                           if ok and p["ms"] else None}
    hbm_rows["pack"] = time_pack(tq, step, pk)
    row = {"value": value, "ms_per_step": ms_step, "weights": nw_job, "weights_this_rank": nw_rank,
           "groups_per_s": value / _GROUP[fmt_main], "roofline": roofline, "hbm_rows": hbm_rows,
           "clocks": clocks, "gpu_launches": step.kernels_per_step() * args.steps,
           "config": config_dict(name, args.scale, world, args.scaling)}
    if not args.no_next_rows:
        row["next_rows"] = next_rows(tq, step, pk, peak_tinst)
    if not args.no_e2e:
        row["e2e"] = run_e2e(tq, wl, step, args, nw_job, barrier, dev)
    del step, sets
    if not keep_wl:
        del wl
        wl = None
    torch.cuda.empty_cache()
    return row, wl


def next_rows(tq, step, pk, peak_tinst):
    """The rows beyond the step, each on the first unit of the workload,
    outside the step's timed region."""
    out = {"dequant_gemv": {f"B={B}": time_gemv(tq, step, pk, B) for B in (1, 8)}}
    if step.units[0].fmt == "int4_g128_asym":
        out["asym_ladder_256_64"] = time_ladder(tq, step, peak_tinst)
        out["int4_g64"] = time_int4_group(tq, step, pk, peak_tinst, tq.INT4_G64_ASYM)
        out["int4_g32"] = time_int4_group(tq, step, pk, peak_tinst, tq.INT4_G32_ASYM)
    out["hessian"] = time_hessian(tq, step, pk)
    out["proxy_full_hessian"] = time_proxy_full(tq, step, pk)
    out["gptq_sweep"] = time_gptq(tq, step, peak_tinst)
    out["fp8_tensor"] = time_fp8(tq, step, pk, peak_tinst)
    out["lloyd_max_2bit"] = time_lloyd(tq, step, pk)
    if step.units[0].fmt == "nvfp4_g16":
        out["nvfp4_w4a4_gemm"] = time_w4a4(tq, step, pk)
    return out


def time_w4a4(tq, step, pk, reps=5):
    """NVFP4 W4A4 product on the first unit: every expert's calibration tokens
    quantized to NVFP4 (tq_quant_nvfp4_act), their scales re-laid out as the
    tensor core's scale tiles, and the block-scaled tcgen05 GEMM against the
    expert's searched records (the weights' scale tiles made once, outside
    the timed calls).  Roofline of the GEMM: the slower of its flops against
    the dense FP4 peak (the measured bf16 figure x 4, the nominal FP4:bf16
    ratio) and its bytes (records, scales, fp32 outputs) against HBM."""
    u, r = step.units[0], step.res[0]
    sets = [(s[0][u.site], s[1][0]) for s in step.sets]
    X0 = sets[0][0]
    E, O, I = u.W.shape
    T = X0.shape[1]
    if I % 32:
        return {"skipped": "I must be a multiple of 32"}
    G = I // 16
    ws = tq.tq_nvfp4_scales_to_mma(r.scales.reshape(E, O, G).contiguous(), E, O, I)
    act = tq.tq_quant_nvfp4_act(X0)
    xs = tq.tq_nvfp4_scales_to_mma(act.scales, E, T, I)
    y = torch.empty((E, T, O), dtype=torch.float32, device=X0.device)
    tq.tq_gemm_nvfp4(act.packed, xs, act.global_scale, r.packed, ws, r.global_scale, E, T, O, I, out=y)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps + 1)]
    ev[0].record()
    for k in range(reps):
        X = sets[k % len(sets)][0]
        tq.tq_quant_nvfp4_act(X, out=act)
        tq.tq_nvfp4_scales_to_mma(act.scales, E, T, I, out=xs)
        ev[2 * k + 1].record()
        tq.tq_gemm_nvfp4(act.packed, xs, act.global_scale, r.packed, ws, r.global_scale, E, T, O, I, out=y)
        ev[2 * k + 2].record()
    torch.cuda.synchronize()
    call_ms = ev[0].elapsed_time(ev[-1]) / reps
    gemm_ms = sum(ev[2 * k + 1].elapsed_time(ev[2 * k + 2]) for k in range(reps)) / reps
    flops = 2 * E * T * O * I
    nbytes = (E * O * G * 8 + E * O * G + E * T * G * 8 + E * T * G + E * T * O * 4)
    fp4_peak = pk["bf16_tflops"] * 4
    t_min = max(flops / (fp4_peak * 1e12), nbytes / (pk["hbm_gbs"] * 1e9))
    return {"gemm_ms": gemm_ms, "call_ms": call_ms, "E": E, "T": T, "O": O, "I": I, "flops": flops,
            "TFLOP/s": flops / (gemm_ms * 1e-3) / 1e12, "fp4_peak_tflops": fp4_peak,
            "frac_tensor": flops / (gemm_ms * 1e-3) / 1e12 / fp4_peak, "bytes": nbytes,
            "GB/s": nbytes / (gemm_ms * 1e-3) / 1e9,
            "bound": "tensor" if flops / (fp4_peak * 1e12) >= nbytes / (pk["hbm_gbs"] * 1e9) else "hbm",
            "frac": t_min / (gemm_ms * 1e-3),
            "note": f"first unit: {E} experts x {T} tokens x {O} x {I}; {reps} calls (activation quantizer + "
                    "scale tiles + GEMM), GEMM timed alone with CUDA events; fp4 peak = measured bf16 x 4 "
                    "(nominal ratio); y fp32"}


def time_pack(tq, step, pk, reps=12):
    """tq_pack (RTN + pack with given scales, the stand-alone form of the fused
    pack) outside the step, rotating through the input sets: on the first
    unit, or on all units in one grouped launch (tq_pack_batch) where the step
    groups them; bytes = weights read + packed records written + scales
    (+ zeros) read."""
    n = len(step.units) if step.grouped else 1
    res = step.res[:n]
    fmt = tq.FORMATS[step.units[0].fmt]
    outs = [torch.empty_like(r.packed) for r in res]
    Wsets = [s[1][:n] for s in step.sets]
    nbytes = sum(W.numel() * W.element_size() + o.numel() + r.scales.numel() * r.scales.element_size()
                 + (0 if r.zeros is None else r.zeros.numel()) for W, o, r in zip(Wsets[0], outs, res))
    scales = [r.scales for r in res]
    zeros = [r.zeros for r in res] if res[0].zeros is not None else None
    gsc = [r.global_scale for r in res] if res[0].global_scale is not None else None

    def call(k):
        Ws = Wsets[k % len(Wsets)]
        if step.grouped:
            tq.tq_pack_batch(Ws, fmt, scales, zeros, gsc, out=outs)
        else:
            r = res[0]
            tq.tq_pack(Ws[0], fmt, r.scales, r.zeros, r.global_scale, out=outs[0])

    for k in range(3):
        call(k)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for k in range(reps):
        call(k)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    gbs = nbytes / (ms * 1e-3) / 1e9
    what = f"all {n} units in one grouped launch" if step.grouped else "first unit"
    return {"ms": ms, "bytes": nbytes, "GB/s": gbs, "frac": gbs / pk["hbm_gbs"],
            "note": f"{what}, back-to-back launches over {len(Wsets)} rotating weight copies"}


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


def time_int4_group(tq, step, pk, peak_tinst, fmt, reps=5):
    """An int4 format with smaller groups (int4-g64, int4-g32) on the first
    unit: the joint search with fused RTN and pack (1024 candidate-element
    evaluations per weight, as for g128) against the FP32 issue roofline, and
    the bf16 dequantization against HBM (records 0.5 B + scale and zero 5/g B
    read, 2 B written per weight)."""
    u = step.units[0]
    m = step._m_for(u)
    Ws = [s[1][0] for s in step.sets]
    E, O, I = u.W.shape
    res = tq.tq_search_groups(Ws[0], m, fmt, want_idx=False, want_loss=False)
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
    if Xs[0].dtype != torch.bfloat16:
        return {"skipped": "the tensor-core path takes bf16 activations"}
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


def run_e2e(tq, wl, step, args, nw_job, barrier, dev):
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
    return {"value": nw_job / (ms / steps * 1e-3), "unit": "weights/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms / steps,
            "pipeline": "3 streams (copy-in, compute, copy-out), double-buffered inputs and outputs"}


if __name__ == "__main__":
    sys.exit(main())
