#!/usr/bin/env python
"""Throughput of the batched block selected inverse (libselinv) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one call of the library's public entry point over one batch of
synthetic input (selected inverse + log det + the solve where the workload
asks for it), all of it on the device.  Default workload: 4096 independent
chains of 64 blocks of 16 (float64, diag load 2.0, one right-hand side).
The metric is b x b blocks per second (value = all ranks' blocks / time).

Under torchrun each rank owns its own slice of chains (batch elements are
independent, so there is no data-path collective: weak scaling); a barrier and
a max-over-ranks of the device-timed region are the only cross-rank steps.
The default workload's inputs (> 2 GB) are larger than L2, so no flush is
needed between its steps; workloads whose inputs fit in L2 (126 MB) get a
256 MB device write before every timed step, outside the step's own events,
and are timed by those per-step events.

``--impl reference`` times the CPU oracle (the plain C implementation the
tests check against) on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_spd_selected_b200 import inputs  # noqa: E402

PROFILES = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = {
    "chain_tiny_kernel": ["chain_tiny.cu", "common.cuh"],
    "chain_small_kernel": ["chain_small.cu", "warp16.cuh", "common.cuh"],
    "chain_mid_kernel": ["chain_mid.cu", "quad32.cuh", "warp16.cuh", "common.cuh"],
    "seg_collect_kernel": ["chain_seg.cu", "quad32.cuh", "warp16.cuh", "common.cuh"],
    "seg_distribute_kernel": ["chain_seg.cu", "quad32.cuh", "warp16.cuh", "common.cuh"],
    "chain_large_kernel": ["chain_large.cu", "common.cuh"],
    "tree_collect_kernel": ["tree.cu", "warp16.cuh", "common.cuh"],
    "chain_backward_kernel": ["chain_backward.cu", "warp16.cuh", "common.cuh"],
    "tree_bw_collect_kernel": ["tree.cu", "warp16.cuh", "common.cuh"],
    "bidiag_inverse_kernel": ["bidiag.cu", "warp16.cuh", "common.cuh"],
    "jn_target_kernel": ["junction.cu", "warp16.cuh", "common.cuh"],
}


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="chain_4096x64_b16", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--dtype", default="f64", choices=["f64", "f32"])
    ap.add_argument("--batch", type=int, default=None, help="override the per-GPU batch (profiling runs)")
    ap.add_argument("--length", type=int, default=None,
                    help="override the chain length / tree size (profiling runs of a smaller case)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--op", default="selinv", choices=["selinv", "sample", "backward", "bidiag"],
                    help="selinv: selected inverse + log det (+ solve); sample: Gaussian draw "
                         "eta = A^-1 r + L^-T z + log det (chains; on trees eta = L^-T z); backward: "
                         "cotangents of diag and lower (edge) from those of G_diag and G_lower (G_edge); "
                         "chains and trees, b <= 16; bidiag: the selected inverse of a block "
                         "lower-bidiagonal matrix with general blocks of the chain workload's shape (b <= 16)")
    ap.add_argument("--configs", default="all", choices=["all", "one"],
                    help="all (default): with the default workload and op, also measure every other workload "
                         "of the metric (and the float32 repeat) and report them under per_config; one: the "
                         "named workload only")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers

def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(ROOT, "sparse_spd_selected_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, dtype: str = "f64"):
    """DRAM bytes per launch from the committed ncu summary of this dtype, if the kernel is unchanged since."""
    suffix = "" if dtype == "f64" else f"_{dtype}"
    path = os.path.join(PROFILES, f"{kernel}__{workload}{suffix}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    s = re.search(r"source_sha256_16:\s*([0-9a-f]+)", txt)
    if not m or not s or s.group(1) != source_hash(kernel):
        return None
    return float(m.group(1))


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.dev = device_index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (getattr(self, "out", "") or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_inputs(w, elems, op):
    g = inputs.generate(w, elements=elems)
    if op == "sample":
        g["z"] = inputs.standard_normals(w.batch, w.L, w.b, w.seed, elems)
    if op == "bidiag":
        g = dict(zip(("diag", "lower"), inputs.bidiag_inputs(w.batch, w.L, w.b, w.seed, 2.0, elems)))
    if op == "backward" and w.kind == "tree":
        g["Gb_diag"], g["Gb_edge"] = inputs.tree_cotangents(w.batch, w.L, w.b, w.seed, elems)
    elif op == "backward":
        g["Gb_diag"], g["Gb_lower"] = inputs.cotangents(w.batch, w.L, w.b, w.seed, elems)
    return g


def oracle_run(oracle, w, g, op):
    if w.kind == "tree" and op == "sample":
        oracle.tree_sample(g["parent"], g["diag"], g["edge"], g["z"])
    elif w.kind == "tree" and op == "backward":
        oracle.tree_backward(g["parent"], g["diag"], g["edge"], g["Gb_diag"], g["Gb_edge"])
    elif w.kind == "tree":
        oracle.tree(g["parent"], g["diag"], g["edge"])
    elif w.kind == "junction":
        oracle.junction(g["diag"], g["edge_index"], g["edge_val"])
    elif op == "sample":
        oracle.chain_sample(g["diag"], g["lower"], g["z"], rhs=g.get("rhs"))
    elif op == "backward":
        oracle.chain_backward(g["diag"], g["lower"], g["Gb_diag"], g["Gb_lower"])
    elif op == "bidiag":
        oracle.bidiag(g["diag"], g["lower"])
    else:
        oracle.chain(g["diag"], g["lower"], g.get("rhs"))


def oracle_workload(w, op):
    """The workload the oracle times: the same, except for the backward, whose
    dense definition costs O((L b)^3) per chain or tree: there chains or trees
    of 512 / b blocks drawn by the same recipe stand in (a few seconds each)."""
    if w.kind == "junction" and w.L * w.b > 512:
        side = max(2, int((512 // w.b) ** 0.5))
        return (dataclasses.replace(w, L=side * side),
                f" (lattices of {side} x {side} blocks drawn like {w.name}'s: the dense definition is O((n b)^3))")
    if op in ("backward", "bidiag") and w.L * w.b > 512:
        n = max(2, 512 // w.b)
        what = "trees" if w.kind == "tree" else "chains"
        return dataclasses.replace(w, L=n), f" ({what} of {n} blocks drawn like {w.name}'s)"
    return w, ""


def cpu_baseline(w, dtype_name, op="selinv", budget_s=10.0):
    """The oracle, as it stands, on a bounded sample of the same workload (host cores)."""
    import oracle
    oracle.build()
    w, note = oracle_workload(w, op)
    n_probe = 32 if w.kind != "grid" else 1
    elems = list(range(min(n_probe, w.batch)))
    g = oracle_inputs(w, elems, op)

    def run(gg):
        oracle_run(oracle, w, gg, op)

    t0 = time.perf_counter()
    run(g)
    dt = time.perf_counter() - t0
    n = int(min(w.batch, max(len(elems), len(elems) * budget_s / max(dt, 1e-6))))
    if n > len(elems):
        elems = list(range(n))
        g = oracle_inputs(w, elems, op)
        t0 = time.perf_counter()
        run(g)
        dt = time.perf_counter() - t0
    blocks = len(elems) * w.L
    unit_name = "trees" if w.kind == "tree" else "chains"
    return {"value": blocks / dt, "unit": "blocks/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{len(elems)} of {w.batch} {unit_name} ({w.name}, float64){note}, {dt:.2f} s"}


_JPLAN = {}


def _lattice_plan(w):
    """The junction plan of a lattice workload (cached; built on the current device)."""
    if w.name not in _JPLAN:
        from sparse_spd_selected_b200 import selinv
        side = int(round(w.L ** 0.5))
        _JPLAN[w.name] = selinv.JunctionPlan(w.L, inputs.grid_edges(side, w.L // side))
    return _JPLAN[w.name]


def _lattice_m(w):
    side = int(round(w.L ** 0.5))
    return inputs.grid_edges(side, w.L // side).shape[1]


def _lattice_nnz(w):
    return _lattice_plan(w).nnz


def junction_flops(w, batch):
    """Nominal flops of the general sparse path: 2 b^3 per block product it takes.
    Per node v with clique N(v) (d = |N(v)|): d(d + 1)/2 updates it sends to
    its ancestors' blocks, d products W = A' P, d^2 + d products in the
    distribute; plus b^3 for the inverse of S_v."""
    import numpy as np
    pl = _lattice_plan(w)
    pos = np.empty(w.L, dtype=np.int64)
    pos[pl.order] = np.arange(w.L)
    i, j = pl.S_index
    later = np.where(pos[i] > pos[j], j, i)          # the earlier-eliminated end owns the pair
    d = np.bincount(later, minlength=w.L).astype(np.float64)
    prods = d * (d + 1) / 2 + d + d * d + d
    return batch * (2.0 * w.b ** 3 * prods.sum() + w.L * float(w.b) ** 3)


def algorithmic_bytes(w, es, batch, op="selinv"):
    """Bytes the method must move: read D and B (or edge) blocks, write G_diag and G_lower
    (or G_edge) blocks, plus the right-hand side and solution when solving.  A draw reads
    D, B, r and z and writes eta (a tree draw has no r)."""
    b2 = w.b * w.b
    if w.kind == "junction":
        # read D and the input blocks, write G_diag and G on the filled pattern S
        return es * b2 * batch * (2 * w.L + _lattice_m(w) + _lattice_nnz(w))
    if op == "bidiag":
        # read M_ii and M_{i+1,i}, write G_ii and G_{i+1,i}
        nodes, edges = batch * w.L, batch * (w.L - 1)
        return es * 2 * b2 * (nodes + edges)
    if op == "backward":
        # read D, G_diag, Gb_diag and B (edge), G_lower (G_edge), Gb_lower (Gb_edge); write Db and Bb (Eb)
        nodes, edges = batch * w.L, batch * (w.L - 1)
        return es * 4 * b2 * (nodes + edges)
    if op == "sample" and w.kind == "tree":
        n = batch * w.L
        return es * (b2 * n + b2 * (n - batch) + 2 * w.b * n)
    if op == "sample":
        nodes, edges = batch * w.L, batch * (w.L - 1)
        return es * (b2 * nodes + b2 * edges + 3 * w.b * nodes)
    if w.kind == "tree":
        n = batch * w.L
        return es * (b2 * n + b2 * (n - batch) + b2 * n + b2 * (n - batch))
    nodes, edges = batch * w.L, batch * (w.L - 1)
    byt = es * (b2 * nodes + b2 * edges + b2 * nodes + b2 * edges)
    if w.solve:
        byt += es * 2 * w.b * nodes
    return byt


def algorithmic_flops(w, batch, op="selinv"):
    """Nominal 7 b^3 flops per block: collect (Cholesky b^3/3 + trsm b^3 + syrk b^3) and
    distribute (inverse 2b^3/3 + trmm b^3 + gemm 2b^3 + symmetric half-gemm b^3).  A draw
    needs the collect only (7 b^3 / 3; its triangular solves are O(b^2)).  The general
    sparse path counts its own products (junction_flops)."""
    if w.kind == "junction":
        return junction_flops(w, batch)
    # backward: the collect's 7/3 b^3, then six products in the reversed distribute
    # step and five in the reversed collect step, 2 b^3 each
    per = {"sample": 7.0 / 3.0, "backward": 73.0 / 3.0}.get(op, 7.0)
    return per * w.b ** 3 * batch * w.L


def fp64_peak_tflops(torch):
    """cuBLAS DGEMM 8192^3 (FP64 tensor cores), best of 5."""
    a = torch.randn(8192, 8192, dtype=torch.float64, device="cuda")
    b = torch.randn_like(a)
    for _ in range(2):
        a @ b
    best = 0.0
    for _ in range(5):
        s, e = torch.cuda.Event(True), torch.cuda.Event(True)
        s.record()
        a @ b
        e.record()
        torch.cuda.synchronize()
        best = max(best, 2 * 8192 ** 3 / (s.elapsed_time(e) / 1e3) / 1e12)
    del a, b
    return best


# ------------------------------------------------------------------ sharding

def shard_elements(rank: int, batch_per_rank: int):
    """Batch elements (chains or trees) owned by `rank`: a contiguous slice.

    Elements are independent, so ranks never exchange data; each element's
    inputs come from its own seeded generator, so the union over ranks is one
    larger batch of distinct elements (weak scaling)."""
    return list(range(rank * batch_per_rank, (rank + 1) * batch_per_rank))


def max_over_ranks(value_ms: float, world: int, device=None) -> float:
    """Slowest rank's time (the job's time): an all-reduce MAX when world > 1."""
    if world <= 1:
        return value_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank: int, steps: int, max_ms: float) -> float:
    """Units processed by all ranks per second of the slowest rank's time."""
    return world * units_per_rank * steps / (max_ms / 1e3)


# ------------------------------------------------------------------ arms

# The workloads the metric is quoted on, one bench line: the headline
# (4096 chains of 64 blocks of 16) carries the top-level keys; every workload,
# the float32 repeat of the long b = 32 chains included, is measured in the
# same run and reported under "per_config".
HEADLINE = "chain_4096x64_b16"
PER_CONFIG = [("chain_1x8_b4", "f64"), ("chain_4096x64_b16", "f64"), ("chain_64x4096_b32", "f64"),
              ("chain_64x4096_b32", "f32"), ("forest_8x32768_b16", "f64"), ("grid_256x128_b128", "f64")]


L2_FLUSH_BYTES = 256 << 20      # more than twice the B200's 126 MB L2


def fits_l2(w):
    """Inputs small enough to stay in L2 between steps (then flushed before each timed step)."""
    return w.L * w.batch * w.b * w.b * 8 <= L2_FLUSH_BYTES


def config_dict(w, batch, world, op, full_size):
    """The bench line's `config`: the same dict for both arms of one workload."""
    l2 = "inputs larger than L2 (no flush)" if not fits_l2(w) else \
        ("inputs fit in L2: a 256 MB device write flushes L2 before every timed step, outside the "
         "step's own CUDA events; time = sum of the per-step event times")
    return {"workload": w.name if full_size else f"{w.name} (batch {batch}, length {w.L} per GPU)",
            "global_batch": batch * world, "block": w.b, "L_or_n": w.L,
            "solve": bool(w.solve) and op in ("selinv", "sample"), "op": op,
            "parallelism": f"dp{world} (independent chains per GPU)", "l2": l2}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w0 = inputs.WORKLOADS[args.workload]
    import oracle
    oracle.build()
    w, note = oracle_workload(w0, args.op)
    n_per_step = {"chain": 64, "tree": 1, "grid": 1, "junction": 4}[w.kind]
    if w.kind == "chain" and w.L * w.b ** 3 > 64 * 16 ** 3 * 64:
        n_per_step = 2
    if args.op in ("backward", "bidiag") and w.kind == "chain":
        n_per_step = 16
    elems = list(range(min(n_per_step, w.batch)))
    g = oracle_inputs(w, elems, args.op)
    times = []
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle_run(oracle, w, g, args.op)
        if it >= args.warmup:
            times.append(time.perf_counter() - t0)
    blocks = len(elems) * w.L
    value = blocks * len(times) / sum(times)
    sample = f"{len(elems)} of {w.batch} {'trees' if w.kind == 'tree' else 'chains'} per step{note}"
    full_size = args.length is None and (args.batch is None or args.batch == w0.batch)
    line = {
        "impl": "reference", "metric": metric_name(args.op, args.dtype), "value": value, "unit": "blocks/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": config_dict(w0, args.batch or w0.batch, args.gpus, args.op, full_size),
        "cpu_baseline": {"value": value, "unit": "blocks/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample + " (the oracle computes in float64)"},
        "e2e": {"value": value, "unit": "blocks/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def metric_name(op, dtype):
    what = {"sample": "draw", "backward": "selinv backward", "bidiag": "bidiag selinv"}.get(op, "selinv")
    return f"{what} blocks/s ({'fp64' if dtype == 'f64' else 'fp32'})"


_FP64_PEAK = {}


def fp64_peak_cached(torch):
    if "v" not in _FP64_PEAK:
        _FP64_PEAK["v"] = fp64_peak_tflops(torch)
    return _FP64_PEAK["v"]


def build_step(w, dtype, op, batch, elems):
    """Inputs, outputs, workspace and the step closure of one workload.

    Returns a dict with step, out, dev_in, host_in, kernel, launches_per_step."""
    import torch
    from sparse_spd_selected_b200 import selinv

    tdt = torch.float64 if dtype == "f64" else torch.float32
    if w.kind == "grid":
        diag, lower, rhs, _ = inputs.grid_inputs_torch(batch, w.b, w.seed, "cuda", tdt, w.solve)
        host_in = {"diag": diag.cpu().pin_memory(), "lower": lower.cpu().pin_memory()}
        if rhs is not None:
            host_in["rhs"] = rhs.cpu().pin_memory()
        if op == "sample":
            host_in["z"] = torch.from_numpy(inputs.standard_normals(batch, w.L, w.b, w.seed, elems)).to(
                tdt).pin_memory()
        g = None
    else:
        g = inputs.generate(w, elements=elems)   # per-element seeds: rank r owns its own slice
        if op == "bidiag":
            if w.kind != "chain" or w.b > 16:
                raise SystemExit("--op bidiag runs on chain workload shapes with b <= 16")
            g = dict(zip(("diag", "lower"), inputs.bidiag_inputs(w.batch, w.L, w.b, w.seed, 2.0, elems)))
        if op == "sample":
            if w.b > 16 and dtype != "f64":
                raise SystemExit("--op sample with b > 16 runs in float64 only")
            g["z"] = inputs.standard_normals(w.batch, w.L, w.b, w.seed, elems)
        if op == "backward":
            if w.b > 16:
                raise SystemExit("--op backward runs on workloads with b <= 16")
            g.pop("rhs", None)
            if w.kind == "tree":
                g["Gb_diag"], g["Gb_edge"] = inputs.tree_cotangents(w.batch, w.L, w.b, w.seed, elems)
            else:
                g["Gb_diag"], g["Gb_lower"] = inputs.cotangents(w.batch, w.L, w.b, w.seed, elems)
        host_in = {}
        for k in [k for k, v in g.items() if v is not None and k not in ("parent", "edge_index")]:
            host_in[k] = torch.from_numpy(g[k]).to(tdt).pin_memory()
            if k != "tau":
                g[k] = None                      # free the float64 host copy as we go
        dev_in = {k: v.to("cuda", non_blocking=True) for k, v in host_in.items()}
        torch.cuda.synchronize()

    if w.kind == "junction":
        plan = _lattice_plan(w)
        kernel = "jn_target_kernel"
        launches_per_step = plan.launches
        out = {"G_diag": torch.empty_like(dev_in["diag"]),
               "G_lower": torch.empty((batch, plan.nnz, w.b, w.b), dtype=tdt, device="cuda"),
               "logdet": torch.empty(batch, dtype=torch.float64, device="cuda"),
               "info": torch.empty(batch, dtype=torch.int32, device="cuda")}
        ws = torch.empty(plan.workspace_size(tdt, w.b, batch), dtype=torch.uint8, device="cuda")

        def step():
            selinv.junction(plan, dev_in["diag"], dev_in["edge_val"], check=False, out=out, workspace=ws)
    elif w.kind == "tree":
        plan = selinv.TreePlan(g["parent"])
        # init, collect sweep, distribute sweep (trees with more than one node), log-det finalize
        launches_per_step = 4 if w.L > 1 else 3
        out = {"G_diag": torch.empty_like(dev_in["diag"]), "G_edge": torch.empty_like(dev_in["diag"]),
               "logdet": torch.empty(batch, dtype=torch.float64, device="cuda"),
               "info": torch.empty(batch, dtype=torch.int32, device="cuda")}
        ws = torch.empty(plan.workspace_size(tdt, w.b), dtype=torch.uint8, device="cuda")
        if op == "backward":
            fwd = selinv.selinv_tree(plan, dev_in["diag"], dev_in["edge"])
            for k in ("G_diag", "G_edge"):
                dev_in[k] = fwd[k]
                host_in[k] = fwd[k].cpu().pin_memory()
            kernel = "tree_bw_collect_kernel"
            out = {"Db": torch.empty_like(dev_in["diag"]), "Eb": torch.empty_like(dev_in["diag"]),
                   "info": out["info"]}
            ws = torch.empty(plan.backward_workspace_size(tdt, w.b), dtype=torch.uint8, device="cuda")

            def step():
                selinv.tree_backward(plan, dev_in["diag"], dev_in["edge"], dev_in["G_diag"], dev_in["G_edge"],
                                     dev_in["Gb_diag"], dev_in["Gb_edge"], check=False, out=out, workspace=ws)
        elif op == "sample":
            kernel = "tree_collect_draw_kernel"
            out = {"eta": torch.empty_like(dev_in["z"]), "logdet": out["logdet"], "info": out["info"]}

            def step():
                selinv.tree_sample(plan, dev_in["diag"], dev_in["edge"], dev_in["z"], check=False, out=out,
                                   workspace=ws)
        else:
            kernel = "tree_collect_kernel"

            def step():
                selinv.selinv_tree(plan, dev_in["diag"], dev_in["edge"], check=False, out=out, workspace=ws)
    else:
        if w.kind == "grid":
            dev_in = {"diag": diag, "lower": lower}
            if rhs is not None:
                dev_in["rhs"] = rhs
            if op == "sample":
                dev_in["z"] = host_in["z"].to("cuda")
        L, b = w.L, w.b
        out = {"G_diag": torch.empty((batch, L, b, b), dtype=tdt, device="cuda"),
               "G_lower": torch.empty((batch, L - 1, b, b), dtype=tdt, device="cuda"),
               "logdet": torch.empty(batch, dtype=torch.float64, device="cuda"),
               "info": torch.empty(batch, dtype=torch.int32, device="cuda")}
        if "rhs" in dev_in:
            out["x"] = torch.empty((batch, L, b), dtype=tdt, device="cuda")
        ws = torch.empty(max(selinv.chain_workspace_size(tdt, batch, L, b, True, "rhs" in dev_in), 1),
                         dtype=torch.uint8, device="cuda")
        launches_per_step = 1
        segments = selinv.chain_segments(batch, L, b, True, "rhs" in dev_in)
        if op == "bidiag":
            kernel = "bidiag_inverse_kernel"
            out = {"G_diag": torch.empty_like(dev_in["diag"]), "G_lower": torch.empty_like(dev_in["lower"]),
                   "info": torch.empty(batch, dtype=torch.int32, device="cuda")}
        elif op == "backward":
            # the forward's outputs are the backward's inputs (computed once, outside the timing)
            fwd = selinv.selinv_chain(dev_in["diag"], dev_in["lower"])
            for k in ("G_diag", "G_lower"):
                dev_in[k] = fwd[k]
                host_in[k] = fwd[k].cpu().pin_memory()
            kernel = "chain_backward_kernel"
            out = {"Db": torch.empty_like(dev_in["diag"]), "Bb": torch.empty_like(dev_in["lower"]),
                   "info": torch.empty(batch, dtype=torch.int32, device="cuda")}
            ws = torch.empty(max(selinv.chain_backward_workspace_size(tdt, batch, L, b), 1), dtype=torch.uint8,
                             device="cuda")
        elif op == "sample":
            kernel = "chain_small_kernel (draw mode)" if b <= 16 else "chain_large_kernel (draw mode)"
            out = {"eta": torch.empty((batch, L, b), dtype=tdt, device="cuda"),
                   "logdet": torch.empty(batch, dtype=torch.float64, device="cuda"),
                   "info": torch.empty(batch, dtype=torch.int32, device="cuda")}
            ws = torch.empty(max(selinv.chain_workspace_size(tdt, batch, L, b, False, True), 1),
                             dtype=torch.uint8, device="cuda")
        elif b <= 8 and L <= 16 and tdt == torch.float64:
            kernel = "chain_tiny_kernel"
        elif b <= 16:
            kernel = "chain_small_kernel"
        elif segments > 0:
            # segments' collect, separators' D', their two-ended chain, segments' distribute, log det
            kernel = "seg_collect_kernel"
            launches_per_step = 5
        elif b <= 32 and "rhs" not in dev_in:
            kernel = "chain_mid_kernel"
        else:
            kernel = "chain_large_kernel"

        if op == "bidiag":
            def step():
                selinv.bidiag(dev_in["diag"], dev_in["lower"], check=False, out=out)
        elif op == "backward":
            def step():
                selinv.chain_backward(dev_in["diag"], dev_in["lower"], dev_in["G_diag"], dev_in["G_lower"],
                                      dev_in["Gb_diag"], dev_in["Gb_lower"], check=False, out=out, workspace=ws)
        elif op == "sample":
            def step():
                selinv.chain_sample(dev_in["diag"], dev_in["lower"], dev_in["z"], dev_in.get("rhs"), check=False,
                                    out=out, workspace=ws)
        else:
            def step():
                selinv.selinv_chain(dev_in["diag"], dev_in["lower"], dev_in.get("rhs"), check=False, out=out,
                                    workspace=ws)
    return {"step": step, "out": out, "dev_in": dev_in, "host_in": host_in, "kernel": kernel,
            "launches_per_step": launches_per_step, "keep": (ws,)}


def graph_device_us(step, stream, reps=50):
    """Device time of one call with the host out of the way: `reps` calls captured
    in one CUDA graph and replayed (the library's calls are stream-ordered and
    allocate nothing when given outputs and workspace)."""
    import torch
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(stream)
    with torch.cuda.stream(s):
        step()                                   # warm the capture stream
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        for _ in range(reps):
            step()
    with torch.cuda.stream(s):                   # replays run on the current stream: time them there
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        for _ in range(5):
            g.replay()
        e.record(s)
    torch.cuda.synchronize()
    us = a.elapsed_time(e) * 1e3 / (5 * reps)
    del g
    return us


def measure(w, dtype, op, batch, steps, warmup, rank, world, local, full_size, want_cpu, want_e2e):
    """One workload, timed as the bench line reports it."""
    import torch
    import torch.distributed as dist

    es = 8 if dtype == "f64" else 4
    cpu = cpu_baseline(w, dtype, op) if want_cpu else None     # host only, before the GPU work
    elems = shard_elements(rank, batch)
    stream = torch.cuda.current_stream()
    S = build_step(w, dtype, op, batch, elems)
    step, out, dev_in, host_in = S["step"], S["out"], S["dev_in"], S["host_in"]
    kernel, launches_per_step = S["kernel"], S["launches_per_step"]

    # correctness guard: the last warm-up step must report every element SPD
    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    if bool((out["info"] != -1).any()):
        raise SystemExit(f"bench input reported not SPD ({w.name})")

    K = steps
    k_start = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    k_end = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dev_index = torch.cuda.current_device()
    try:
        dev_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[local])
    except Exception:
        pass
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    small = fits_l2(w)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda") if small else None
    with ClockSampler(dev_index) as clk:
        t_start.record(stream)
        for i in range(K):
            if flush is not None:
                flush.fill_(i & 0xFF)            # evicts this step's inputs and outputs from L2
            k_start[i].record(stream)
            step()
            k_end[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    kernel_ms = sum(a.elapsed_time(b_) for a, b_ in zip(k_start, k_end)) / K
    if small:
        elapsed_ms = kernel_ms * K               # the flushes between steps are not the workload's time
    del flush
    elapsed_ms = max_over_ranks(elapsed_ms, world, "cuda")
    nodes_per_rank = batch * w.L
    value = job_throughput(world, nodes_per_rank, K, elapsed_ms)
    device_us = graph_device_us(step, stream) if small else None

    # end to end through the same call, inputs from pinned host memory, outputs read back
    e2e = None
    if want_e2e and host_in is not None:
        host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in out.items()}
        Ke = max(1, min(3, K))
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(Ke):
            for k, v in host_in.items():
                if k in dev_in:
                    dev_in[k].copy_(v, non_blocking=True)
            step()
            for k, v in out.items():
                host_out[k].copy_(v, non_blocking=True)
        e.record(stream)
        torch.cuda.synchronize()
        e2e_ms = s.elapsed_time(e)
        e2e_ms = max_over_ranks(e2e_ms, world, "cuda")
        h2d = sum(v.numel() * v.element_size() for k, v in host_in.items() if k in dev_in)
        d2h = sum(v.numel() * v.element_size() for v in out.values())
        e2e = {"value": job_throughput(world, nodes_per_rank, Ke, e2e_ms), "unit": "blocks/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    hbm, src = hbm_peak()
    byt = algorithmic_bytes(w, es, batch, op)
    t_ms = kernel_ms
    hbm_achieved = byt / (t_ms / 1e3) / 1e9
    flops = algorithmic_flops(w, batch, op)
    flop_rate = flops / (t_ms / 1e3) / 1e12
    traffic = profiled_traffic(kernel, w.name, dtype) if full_size else None
    hbm_src = f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else "fallback 6650 GB/s"
    ridge = 35.5e12 / (hbm * 1e9)                      # FP64 flop per byte where the two roofs meet
    contraction = w.kind == "junction" and flops / byt > ridge
    hbm_side = {"achieved": hbm_achieved, "peak": hbm, "unit": "GB/s", "frac": hbm_achieved / hbm,
                "peak_source": hbm_src}
    # the segmented b = 32 path reads and writes float32 but computes in float64
    # (operands widened in registers, the FP64 tensor-core products and inverse)
    arith = "f64" if dtype == "f64" or kernel == "seg_collect_kernel" else dtype
    if (w.b >= 32 or op == "backward" or contraction) and arith == "f64":
        # arithmetic intensity 7 b^3 / (32 b^2) flop/byte: past the FP64 ridge from b = 32 on
        peak = fp64_peak_cached(torch)
        roof = {"bound": "tensor", "achieved": flop_rate, "peak": peak, "unit": "TFLOP/s",
                "frac": flop_rate / peak, "traffic": traffic,
                "peak_source": "measured in this run: cuBLAS DGEMM 8192^3 (FP64 tensor cores)",
                "algorithmic_flops_per_launch": flops, "kernel": kernel, "hbm": hbm_side}
        if arith != dtype:
            roof["note"] = f"{dtype} inputs and outputs, float64 arithmetic on the FP64 tensor cores"
    elif w.b >= 32:
        # fp32 runs on the FP32 pipes: 148 SMs x 128 lanes x 2 flop x 1965 MHz
        peak = 148 * 128 * 2 * 1.965e9 / 1e12
        roof = {"bound": "alu", "achieved": flop_rate, "peak": peak, "unit": "TFLOP/s",
                "frac": flop_rate / peak, "traffic": traffic,
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 flop x 1965 MHz max SM clock",
                "algorithmic_flops_per_launch": flops, "kernel": kernel, "hbm": hbm_side}
    else:
        roof = {"bound": "hbm", "achieved": hbm_achieved, "peak": hbm, "unit": "GB/s", "frac": hbm_achieved / hbm,
                "traffic": traffic, "peak_source": hbm_src, "algorithmic_bytes_per_launch": byt, "kernel": kernel}
    if small:
        roof["note"] = ("inputs fit in L2: achieved uses the per-step device time with L2 flushed before "
                        "each step; device_us_per_call is one call's time inside a CUDA graph of "
                        "back-to-back calls (warm L2)")
    res = {"value": value, "ms_per_step": elapsed_ms / K, "kernel_ms": kernel_ms, "roofline": roof,
           "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": K * launches_per_step, "clocks": clk.summary(),
           "kernel": kernel, "config": config_dict(w, batch, world, op, full_size), "dtype": arith}
    if arith != dtype:
        res["data_dtype"] = dtype
    if device_us is not None:
        res["device_us_per_call"] = device_us
    del S, step, out, dev_in, host_in
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    w = inputs.WORKLOADS[args.workload]
    full_size = args.length is None and (args.batch is None or args.batch == w.batch)
    if args.length is not None:
        w = dataclasses.replace(w, L=args.length)
    batch = args.batch or w.batch
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    head = measure(w, args.dtype, args.op, batch, args.steps, args.warmup, rank, world, local, full_size,
                   want_cpu, not args.no_e2e)
    per_config = None
    if args.configs == "all" and world == 1 and full_size and args.op == "selinv" and w.name == HEADLINE \
            and args.dtype == "f64":
        per_config = {}
        for name, dt in PER_CONFIG:
            key = name if dt == "f64" else f"{name}_{dt}"
            if name == w.name and dt == args.dtype:
                r = head
            else:
                wc = inputs.WORKLOADS[name]
                r = measure(wc, dt, "selinv", wc.batch, args.steps, args.warmup, rank, world, local, True,
                            want_cpu, not args.no_e2e)
            per_config[key] = {k: r[k] for k in ("value", "ms_per_step", "kernel_ms", "roofline", "cpu_baseline",
                                                 "e2e", "clocks", "gpu_launches", "dtype", "config")}
            for k in ("device_us_per_call", "data_dtype"):
                if k in r:
                    per_config[key][k] = r[k]
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": metric_name(args.op, args.dtype),
        "value": head["value"], "unit": "blocks/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": head["dtype"], "data": "synthetic",
        "config": head["config"],
        "roofline": head["roofline"],
        "cpu_baseline": head["cpu_baseline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"] + sum(
            v["gpu_launches"] for k, v in (per_config or {}).items() if k != w.name),
        "clocks": head["clocks"],
        "kernel_ms": head["kernel_ms"],
    }
    for k in ("device_us_per_call", "data_dtype"):
        if k in head:
            line[k] = head[k]
    if per_config is not None:
        line["per_config"] = per_config
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
