"""Benchmark of the fused EAAS + on-the-fly equivariant attention hot path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
                    [--decompose]

One step = one pass of the whole hot path over one synthetic system:
radius graph (egat_build_graph) -> attention plan (egat_build_attention_plan,
tensor-core shapes) -> EAAS source coupling (egat_eaas_couple_planned with the
plan's rotations on tensor-core shapes, egat_eaas_couple otherwise) -> on-the-fly
attention with the target coupling fused (egat_otf_attention_tiled on
tensor-core shapes, egat_otf_attention_coupled otherwise).
The default workload is the 32,768-atom, K = 256, lmax = 2, bf16-storage
system.  Inputs are resident in HBM when the timed region starts; L2 is
flushed (a 256 MiB write) before every timed step, outside the step's events.

Prints ONE JSON line (rank 0).  ``value`` is atoms/s over all ranks; edges/s,
per-kernel times, the roofline of the dominant kernel, the CPU oracle baseline,
an end-to-end figure through host buffers, the backward pass and the forward
step of the other two bf16 workloads (4,096 atoms; 100,000 atoms at lmax 3)
ride along.

Roofline of the dominant kernel (the fused attention): ``achieved`` is its
compulsory bytes — every input row read once (h' and k of every source, q and
r of every target, the padded neighbour lists) and the output written once —
over its CUDA-event time; ``traffic`` is the DRAM traffic ncu measured for the
same kernel build and workload (null when the kernel sources changed since).
The per-edge accounting of the method (each neighbour's key and value rows
loaded once per edge) rides along as ``effective``: the kernel serves those
loads from L2 and shared memory, so that figure exceeds the HBM peak and is
not a bound.

Multi-GPU (torchrun, N > 1): ONE system is split across the ranks by space
(``equivariant_graph_attention_b200.halo``: each rank couples its own atoms,
one all-to-all exchanges the boundary atoms' h' and k rows, each rank runs the
attention of its own atoms) and the line reports the system's atoms per second
of the slowest rank's decomposed step (strong scaling).  ``--replicas`` runs
independent systems instead (same shape, seeded by rank; no data-path
collective; weak scaling); ``--decompose`` forces the split at N = 1 too.
Timing is the max over ranks.  ``--impl reference`` times the CPU oracle on the
same workload (rank 0 only, on the host's cores).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from equivariant_graph_attention_b200 import synth  # noqa: E402

METRIC = "atoms/s & edges/s, fused EAAS+on-the-fly attention; % of HBM roofline"
DEFAULT_WORKLOAD = "uniform32768_K256_l2_bf16"
EXTRA_WORKLOADS = ["uniform4096_l2_bf16", "uniform100000_l3_bf16"]
FLUSH_BYTES = 256 << 20
#: kernels this library launches per step: graph (assign, scan x3, scatter,
#: rank, fill, truncated-row fix) + attention plan (tensor-core shapes: unions,
#: masks and tile records in one kernel; a second for the records at lmax 3)
#: + source coupling + fused attention
LAUNCHES_GRAPH = 8


def launches_plan(lmax: int) -> int:
    return 1 if lmax <= 2 else 2
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attention_traffic.json")
KERNEL_SOURCES = ["equivariant_graph_attention_b200/csrc/attention.cu",
                  "equivariant_graph_attention_b200/csrc/attention_tc.cu",
                  "equivariant_graph_attention_b200/csrc/plan.cu",
                  "equivariant_graph_attention_b200/csrc/egat_device.cuh",
                  "equivariant_graph_attention_b200/csrc/egat_async.cuh"]
#: library kernels per decomposed step and rank besides the plan: three row
#: gathers (own h, q, k), the source coupling, two send-buffer gathers and the
#: attention
DECOMP_LAUNCHES = 7
#: oracle worker processes at most (each holds its own copy of a few hundred MB)
MAX_ORACLE_WORKERS = 32


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


def storage_bytes(wl: synth.Workload) -> int:
    return 2 if wl.dtype == "bf16" else 4


def attention_bytes(wl: synth.Workload, edges: int) -> dict:
    """Bytes of steps 3+4 (the fused attention).

    compulsory: every row the kernel needs, once — the value (h') and key row
    of every source, the query row and position of every target, its padded
    neighbour-list row and count, and its float32 output row.
    per_edge: the method's own accounting — per target its list row, count,
    q_i, r_i and output row, and per real edge the neighbour's key and value
    rows (each neighbour row loaded once per edge).
    """
    s = storage_bytes(wl)
    N, D, C, H, dk, K = wl.n, wl.D, wl.C, wl.H, wl.dk, wl.K
    per_target = K * 4 + 4 + H * dk * s + 12 + D * C * 4
    compulsory = N * (D * C * s + H * dk * s) + N * per_target
    per_edge = N * per_target + edges * (D * C * s + H * dk * s)
    return {"compulsory": compulsory, "per_edge": per_edge}


def eaas_bytes(wl: synth.Workload) -> int:
    """Step 2: read h and r, write h' (each once)."""
    s = storage_bytes(wl)
    return wl.n * (2 * wl.D * wl.C * s + 12)


def edge_count(wl: synth.Workload, data: dict) -> int:
    """Real edges of the padded graph: sum over atoms of min(degree, K) (a k-d
    tree count on the integer grid, the same rows the library keeps)."""
    from scipy.spatial import cKDTree
    p = data["pos_q"].astype(np.float64)
    tree = cKDTree(p)
    deg = np.array([len(x) - 1 for x in tree.query_ball_point(p, float(wl.cutoff_q))])
    return int(np.minimum(deg, wl.K).sum())


def config_of(wl: synth.Workload, edges: int, ranks: int, decompose: bool = False) -> dict:
    """The ``config`` dict both arms print."""
    par = (f"one system split across {ranks} ranks by space (halo exchange)" if decompose
           else f"{ranks} independent systems (one per GPU)")
    return {"workload": wl.name, "atoms": wl.n, "edges": edges, "K": wl.K, "lmax": wl.lmax,
            "C": wl.C, "H": wl.H, "dk": wl.dk, "cutoff_A": wl.cutoff, "storage": wl.dtype,
            "accumulate": "f32",
            "l2": "flushed before every timed step (256 MiB write, untimed)",
            "parallelism": par}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- oracle
# The oracle is plain single-threaded numpy.  To time it on all host cores,
# targets are split over worker processes forked BEFORE any CUDA call (rank 0
# creates the pool first thing); each worker holds the workload's arrays from
# the fork and limits its BLAS threads to one.
_ORACLE_DATA: dict = {}


def _oracle_worker_init():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def _oracle_targets(rows) -> float:
    """Seconds the CPU oracle takes for the forward pass of targets ``rows``:
    their brute-force neighbour rows, the source coupling of the atoms they
    need, two-pass attention and target coupling."""
    from oracle.attention import forward
    from oracle.graph import radius_graph
    wl, data = _ORACLE_DATA["wl"], _ORACLE_DATA["data"]
    rows = np.asarray(rows, dtype=np.int64)
    t0 = time.perf_counter()
    lists, _ = radius_graph(data["pos_q"], wl.cutoff_q, K=wl.K, rows=rows)
    forward(data["h"], data["pos"], data["q"], data["k"], data["w1"], data["w2"], wl.lmax,
            lists, targets=rows)
    return time.perf_counter() - t0


class OraclePool:
    """A fork pool of oracle workers over one workload (created before CUDA)."""

    def __init__(self, wl: synth.Workload, data: dict, workers: int):
        import multiprocessing as mp
        _ORACLE_DATA.update(wl=wl, data=data)
        self.wl = wl
        self.workers = max(1, workers)
        self.pool = mp.get_context("fork").Pool(self.workers, initializer=_oracle_worker_init)

    def rate(self, per_worker: int, seed: int) -> tuple[float, float, int]:
        """(atoms/s, wall seconds, targets) over ``per_worker`` random targets per worker."""
        n = min(self.wl.n, per_worker * self.workers)
        rows = np.random.default_rng(seed).choice(self.wl.n, size=n, replace=False)
        chunks = [rows[i::self.workers] for i in range(self.workers)]
        t0 = time.perf_counter()
        self.pool.map(_oracle_targets, chunks, chunksize=1)
        wall = time.perf_counter() - t0
        return n / wall, wall, n

    def close(self):
        self.pool.terminate()
        self.pool.join()


def oracle_workers_default() -> int:
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    return max(1, min(cores, MAX_ORACLE_WORKERS))


def single_thread_rate(n_targets: int, seed: int) -> tuple[float, float]:
    """(atoms/s, seconds) of the oracle on one thread in this process."""
    try:
        from threadpoolctl import threadpool_limits
        lim = threadpool_limits(1)
    except Exception:
        lim = None
    wl = _ORACLE_DATA["wl"]
    rows = np.random.default_rng(seed).choice(wl.n, size=n_targets, replace=False)
    secs = _oracle_targets(rows)
    if lim is not None:
        lim.restore_original_limits()
    return n_targets / secs, secs


# ---------------------------------------------------------------------------- distributed
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks (the job's time is its slowest rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device) -> float:
    """`value` summed over all ranks (units processed by the whole job)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_rate(local_units: float, local_ms: float, device) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time."""
    return sum_over_ranks(local_units, device) / (max_over_ranks(local_ms, device) / 1000.0)


def run_reference(args, wl: synth.Workload):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    data = synth.make(wl)
    edges = edge_count(wl, data)
    workers = args.cpu_workers or oracle_workers_default()
    pool = OraclePool(wl, data, workers)
    try:
        for w in range(args.warmup):
            pool.rate(1, seed=99 + w)
        secs, atoms = 0.0, 0
        for s in range(args.steps):
            _, wall, n = pool.rate(args.ref_targets, seed=s)
            secs += wall
            atoms += n
    finally:
        pool.close()
    value = atoms / secs
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "atoms/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * secs / args.steps, "higher_is_better": True,
        "scaling": "strong" if args.decompose else "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl, edges, args.gpus, args.decompose),
        "cpu_baseline": {"value": value, "unit": "atoms/s", "cores": workers,
                         "kind": "oracle",
                         "sample": f"{args.ref_targets} random target atoms per worker and step "
                                   f"({workers} worker processes) of the {wl.n}-atom system "
                                   f"(brute-force neighbour rows, dense source coupling of their "
                                   f"neighbours, two-pass attention, dense target coupling)"},
        "e2e": {"value": value, "unit": "atoms/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- GPU arm
class ForwardStep:
    """Device inputs, outputs and the four calls of one forward step."""

    def __init__(self, wl, data, dev, attention: str = "auto"):
        import ctypes
        import torch
        from equivariant_graph_attention_b200 import egat
        self.wl, self.dev, self.egat = wl, dev, egat
        self.lib = lib = egat.load_library()
        st = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        self.st = st

        def td(x, dt):
            return torch.from_numpy(np.ascontiguousarray(x)).to(dev, dtype=dt)

        self.h, self.q, self.k = td(data["h"], st), td(data["q"], st), td(data["k"], st)
        self.pos, self.pos_q = td(data["pos"], torch.float32), td(data["pos_q"], torch.int32)
        self.w1, self.w2 = td(data["w1"], torch.float32), td(data["w2"], torch.float32)
        self.shape = egat.Shape(n=wl.n, lmax=wl.lmax, C=wl.C, H=wl.H, dk=wl.dk, K=wl.K,
                                dtype=wl.dtype)
        self.cshape = self.shape.c()
        self.gws = torch.empty(egat.egat_graph_workspace_bytes(wl.n), dtype=torch.uint8,
                               device=dev)
        self.nbr = torch.empty((wl.n, wl.K), dtype=torch.int32, device=dev)
        self.cnt = torch.empty(wl.n, dtype=torch.int32, device=dev)
        self.order = torch.empty(wl.n, dtype=torch.int32, device=dev)
        self.ovf = torch.zeros(1, dtype=torch.int32, device=dev)
        self.hp = torch.empty((wl.n, wl.D, wl.C), dtype=st, device=dev)
        self.out = torch.empty((wl.n, wl.D, wl.C), dtype=torch.float32, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self.sp = self.stream.cuda_stream
        plan_sz = ctypes.c_size_t(0)
        self.tiled = (lib.egat_attention_plan_bytes(ctypes.byref(self.cshape),
                                                    ctypes.byref(plan_sz)) == 0
                      and wl.dtype == "bf16" and wl.C == 128 and wl.H == 16 and wl.dk == 16
                      and attention != "per-target")
        if attention == "tiled" and not self.tiled:
            raise SystemExit("the tensor-core attention path does not support this workload")
        self.plan = torch.empty(max(plan_sz.value, 16), dtype=torch.uint8, device=dev)
        self.attn_name = "otf_attention_tiled" if self.tiled else "otf_attention_coupled"
        self.launches = LAUNCHES_GRAPH + (launches_plan(wl.lmax) if self.tiled else 0) + 2

    def graph(self):
        e, w = self.egat, self.wl
        rc = self.lib.egat_build_graph(self.pos_q.data_ptr(), w.n, w.cutoff_q, w.K, 0,
                                       self.nbr.data_ptr(), self.cnt.data_ptr(), 0,
                                       self.order.data_ptr(), self.ovf.data_ptr(),
                                       self.gws.data_ptr(), self.gws.numel(), self.sp)
        e._check("egat_build_graph", rc)

    def build_plan(self):
        import ctypes
        if self.tiled:
            rc = self.lib.egat_build_attention_plan(
                ctypes.byref(self.cshape), self.nbr.data_ptr(), self.cnt.data_ptr(),
                self.order.data_ptr(), self.pos.data_ptr(), self.plan.data_ptr(),
                self.plan.numel(), self.sp)
            self.egat._check("egat_build_attention_plan", rc)

    def couple(self):
        import ctypes
        if self.tiled:   # rotations from the plan's tile records
            rc = self.lib.egat_eaas_couple_planned(ctypes.byref(self.cshape), self.h.data_ptr(),
                                                   self.plan.data_ptr(), self.w1.data_ptr(),
                                                   self.hp.data_ptr(), self.sp)
            self.egat._check("egat_eaas_couple_planned", rc)
        else:
            rc = self.lib.egat_eaas_couple(ctypes.byref(self.cshape), self.h.data_ptr(),
                                           self.pos.data_ptr(), self.w1.data_ptr(),
                                           self.hp.data_ptr(), self.sp)
            self.egat._check("egat_eaas_couple", rc)

    def attend(self):
        import ctypes
        if self.tiled:
            rc = self.lib.egat_otf_attention_tiled(ctypes.byref(self.cshape), self.q.data_ptr(),
                                                   self.k.data_ptr(), self.hp.data_ptr(),
                                                   self.plan.data_ptr(), self.w2.data_ptr(),
                                                   self.out.data_ptr(), 1, self.sp)
            self.egat._check("egat_otf_attention_tiled", rc)
        else:
            rc = self.lib.egat_otf_attention_coupled(
                ctypes.byref(self.cshape), self.q.data_ptr(), self.k.data_ptr(),
                self.hp.data_ptr(), self.nbr.data_ptr(), self.cnt.data_ptr(),
                self.order.data_ptr(), self.pos.data_ptr(), self.w2.data_ptr(),
                self.out.data_ptr(), self.sp)
            self.egat._check("egat_otf_attention_coupled", rc)

    def run(self):
        self.graph()
        self.build_plan()
        self.couple()
        self.attend()

    def timed(self, steps: int, warmup: int, flush, barrier=None) -> dict:
        """Per-kernel and per-step CUDA-event times (ms, means over ``steps``)."""
        import torch
        for _ in range(warmup):
            flush.fill_(1)
            self.run()
        torch.cuda.synchronize(self.dev)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
        if barrier is not None:
            barrier()
        torch.cuda.synchronize(self.dev)
        for s in range(steps):
            flush.fill_(s & 0xff)
            e = ev[s]
            e[0].record(self.stream)
            self.graph()
            e[1].record(self.stream)
            self.build_plan()
            e[2].record(self.stream)
            self.couple()
            e[3].record(self.stream)
            self.attend()
            e[4].record(self.stream)
        torch.cuda.synchronize(self.dev)
        if barrier is not None:
            barrier()
        mean = lambda a, b: sum(e[a].elapsed_time(e[b]) for e in ev) / steps
        return {"graph": mean(0, 1), "plan": mean(1, 2), "eaas": mean(2, 3),
                "attn": mean(3, 4), "step": mean(0, 4)}


def roofline(wl: synth.Workload, edges: int, attn_ms: float, attn_name: str, peaks: dict,
             eaas_ms: float) -> dict:
    """Roofline record of the fused attention (see the module docstring)."""
    b = attention_bytes(wl, edges)
    sec = attn_ms / 1000.0
    achieved = b["compulsory"] / sec / 1e9
    traffic = l2_to_sm = None
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            recs = json.load(f)
        for rec in (recs if isinstance(recs, list) else [recs]):
            if rec.get("source_sha") == kernel_source_sha() and rec.get("workload") == wl.name:
                traffic = rec.get("dram_bytes_per_launch")
                l2_to_sm = rec.get("l2_to_sm_bytes_per_launch")
    out = {"bound": "hbm", "kernel": attn_name, "achieved": achieved, "peak": peaks["hbm_gbs"],
           "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
           "algorithmic_bytes": b["compulsory"],
           "algorithmic": "compulsory bytes: every input row read once, the output written once",
           "peak_source": peaks["source"]}
    if traffic:
        out["dram_frac"] = traffic / sec / 1e9 / peaks["hbm_gbs"]
    out["effective"] = {"bytes": b["per_edge"], "achieved": b["per_edge"] / sec / 1e9,
                        "effective_frac": b["per_edge"] / sec / 1e9 / peaks["hbm_gbs"],
                        "what": "each neighbour's key and value rows counted once per edge; "
                                "served from L2 and shared memory, not a bound"}
    if l2_to_sm:
        out["l2_to_sm"] = {"bytes": l2_to_sm, "achieved": l2_to_sm / sec / 1e9,
                           "unit": "GB/s", "source": "ncu l1tex__m_xbar2l1tex_read_bytes"}
    eb = eaas_bytes(wl)
    out["eaas_couple"] = {"bytes": eb, "achieved": eb / (eaas_ms / 1000.0) / 1e9,
                          "frac": eb / (eaas_ms / 1000.0) / 1e9 / peaks["hbm_gbs"]}
    return out


def other_workloads(names, args, dev, flush, peaks) -> dict:
    """The forward step of other workloads, timed as the main one (one rank)."""
    import torch
    out = {}
    clocks = ClockSampler(dev.index or 0)
    time.sleep(0.3)
    for name in names:
        wl = synth.WORKLOADS[name]
        data = synth.make(wl)
        fs = ForwardStep(wl, data, dev, args.attention)
        t = fs.timed(args.extra_steps, 3, flush)
        edges = int(fs.cnt.sum().item())
        # the backward pass of this workload (dL/dh, dL/dq, dL/dk, dL/dr)
        gen = torch.Generator(device="cpu").manual_seed(4321)
        G = torch.randn((wl.n, wl.D, wl.C), generator=gen, dtype=torch.float32).to(dev)
        bws_t = torch.empty(max(fs.egat.egat_backward_workspace_bytes(fs.shape), 16),
                            dtype=torch.uint8, device=dev)
        grads = [torch.empty((wl.n, wl.D, wl.C), dtype=torch.float32, device=dev),
                 torch.empty((wl.n, wl.H, wl.dk), dtype=torch.float32, device=dev),
                 torch.empty((wl.n, wl.H, wl.dk), dtype=torch.float32, device=dev),
                 torch.empty((wl.n, 3), dtype=torch.float32, device=dev)]

        def bwd():
            import ctypes
            rc = fs.lib.egat_backward(ctypes.byref(fs.cshape), fs.h.data_ptr(), fs.pos.data_ptr(),
                                      fs.q.data_ptr(), fs.k.data_ptr(), fs.nbr.data_ptr(),
                                      fs.cnt.data_ptr(), fs.order.data_ptr(), fs.w1.data_ptr(),
                                      fs.w2.data_ptr(), G.data_ptr(), bws_t.data_ptr(),
                                      bws_t.numel(), *(x.data_ptr() for x in grads), fs.sp)
            fs.egat._check("egat_backward", rc)

        bwd()
        torch.cuda.synchronize(dev)
        bms = []
        for _ in range(max(1, args.backward_steps)):
            flush.fill_(3)
            ba, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ba.record(fs.stream)
            bwd()
            bb.record(fs.stream)
            torch.cuda.synchronize(dev)
            bms.append(ba.elapsed_time(bb))
        del G, bws_t, grads
        out[name] = {"atoms_per_s": wl.n / (t["step"] / 1000.0),
                     "edges_per_s": edges / (t["step"] / 1000.0), "ms_per_step": t["step"],
                     "edges": edges,
                     "kernel_ms": {"build_graph": t["graph"], "attention_plan": t["plan"],
                                   "eaas_couple": t["eaas"], fs.attn_name: t["attn"]},
                     "roofline": roofline(wl, edges, t["attn"], fs.attn_name, peaks, t["eaas"]),
                     "backward_ms": sum(bms) / len(bms),
                     "gpu_launches": fs.launches * args.extra_steps}
        del fs
        torch.cuda.empty_cache()
    clk = clocks.stop()
    for v in out.values():
        v["clocks"] = clk
    return out


def run_decomposed(args, wl: synth.Workload):
    """One system split across the ranks by space: each rank couples its own
    atoms, exchanges the boundary atoms' h' and k rows (NCCL all-to-all, also
    at one rank), builds the attention plan over its local arrays and runs the
    fused attention for its own atoms (halo.forward_rank).  The graph and the
    halo plan are built once, outside the timed region; every rank holds the
    replicated inputs and reads only its own rows.  value = the system's atoms
    per step over the slowest rank's step time (strong scaling: the total work
    is fixed)."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from equivariant_graph_attention_b200 import egat, halo

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    if ws == 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29512")
        os.environ.setdefault("RANK", "0")
        os.environ.setdefault("WORLD_SIZE", "1")
    dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    data = synth.make(wl)                                   # one shared system
    fs = ForwardStep(wl, data, dev, args.attention)
    fs.graph()
    torch.cuda.synchronize(dev)
    nbr, cnt, order = fs.nbr.cpu().numpy(), fs.cnt.cpu().numpy(), fs.order.cpu().numpy()
    plan = halo.build_plan(nbr, cnt, order, ws, rank)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        return halo.forward_rank(plan, fs.shape, fs.h, fs.pos, fs.q, fs.k, fs.w1, fs.w2)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    clocks = ClockSampler(local)
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize(dev)
    for s in range(args.steps):
        flush.fill_(s & 0xff)
        ev[s][0].record(stream)
        step()
        ev[s][1].record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    t_step = max_over_ranks(ms, dev)

    # end to end: every step copies this rank's rows of h, q, k (pinned host
    # memory, prepared once) and the replicated positions in, runs the
    # decomposed forward and copies this rank's output rows out
    own = plan.owned
    host = {nm: torch.from_numpy(np.ascontiguousarray(data[nm][own])).to(dtype=fs.st).pin_memory()
            for nm in ("h", "q", "k")}
    host["pos"] = torch.from_numpy(np.ascontiguousarray(data["pos"])).pin_memory()
    devb = {nm: torch.empty(t.shape, dtype=t.dtype, device=dev) for nm, t in host.items()}
    out_host = torch.empty((plan.n_owned, wl.D, wl.C), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()

    def e2e_step():
        for nm, t in host.items():
            devb[nm].copy_(t, non_blocking=True)
        o = halo.forward_rank(plan, fs.shape, devb["h"], devb["pos"], devb["q"], devb["k"], fs.w1,
                              fs.w2, own_rows=True)
        out_host.copy_(o, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    eb.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(ea.elapsed_time(eb) / args.e2e_steps, dev)
    ref_out = halo.forward_rank(plan, fs.shape, fs.h, fs.pos, fs.q, fs.k, fs.w1, fs.w2)
    torch.cuda.synchronize(dev)
    e2e_ok = bool(torch.equal(out_host.to(dev), ref_out))
    edges = int(cnt.sum())
    row_bytes = wl.D * wl.C * storage_bytes(wl) + wl.H * wl.dk * storage_bytes(wl)
    halo_max = max_over_ranks(plan.halo.size, dev)
    status = fs.lib.egat_take_device_status(stream.cuda_stream)
    if status != egat.EGAT_OK:
        raise RuntimeError(f"device status after the runs: {fs.lib.egat_strerror(status).decode()}")
    if rank == 0:
        line = {
            "metric": METRIC, "value": wl.n / (t_step / 1000.0), "unit": "atoms/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": config_of(wl, edges, ws, decompose=True),
            "edges_per_s": edges / (t_step / 1000.0),
            "e2e": {"value": wl.n / (e2e_ms / 1000.0), "unit": "atoms/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "what": "each rank: its rows of h, q, k and the positions in, its output rows "
                            "out, every step", "matches_device_result": e2e_ok},
            "gpu_launches": (DECOMP_LAUNCHES + launches_plan(wl.lmax)) * args.steps,
            "roofline": None,
            "roofline_note": "per-kernel rooflines are reported by the single-system line",
            "decomposition": {"owned_per_rank": int(plan.n_owned), "halo_atoms_max": int(halo_max),
                              "exchange_bytes_max": int(halo_max) * row_bytes,
                              "step": "couple own atoms, exchange h' and k halo rows (NCCL "
                                      "all-to-all), attention plan over local arrays, fused "
                                      "attention of own atoms; graph and halo plan built once, "
                                      "untimed"},
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=synth.WORKLOAD_ORDER)
    ap.add_argument("--impl", default="egat", choices=["egat", "reference"])
    ap.add_argument("--ref-targets", type=int, default=4,
                    help="reference arm: random targets per oracle worker and step")
    ap.add_argument("--cpu-targets", type=int, default=8,
                    help="cpu_baseline: random targets per oracle worker")
    ap.add_argument("--cpu-workers", type=int, default=0,
                    help="oracle worker processes (0: the host's cores, at most 32)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--backward-steps", type=int, default=5,
                    help="timed calls of egat_backward reported beside the forward (0: skip)")
    ap.add_argument("--extra-steps", type=int, default=10,
                    help="timed steps of each other workload (0: skip them)")
    ap.add_argument("--attention", default="auto", choices=["auto", "tiled", "per-target"],
                    help="steps 3+4 kernel: tensor-core tiles when the shape allows (auto), or "
                         "the per-target kernel")
    ap.add_argument("--decompose", action="store_true",
                    help="split one system across the ranks by space (halo exchange); the "
                         "default when more than one rank runs")
    ap.add_argument("--replicas", action="store_true",
                    help="with more than one rank: independent systems, one per rank")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.decompose and args.replicas:
        ap.error("--decompose and --replicas exclude each other")
    ws0, _, _ = dist_env()
    args.decompose = args.decompose or (ws0 > 1 and not args.replicas)
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
        return
    if args.decompose:
        run_decomposed(args, wl)
        return

    ws, rank, local = dist_env()
    data = synth.make(wl, seed=rank)
    pool = None
    if rank == 0 and not args.no_cpu_baseline:
        # forked before the first CUDA call of this process
        pool = OraclePool(wl, data, args.cpu_workers or oracle_workers_default())

    import ctypes
    import torch
    import torch.distributed as dist
    from equivariant_graph_attention_b200 import egat

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    barrier = dist.barrier if ws > 1 else None
    egat.load_library()

    fs = ForwardStep(wl, data, dev, args.attention)
    lib, shape, cshape, st = fs.lib, fs.shape, fs.cshape, fs.st
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    fs.run()
    torch.cuda.synchronize(dev)
    edges = int(fs.cnt.sum().item())
    clocks = ClockSampler(local)
    time.sleep(0.3)
    t = fs.timed(args.steps, args.warmup, flush, barrier)
    clk = clocks.stop()
    total_ms = t["step"] * args.steps
    # every rank ran its own system: atoms and edges add up over ranks, the
    # job's time is the slowest rank's
    value = job_rate(wl.n * args.steps, total_ms, dev)
    edges_per_s = job_rate(edges * args.steps, total_ms, dev)
    t_step = max_over_ranks(total_ms, dev) / args.steps
    out = fs.out

    # ------------------------------------------------------------------ e2e
    # the same step through the public C ABI (egat_build_graph + egat_forward)
    # with the inputs in pinned host memory: every step copies its inputs in,
    # builds the graph, runs the fused forward and copies ^h out.  Steps are
    # independent systems, so they are pipelined the way a caller would: a
    # copy-in stream, a compute stream and a copy-out stream with double-
    # buffered inputs and outputs, ordered by events (step i's compute waits
    # for its copy-in and for the copy-out that last used its output buffer).
    names = ("h", "q", "k", "pos", "pos_q", "w1", "w2")
    dtypes = {nm: (st if nm in ("h", "q", "k") else (torch.int32 if nm == "pos_q" else torch.float32))
              for nm in names}
    NB = 2
    host_in = [{nm: torch.from_numpy(np.ascontiguousarray(data[nm])).to(dtype=dtypes[nm]).pin_memory()
                for nm in names} for _ in range(NB)]
    dev_in = [{nm: torch.empty(host_in[0][nm].shape, dtype=dtypes[nm], device=dev) for nm in names}
              for _ in range(NB)]
    dev_out = [torch.empty_like(out) for _ in range(NB)]
    host_out = [torch.empty(out.shape, dtype=torch.float32).pin_memory() for _ in range(NB)]
    fws = torch.empty(egat.egat_forward_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    h2d = sum(x.numel() * x.element_size() for x in host_in[0].values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    s_in, s_c, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(NB)]
    ev_c = [torch.cuda.Event() for _ in range(NB)]
    ev_out = [torch.cuda.Event() for _ in range(NB)]
    nbr, cnt, order, ovf, gws = fs.nbr, fs.cnt, fs.order, fs.ovf, fs.gws

    def e2e_step(i):
        b = i % NB
        di = dev_in[b]
        s_in.wait_event(ev_c[b])               # step i - NB no longer reads these inputs
        with torch.cuda.stream(s_in):
            for nm in names:
                di[nm].copy_(host_in[b][nm], non_blocking=True)
        ev_in[b].record(s_in)
        s_c.wait_event(ev_in[b])
        s_c.wait_event(ev_out[b])              # step i - NB's result has been copied out
        cs_ = s_c.cuda_stream
        rc = lib.egat_build_graph(di["pos_q"].data_ptr(), wl.n, wl.cutoff_q, wl.K, 0,
                                  nbr.data_ptr(), cnt.data_ptr(), 0, order.data_ptr(),
                                  ovf.data_ptr(), gws.data_ptr(), gws.numel(), cs_)
        egat._check("egat_build_graph", rc)
        rc = lib.egat_forward(ctypes.byref(cshape), di["h"].data_ptr(), di["pos"].data_ptr(),
                              di["q"].data_ptr(), di["k"].data_ptr(), nbr.data_ptr(),
                              cnt.data_ptr(), order.data_ptr(), di["w1"].data_ptr(),
                              di["w2"].data_ptr(), fws.data_ptr(), fws.numel(),
                              dev_out[b].data_ptr(), cs_)
        egat._check("egat_forward", rc)
        ev_c[b].record(s_c)
        s_out.wait_event(ev_c[b])
        with torch.cuda.stream(s_out):
            host_out[b].copy_(dev_out[b], non_blocking=True)
        ev_out[b].record(s_out)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if ws > 1:
        dist.barrier()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(s_in)
    for i in range(args.e2e_steps):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_c)
    eb.record(s_out)
    torch.cuda.synchronize(dev)
    e2e_ms = ea.elapsed_time(eb)
    e2e_value = job_rate(wl.n * args.e2e_steps, e2e_ms, dev)
    e2e_ms = max_over_ranks(e2e_ms, dev)
    e2e_ok = bool(torch.equal(host_out[0].to(dev), out))   # pipelined result == device-timed result
    # ------------------------------------------------------------------ backward
    # gradients of <G, ^h> for a seeded upstream gradient G (egat_backward:
    # dL/dh, dL/dq, dL/dk, dL/dr; the attention is recomputed, in-lists built inside),
    # each call after an L2 flush, timed with events on the launching stream
    bwd = None
    if args.backward_steps > 0:
        gen = torch.Generator(device="cpu").manual_seed(1234 + rank)
        G = torch.randn((wl.n, wl.D, wl.C), generator=gen, dtype=torch.float32).to(dev)
        bws_t = torch.empty(max(egat.egat_backward_workspace_bytes(shape), 16), dtype=torch.uint8,
                            device=dev)
        dh_t = torch.empty((wl.n, wl.D, wl.C), dtype=torch.float32, device=dev)
        dq_t = torch.empty((wl.n, wl.H, wl.dk), dtype=torch.float32, device=dev)
        dk_t = torch.empty((wl.n, wl.H, wl.dk), dtype=torch.float32, device=dev)
        dr_t = torch.empty((wl.n, 3), dtype=torch.float32, device=dev)

        def backward_call(with_positions=True):
            rc = lib.egat_backward(ctypes.byref(cshape), fs.h.data_ptr(), fs.pos.data_ptr(),
                                   fs.q.data_ptr(), fs.k.data_ptr(), nbr.data_ptr(),
                                   cnt.data_ptr(), order.data_ptr(), fs.w1.data_ptr(),
                                   fs.w2.data_ptr(), G.data_ptr(), bws_t.data_ptr(),
                                   bws_t.numel(), dh_t.data_ptr(), dq_t.data_ptr(),
                                   dk_t.data_ptr(), dr_t.data_ptr() if with_positions else None,
                                   fs.sp)
            egat._check("egat_backward", rc)

        def timed_calls(with_positions):
            ms = []
            for _ in range(args.backward_steps):
                flush.fill_(3)
                ba, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                ba.record(fs.stream)
                backward_call(with_positions)
                bb.record(fs.stream)
                torch.cuda.synchronize(dev)
                ms.append(ba.elapsed_time(bb))
            return sum(ms) / len(ms)

        fs.graph()                                        # this system's neighbour lists
        backward_call()                                   # warm-up
        torch.cuda.synchronize(dev)
        t_bwd = timed_calls(True)
        # the same call without dL/dr (training on energies: no forces wanted)
        t_nodr = timed_calls(False)
        bwd = {"ms": max_over_ranks(t_bwd, dev),
               "ms_without_positions": max_over_ranks(t_nodr, dev),
               "atoms_per_s": job_rate(wl.n, t_bwd, dev),
               "edges_per_s": job_rate(edges, t_bwd, dev),
               "what": "dL/dh, dL/dq, dL/dk, dL/dr of <G, ^h> (egat_backward), L2 flushed "
                       "before each call; ms_without_positions: the same call without dL/dr"}

    peaks = measured_peaks()

    # ------------------------------------------------------------------ next rows
    # the invariant query/key projection (tensor cores on this shape) and the
    # edge-centric eSCN convolution on the same system and graph, each call
    # after an L2 flush, timed with events on the launching stream
    def timed_calls(fn, k=args.steps):
        ms = []
        for _ in range(k):
            flush.fill_(5)
            ba, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ba.record(fs.stream)
            fn()
            bb.record(fs.stream)
            torch.cuda.synchronize(dev)
            ms.append(ba.elapsed_time(bb))
        return sum(ms) / len(ms)

    wts = synth.projection_weights(wl, seed=rank)
    wq, wk = (torch.from_numpy(wts[x]).to(dev) for x in ("wq", "wk"))
    qo, ko = torch.empty_like(fs.q), torch.empty_like(fs.k)

    def projection_call():
        rc = lib.egat_qk_projection(ctypes.byref(cshape), fs.h.data_ptr(), wq.data_ptr(),
                                    wk.data_ptr(), qo.data_ptr(), ko.data_ptr(), fs.sp)
        egat._check("egat_qk_projection", rc)

    projection_call()
    t_proj = timed_calls(projection_call)
    s_b = storage_bytes(wl)
    proj_bytes = wl.n * (wl.C + 2 * wl.H * wl.dk) * s_b
    proj = {"ms": max_over_ranks(t_proj, dev), "bytes": proj_bytes,
            "achieved_gbs": proj_bytes / (t_proj / 1000.0) / 1e9,
            "frac": proj_bytes / (t_proj / 1000.0) / 1e9 / peaks["hbm_gbs"],
            "flops": 2 * 2 * wl.n * wl.C * wl.H * wl.dk,
            "tensor_cores": bool(wl.dtype == "bf16" and wl.C == 128 and wl.H * wl.dk == 256),
            "what": "q, k from the degree-0 channels (egat_qk_projection); bytes: degree-0 "
                    "slices in, q and k out"}
    mmax = wl.lmax
    ew = torch.from_numpy(synth.escn_weights(wl, mmax, seed=rank)).to(dev)
    eo = torch.empty_like(fs.out)
    fs.graph()

    def escn_call():
        rc = lib.egat_escn_conv(ctypes.byref(cshape), mmax, fs.h.data_ptr(), fs.pos.data_ptr(),
                                nbr.data_ptr(), cnt.data_ptr(), order.data_ptr(), ew.data_ptr(),
                                eo.data_ptr(), fs.sp)
        egat._check("egat_escn_conv", rc)

    escn_call()
    t_escn = timed_calls(escn_call, max(3, args.steps // 4))
    escn = {"ms": max_over_ranks(t_escn, dev), "mmax": mmax,
            "edges_per_s": job_rate(edges, t_escn, dev),
            "atoms_per_s": job_rate(wl.n, t_escn, dev),
            "vs_forward_step": t_escn / t_step,
            "what": "edge-centric eSCN convolution (egat_escn_conv: per edge rotate into the "
                    "edge frame, SO(2) linear layer, rotate back, sum) on the same graph; "
                    "the comparison workload of the node-centric path"}
    extra = None
    if rank == 0 and args.extra_steps > 0:
        extra = other_workloads([n for n in EXTRA_WORKLOADS if n != wl.name], args, dev, flush,
                                peaks)

    # no bounded device wait may have given up in any of the runs above
    status = lib.egat_take_device_status(torch.cuda.current_stream(dev).cuda_stream)
    if status != egat.EGAT_OK:
        raise RuntimeError(f"device status after the runs: {lib.egat_strerror(status).decode()}")

    cpu = None
    if pool is not None:
        pool.rate(1, seed=123)                    # warm the workers (imports, caches)
        v_all, wall, n_all = pool.rate(args.cpu_targets, seed=7)
        pool.close()
        v_one, secs_one = single_thread_rate(max(4, args.cpu_targets), seed=8)
        cpu = {"value": v_all, "unit": "atoms/s", "cores": pool.workers, "kind": "oracle",
               "sample": f"{n_all} random target atoms of the {wl.n}-atom system over "
                         f"{pool.workers} worker processes, one thread each (brute-force "
                         f"neighbour rows, dense source coupling of their neighbours, "
                         f"two-pass attention, dense target coupling), {wall:.1f} s wall",
               "single_thread": {"value": v_one, "unit": "atoms/s", "cores": 1,
                                 "sample": f"{max(4, args.cpu_targets)} targets, "
                                           f"{secs_one:.1f} s"}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "atoms/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": config_of(wl, edges, ws),
            "edges_per_s": edges_per_s,
            "kernel_ms": {"build_graph": t["graph"], "attention_plan": t["plan"],
                          "eaas_couple": t["eaas"], fs.attn_name: t["attn"]},
            "roofline": roofline(wl, edges, t["attn"], fs.attn_name, peaks, t["eaas"]),
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "atoms/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.e2e_steps,
                    "pipelined": "copy-in / compute / copy-out streams, 2 buffers",
                    "matches_device_result": e2e_ok},
            "backward": bwd,
            "qk_projection": proj,
            "escn_conv": escn,
            "other_workloads": extra,
            "gpu_launches": fs.launches * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
