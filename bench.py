"""Benchmark of the fused EAAS + on-the-fly equivariant attention hot path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole hot path over one synthetic system:
radius graph (egat_build_graph) -> attention plan (egat_build_attention_plan,
tensor-core shapes) -> EAAS source coupling (egat_eaas_couple_planned with the
plan's rotations on tensor-core shapes, egat_eaas_couple otherwise) -> on-the-fly
attention with the target coupling fused (egat_otf_attention_tiled on
tensor-core shapes, egat_otf_attention_coupled otherwise).
The default workload is the 32,768-atom, K = 256, ℓmax = 2, bf16-storage
system.  Inputs are resident in HBM when the timed region starts; L2 is
flushed (a 256 MiB write) before every timed step, outside the step's events.

Prints ONE JSON line (rank 0).  ``value`` is atoms/s over all ranks; edges/s,
per-kernel times, the roofline of the dominant kernel, the CPU oracle baseline
and an end-to-end figure through host buffers ride along.

Multi-GPU (torchrun): every rank runs its own independent system (same shape,
seeded by rank) — the units are independent problems, so there is no
data-path collective; timing is the max over ranks.  ``--impl reference``
times the CPU oracle on the same workload (rank 0 only).
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
FLUSH_BYTES = 256 << 20
#: kernels this library launches per step: graph (assign, scan x3, scatter,
#: rank, fill, truncated-row fix) + attention plan (tensor-core shapes: unions
#: and masks, tile records) + source coupling + fused attention
LAUNCHES_GRAPH = 8
LAUNCHES_PLAN = 2
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attention_traffic.json")
KERNEL_SOURCES = ["equivariant_graph_attention_b200/csrc/attention.cu",
                  "equivariant_graph_attention_b200/csrc/attention_tc.cu",
                  "equivariant_graph_attention_b200/csrc/plan.cu",
                  "equivariant_graph_attention_b200/csrc/egat_device.cuh",
                  "equivariant_graph_attention_b200/csrc/egat_async.cuh"]


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


def algorithmic_bytes(wl: synth.Workload, cnt: np.ndarray) -> dict:
    """Bytes the method itself moves, per kernel (each counted once).

    attention (steps 3+4): per target the padded list row (K*4) and count (4),
    q_i, r_i (12) and the float32 output row; per real edge the neighbour's
    key and value rows.  source coupling (step 2): read h, write h', r.
    """
    s = 2 if wl.dtype == "bf16" else 4
    N, D, C, H, dk, K = wl.n, wl.D, wl.C, wl.H, wl.dk, wl.K
    E = int(cnt.sum())
    attn = N * (K * 4 + 4 + H * dk * s + 12 + D * C * 4) + E * (D * C * s + H * dk * s)
    eaas = N * (2 * D * C * s + 12)
    return {"attention": attn, "eaas": eaas, "edges": E}


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
def oracle_sample(wl: synth.Workload, data: dict, n_targets: int, seed: int = 0) -> float:
    """Seconds the CPU oracle takes for the forward pass of ``n_targets``
    sampled targets (their brute-force neighbour rows, the source coupling of
    the atoms they need, two-pass attention and target coupling)."""
    from oracle.attention import forward
    from oracle.graph import radius_graph

    rows = np.random.default_rng(seed).choice(wl.n, size=n_targets, replace=False)
    t0 = time.perf_counter()
    lists, _ = radius_graph(data["pos_q"], wl.cutoff_q, K=wl.K, rows=rows)
    forward(data["h"], data["pos"], data["q"], data["k"], data["w1"], data["w2"], wl.lmax,
            lists, targets=rows)
    return time.perf_counter() - t0


def cpu_threads_used() -> int:
    # numpy einsum and the integer neighbour search run on one thread
    return 1


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
    per_step_targets = args.ref_targets
    for _ in range(args.warmup):
        oracle_sample(wl, data, max(1, per_step_targets // 4), seed=99)
    secs = [oracle_sample(wl, data, per_step_targets, seed=s) for s in range(args.steps)]
    total = float(sum(secs))
    value = per_step_targets * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "atoms/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "atoms": wl.n, "K": wl.K, "lmax": wl.lmax, "C": wl.C,
                   "H": wl.H, "dk": wl.dk, "cutoff_A": wl.cutoff},
        "cpu_baseline": {"value": value, "unit": "atoms/s", "cores": cpu_threads_used(),
                         "kind": "oracle",
                         "sample": f"{per_step_targets} random target atoms per step of the "
                                   f"{wl.n}-atom system (neighbour rows, source coupling of "
                                   f"their neighbours, attention, target coupling)"},
        "e2e": {"value": value, "unit": "atoms/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=synth.WORKLOAD_ORDER)
    ap.add_argument("--impl", default="egat", choices=["egat", "reference"])
    ap.add_argument("--ref-targets", type=int, default=64)
    ap.add_argument("--cpu-targets", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--backward-steps", type=int, default=5,
                    help="timed calls of egat_backward reported beside the forward (0: skip)")
    ap.add_argument("--attention", default="auto", choices=["auto", "tiled", "per-target"],
                    help="steps 3+4 kernel: tensor-core tiles when the shape allows (auto), or "
                         "the per-target kernel")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
        return

    import torch
    import torch.distributed as dist
    from equivariant_graph_attention_b200 import egat

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    egat.load_library()

    data = synth.make(wl, seed=rank)
    st = torch.bfloat16 if wl.dtype == "bf16" else torch.float32

    def td(x, dt):
        return torch.from_numpy(np.ascontiguousarray(x)).to(dev, dtype=dt)

    h, q, k = td(data["h"], st), td(data["q"], st), td(data["k"], st)
    pos, pos_q = td(data["pos"], torch.float32), td(data["pos_q"], torch.int32)
    w1, w2 = td(data["w1"], torch.float32), td(data["w2"], torch.float32)
    shape = egat.Shape(n=wl.n, lmax=wl.lmax, C=wl.C, H=wl.H, dk=wl.dk, K=wl.K, dtype=wl.dtype)
    gws = torch.empty(egat.egat_graph_workspace_bytes(wl.n), dtype=torch.uint8, device=dev)
    nbr = torch.empty((wl.n, wl.K), dtype=torch.int32, device=dev)
    cnt = torch.empty(wl.n, dtype=torch.int32, device=dev)
    order = torch.empty(wl.n, dtype=torch.int32, device=dev)
    ovf = torch.zeros(1, dtype=torch.int32, device=dev)
    hp = torch.empty((wl.n, wl.D, wl.C), dtype=st, device=dev)
    out = torch.empty((wl.n, wl.D, wl.C), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    lib = egat.load_library()
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    cshape = shape.c()
    import ctypes

    def graph():
        rc = lib.egat_build_graph(pos_q.data_ptr(), wl.n, wl.cutoff_q, wl.K, 0, nbr.data_ptr(),
                                  cnt.data_ptr(), 0, order.data_ptr(), ovf.data_ptr(),
                                  gws.data_ptr(), gws.numel(), sp)
        egat._check("egat_build_graph", rc)


    plan_sz = ctypes.c_size_t(0)
    tiled = (lib.egat_attention_plan_bytes(ctypes.byref(cshape), ctypes.byref(plan_sz)) == 0
             and wl.dtype == "bf16" and wl.C == 128 and wl.H == 16 and wl.dk == 16
             and args.attention != "per-target")
    if args.attention == "tiled" and not tiled:
        raise SystemExit("the tensor-core attention path does not support this workload")
    plan = torch.empty(max(plan_sz.value, 16), dtype=torch.uint8, device=dev)

    def build_plan():
        if tiled:
            rc = lib.egat_build_attention_plan(ctypes.byref(cshape), nbr.data_ptr(),
                                               cnt.data_ptr(), order.data_ptr(), pos.data_ptr(),
                                               plan.data_ptr(), plan.numel(), sp)
            egat._check("egat_build_attention_plan", rc)

    def couple():
        if tiled:   # rotations from the plan's tile records
            rc = lib.egat_eaas_couple_planned(ctypes.byref(cshape), h.data_ptr(), plan.data_ptr(),
                                              w1.data_ptr(), hp.data_ptr(), sp)
            egat._check("egat_eaas_couple_planned", rc)
        else:
            rc = lib.egat_eaas_couple(ctypes.byref(cshape), h.data_ptr(), pos.data_ptr(),
                                      w1.data_ptr(), hp.data_ptr(), sp)
            egat._check("egat_eaas_couple", rc)

    def attend():
        if tiled:
            rc = lib.egat_otf_attention_tiled(ctypes.byref(cshape), q.data_ptr(), k.data_ptr(),
                                              hp.data_ptr(), plan.data_ptr(), w2.data_ptr(),
                                              out.data_ptr(), 1, sp)
            egat._check("egat_otf_attention_tiled", rc)
        else:
            rc = lib.egat_otf_attention_coupled(ctypes.byref(cshape), q.data_ptr(), k.data_ptr(),
                                                hp.data_ptr(), nbr.data_ptr(), cnt.data_ptr(),
                                                order.data_ptr(), pos.data_ptr(), w2.data_ptr(),
                                                out.data_ptr(), sp)
            egat._check("egat_otf_attention_coupled", rc)
    attn_name = "otf_attention_tiled" if tiled else "otf_attention_coupled"
    launches_per_step = LAUNCHES_GRAPH + (LAUNCHES_PLAN if tiled else 0) + 2

    for _ in range(args.warmup):
        flush.fill_(1)
        graph()
        build_plan()
        couple()
        attend()
    torch.cuda.synchronize(dev)
    cnt_host = cnt.cpu().numpy()
    alg = algorithmic_bytes(wl, cnt_host)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for s in range(args.steps):
        flush.fill_(s & 0xff)
        e = ev[s]
        e[0].record(stream)
        graph()
        e[1].record(stream)
        build_plan()
        e[2].record(stream)
        couple()
        e[3].record(stream)
        attend()
        e[4].record(stream)
    torch.cuda.synchronize(dev)
    if ws > 1:
        dist.barrier()
    clk = clocks.stop()

    t_graph = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    t_plan = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    t_eaas = sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps
    t_attn = sum(e[3].elapsed_time(e[4]) for e in ev) / args.steps
    t_step = sum(e[0].elapsed_time(e[4]) for e in ev) / args.steps      # ms
    total_ms = t_step * args.steps
    # every rank ran its own system: atoms and edges add up over ranks, the
    # job's time is the slowest rank's
    value = job_rate(wl.n * args.steps, total_ms, dev)
    edges_per_s = job_rate(alg["edges"] * args.steps, total_ms, dev)
    t_step = max_over_ranks(total_ms, dev) / args.steps

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
    h2d = sum(t.numel() * t.element_size() for t in host_in[0].values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    s_in, s_c, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(NB)]
    ev_c = [torch.cuda.Event() for _ in range(NB)]
    ev_out = [torch.cuda.Event() for _ in range(NB)]

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

        def backward_call():
            rc = lib.egat_backward(ctypes.byref(cshape), h.data_ptr(), pos.data_ptr(), q.data_ptr(),
                                   k.data_ptr(), nbr.data_ptr(), cnt.data_ptr(), order.data_ptr(),
                                   w1.data_ptr(), w2.data_ptr(), G.data_ptr(), bws_t.data_ptr(),
                                   bws_t.numel(),
                                   dh_t.data_ptr(), dq_t.data_ptr(), dk_t.data_ptr(),
                                   dr_t.data_ptr(), sp)
            egat._check("egat_backward", rc)

        graph()                                           # this system's neighbour lists
        backward_call()                                   # warm-up
        torch.cuda.synchronize(dev)
        bms = []
        for _ in range(args.backward_steps):
            flush.fill_(3)
            ba, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ba.record(torch.cuda.current_stream(dev))
            backward_call()
            bb.record(torch.cuda.current_stream(dev))
            torch.cuda.synchronize(dev)
            bms.append(ba.elapsed_time(bb))
        t_bwd = sum(bms) / len(bms)
        # the same call without dL/dr (training on energies: no forces wanted)
        nms = []
        for _ in range(args.backward_steps):
            flush.fill_(3)
            ba, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ba.record(torch.cuda.current_stream(dev))
            rc = lib.egat_backward(ctypes.byref(cshape), h.data_ptr(), pos.data_ptr(), q.data_ptr(),
                                   k.data_ptr(), nbr.data_ptr(), cnt.data_ptr(), order.data_ptr(),
                                   w1.data_ptr(), w2.data_ptr(), G.data_ptr(), bws_t.data_ptr(),
                                   bws_t.numel(), dh_t.data_ptr(), dq_t.data_ptr(), dk_t.data_ptr(),
                                   None, sp)
            egat._check("egat_backward", rc)
            bb.record(torch.cuda.current_stream(dev))
            torch.cuda.synchronize(dev)
            nms.append(ba.elapsed_time(bb))
        t_nodr = sum(nms) / len(nms)
        bwd = {"ms": max_over_ranks(t_bwd, dev),
               "ms_without_positions": max_over_ranks(t_nodr, dev),
               "atoms_per_s": job_rate(wl.n, t_bwd, dev),
               "edges_per_s": job_rate(alg["edges"], t_bwd, dev),
               "what": "dL/dh, dL/dq, dL/dk, dL/dr of <G, ^h> (egat_backward), L2 flushed "
                       "before each call; ms_without_positions: the same call without dL/dr"}

    # no bounded device wait may have given up in any of the runs above
    status = lib.egat_take_device_status(torch.cuda.current_stream(dev).cuda_stream)
    if status != egat.EGAT_OK:
        raise RuntimeError(f"device status after the runs: {lib.egat_strerror(status).decode()}")

    # ------------------------------------------------------------------ roofline
    peaks = measured_peaks()
    achieved = alg["attention"] / (t_attn / 1000.0) / 1e9      # GB/s
    traffic = None
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        if rec.get("source_sha") == kernel_source_sha() and rec.get("workload") == wl.name:
            traffic = rec.get("dram_bytes_per_launch")

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        oracle_sample(wl, data, 4, seed=123)        # warm caches / imports
        secs = oracle_sample(wl, data, args.cpu_targets, seed=7)
        cpu = {"value": args.cpu_targets / secs, "unit": "atoms/s", "cores": cpu_threads_used(),
               "kind": "oracle",
               "sample": f"{args.cpu_targets} random target atoms of the {wl.n}-atom system "
                         f"(brute-force neighbour rows, dense source coupling of their "
                         f"neighbours, two-pass attention, dense target coupling), "
                         f"{secs:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "atoms/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": {"workload": wl.name, "atoms": wl.n, "edges": alg["edges"], "K": wl.K,
                       "lmax": wl.lmax, "C": wl.C, "H": wl.H, "dk": wl.dk,
                       "cutoff_A": wl.cutoff, "accumulate": "f32",
                       "l2": "flushed before every timed step (256 MiB write, untimed)",
                       "parallelism": f"{ws} independent systems (one per GPU)"},
            "edges_per_s": edges_per_s,
            "kernel_ms": {"build_graph": t_graph, "attention_plan": t_plan,
                          "eaas_couple": t_eaas, attn_name: t_attn},
            "roofline": {"bound": "hbm", "kernel": attn_name,
                         "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                         "algorithmic_bytes": alg["attention"], "peak_source": peaks["source"]},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "atoms/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.e2e_steps,
                    "pipelined": "copy-in / compute / copy-out streams, 2 buffers",
                    "matches_device_result": e2e_ok},
            "backward": bwd,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
