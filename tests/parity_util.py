"""Helpers shared by the GPU parity tests: device inputs and the error metric.

Error metric (the pages give a tolerance but no metric).  The plainest reading
of "max relative error" that is well posed near zero: for every atom i and
degree l, the irrep feature block v = out[i, l^2:(l+1)^2, :] (all components
m and all C channels) gives e = ||v_gpu - v_ref|| / ||v_ref|| (Frobenius
norms), and the reported error is the maximum over (i, l).  A block whose
reference is exactly zero (an atom without neighbours) must be zero on the GPU
too.  The norm is rotation invariant, so the metric does not depend on the
frame.  Bars: 1e-4 for float32 storage, 2e-2 for bf16 storage with float32
accumulation.
"""
from __future__ import annotations

import numpy as np
import torch

from equivariant_graph_attention_b200 import synth

TOL = {"f32": 1e-4, "bf16": 2e-2}


def block_rel_error(gpu: np.ndarray, ref: np.ndarray, lmax: int) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape
    worst = 0.0
    for l in range(lmax + 1):
        g = gpu[:, l * l:(l + 1) ** 2, :].reshape(gpu.shape[0], -1)
        r = ref[:, l * l:(l + 1) ** 2, :].reshape(ref.shape[0], -1)
        nr = np.linalg.norm(r, axis=1)
        ne = np.linalg.norm(g - r, axis=1)
        zero = nr == 0.0
        if np.any(zero):
            assert np.all(ne[zero] == 0.0), "nonzero output where the reference is exactly zero"
        if np.any(~zero):
            worst = max(worst, float(np.max(ne[~zero] / nr[~zero])))
    return worst


def device_inputs(wl: synth.Workload, data: dict, device="cuda") -> dict:
    """Inputs on the device in the storage type the workload names."""
    st = torch.bfloat16 if wl.dtype == "bf16" else torch.float32

    def f(x, dt):
        return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dt)

    return {"h": f(data["h"], st), "q": f(data["q"], st), "k": f(data["k"], st),
            "pos": f(data["pos"], torch.float32), "pos_q": f(data["pos_q"], torch.int32),
            "w1": f(data["w1"], torch.float32), "w2": f(data["w2"], torch.float32)}


def shape_of(wl: synth.Workload, n=None, mode="padded", n_edges=0):
    from equivariant_graph_attention_b200.egat import Shape
    return Shape(n=wl.n if n is None else n, lmax=wl.lmax, C=wl.C, H=wl.H, dk=wl.dk, K=wl.K,
                 dtype=wl.dtype, graph_mode=mode, n_edges=n_edges)


def sample_targets(wl: synth.Workload, full_degree: np.ndarray, count: int = 40, seed: int = 5):
    """A deterministic sample of target atoms: random ones plus the highest
    degree atoms (truncated rows) and the last atom (ragged tail)."""
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(wl.n, size=min(count, wl.n), replace=False).tolist())
    pick |= set(np.argsort(-full_degree, kind="stable")[:8].tolist())
    pick.add(wl.n - 1)
    return sorted(pick)
