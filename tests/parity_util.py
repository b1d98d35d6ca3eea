"""Helpers shared by the GPU parity tests: device inputs and the error metrics.

The pages give a tolerance ("max relative error" 1e-4 for float32 storage,
2e-2 for bf16 storage with float32 accumulation) but no metric.  Two are used,
both rotation invariant:

* channel_rel_error (the primary metric): every (atom, degree l, channel c)
  irrep vector v = out[i, l^2:(l+1)^2, c] (2l+1 components) gives
  e = ||v_gpu - v_ref|| / max(||v_ref||, floor * RMS_l), with RMS_l the root
  mean square of ||v_ref|| over the atoms and channels compared at degree l;
  the error is the maximum over (i, l, c).  One wrong channel or head fails
  it: nothing averages over channels.  vec_rel_error is the same over the
  rows of a query, key or gradient array.
* block_rel_error: the same per (atom, degree) over the whole (2l+1) x C
  block, Frobenius norms; a block whose reference is exactly zero (an atom
  without neighbours) must be exactly zero on the GPU.

The floor.  A channel whose reference norm is small because its terms cancel
cannot be resolved relative to itself: the two sides differ by roundings of
the terms, not of the result.  So the floor comes from the arithmetic that
separates the two sides:

* FLOOR["bf16"] = 1e-3: identical inputs, float32 arithmetic, bf16 bar.
* FLOOR["f32"] = 128 * 2^-24 / 1e-4 (about 0.076): identical inputs, float32
  arithmetic, float32 bar: a 1e-3 floor would ask for results within 1.7
  float32 units of the RMS, and the measured differences of float32 paths
  reach 3e-7 to 3.5e-6 of the RMS at degree 0 (coupling terms of
  |r|^l-scaled size cancelling after chains of dozens of float32 operations:
  projection, softmax, aggregation, two couplings), so 128 units are allowed.
* ROUNDING_FLOOR = 2^-9 / 2e-2 (about 0.098): where one side rounds an
  intermediate that the other keeps: h' stored in bf16 between the source
  coupling and the attention (the composed bf16 forward, compared with the
  oracle that stores its own h' in bf16 as the workloads specify, where
  rounding boundaries may still fall either way), and the tf32 products of
  the tiled backward (4 tf32 units = one bf16 unit).  One bf16 unit of a
  channel of RMS size must stay within the bar.  Against the float64 oracle
  without that storage model, the bf16 rounding of h' alone puts the oracle
  itself at a per-channel error of 2.5 at the 1e-3 floor.
"""
from __future__ import annotations

import numpy as np
import torch

from equivariant_graph_attention_b200 import synth

TOL = {"f32": 1e-4, "bf16": 2e-2}
#: per-channel floors (fractions of the degree's RMS norm) where both sides read
#: identical inputs and compute in float32 / float64
FLOOR = {"f32": 128 * 2.0 ** -24 / TOL["f32"], "bf16": 1e-3}
#: per-channel floor where one side rounds an intermediate to bf16 (or tf32
#: products) that the other keeps: one bf16 unit over the bar
ROUNDING_FLOOR = 2.0 ** -9 / TOL["bf16"]
#: per-channel floor of the backward's gradients (tf32 products on bf16 shapes)
BWD_FLOOR = {"f32": FLOOR["f32"], "bf16": ROUNDING_FLOOR}


def channel_rel_error(gpu: np.ndarray, ref: np.ndarray, lmax: int, floor: float) -> float:
    """max over (atom, l, channel) of ||v_gpu - v_ref|| / max(||v_ref||, floor RMS_l)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape
    worst = 0.0
    for l in range(lmax + 1):
        r = ref[:, l * l:(l + 1) ** 2, :]
        nr = np.linalg.norm(r, axis=1)                       # [atoms, C]
        ne = np.linalg.norm(gpu[:, l * l:(l + 1) ** 2, :] - r, axis=1)
        rms = float(np.sqrt(np.mean(nr ** 2))) if nr.size else 0.0
        if rms == 0.0:
            assert np.all(ne == 0.0), "nonzero output where the reference is exactly zero"
            continue
        worst = max(worst, float(np.max(ne / np.maximum(nr, floor * rms))))
    return worst


def vec_rel_error(gpu: np.ndarray, ref: np.ndarray, floor: float) -> float:
    """The per-vector metric over the last axis (a query/key row of one head,
    a gradient row): max of ||v_gpu - v_ref|| / max(||v_ref||, floor RMS)."""
    g = np.asarray(gpu, dtype=np.float64).reshape(-1, np.shape(gpu)[-1])
    r = np.asarray(ref, dtype=np.float64).reshape(-1, np.shape(ref)[-1])
    nr = np.linalg.norm(r, axis=1)
    ne = np.linalg.norm(g - r, axis=1)
    rms = float(np.sqrt(np.mean(nr ** 2))) if nr.size else 0.0
    if rms == 0.0:
        assert np.all(ne == 0.0), "nonzero output where the reference is exactly zero"
        return 0.0
    return float(np.max(ne / np.maximum(nr, floor * rms)))


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
