"""Seeded synthetic inputs for the equivariant graph attention hot path.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It holds no arithmetic of the method itself: it only draws
atom positions, features and weights, rounds them to the storage formats the
kernels read, and enumerates the coupling-path order that fixes the weight
layout (an interface fact).

Workloads follow the systems the pages describe or measure on:

* "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §4.3 (216-water RDF
  box), §1.1 (32,768-atom systems), §3.2 (K = 256 neighbours, 10^5 atoms) and
  §5.1 (num_heads 16, channels 128, edge_cutoff 5 Å, ℓ_max 2-3).

Position recipe (all workloads): random sequential addition.  Candidates are
drawn in blocks of 4096 from uniform(0, side)^3 and accepted in order when no
already accepted point lies closer than 0.9 Å.  The centroid (fp64) is then
subtracted and coordinates are rounded to the 2^-16 Å grid.  The water box
instead places oxygens on a jittered 6^3 grid and adds two hydrogens per
oxygen in a uniformly random orientation.

Feature recipe: ``numpy.random.default_rng([seed, tag])`` with tag 1 -> h,
2 -> q, 3 -> k, 4 -> w1, 5 -> w2, 6 -> wq, 7 -> wk (the invariant query/key
projection weights, float32 [C][H*dk], N(0, 1/C)), 8 -> the SO(2) weights of
the edge-centric comparison convolution (float32 [NW][C], N(0, 1/(lmax+1))).  h, q, k ~ N(0, 1); the weight of path p is
N(0, 1/fan_in(ℓo(p))) with fan_in the number of paths that feed ℓo.  For the
bf16 workloads h, q and k are rounded to bf16 (round to nearest even) and
returned as float32 arrays that hold exactly those values.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import numpy as np

#: positions are integers on this grid (Å per unit)
GRID_BITS = 16
GRID_QUANTUM = 2.0 ** -GRID_BITS

MIN_DIST = 0.9          # Å, random sequential addition exclusion distance
RSA_BLOCK = 4096        # candidates drawn per block


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    system: str          # "cube" or "water"
    n: int               # atoms
    side: float          # Å, edge of the box the atoms are drawn in
    cutoff: float        # Å, radius-graph cutoff (inclusive)
    K: int               # padded neighbour slots per atom
    lmax: int            # highest irrep degree
    C: int               # channels per degree
    H: int               # attention heads
    dk: int              # key / query width per head
    dtype: str           # storage of h, q, k and h': "f32" or "bf16"

    @property
    def D(self) -> int:
        return (self.lmax + 1) ** 2

    @property
    def cutoff_q(self) -> int:
        return cutoff_to_grid(self.cutoff)


def _cube_side(n: int, density: float = 0.1) -> float:
    return float((n / density) ** (1.0 / 3.0))


#: the five synthetic systems, smallest first
WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("uniform64_l1_f32", "cube", 64, 10.0, 5.0, 32, 1, 16, 2, 8, "f32"),
    Workload("water216_l2_f32", "water", 648, 18.6, 5.0, 64, 2, 128, 16, 16, "f32"),
    Workload("uniform4096_l2_bf16", "cube", 4096, _cube_side(4096), 5.0, 64, 2, 128, 16, 16, "bf16"),
    Workload("uniform32768_K256_l2_bf16", "cube", 32768, _cube_side(32768), 8.2, 256, 2, 128, 16, 16, "bf16"),
    Workload("uniform100000_l3_bf16", "cube", 100000, _cube_side(100000), 5.0, 96, 3, 128, 16, 16, "bf16"),
]}
WORKLOAD_ORDER: List[str] = list(WORKLOADS)


def cutoff_to_grid(cutoff: float) -> int:
    """Cutoff in grid units, rounded to nearest."""
    return int(np.rint(cutoff / GRID_QUANTUM))


def coupling_paths(lmax: int) -> List[Tuple[int, int, int]]:
    """Coupling paths (ℓi, ℓf, ℓo) in the order the weight rows use.

    Order: ℓo ascending, then ℓi ascending, then ℓf ascending, keeping every
    triple with |ℓi - ℓf| <= ℓo <= ℓi + ℓf and all three <= lmax.
    """
    out = []
    for lo in range(lmax + 1):
        for li in range(lmax + 1):
            for lf in range(lmax + 1):
                if abs(li - lf) <= lo <= li + lf:
                    out.append((li, lf, lo))
    return out


def _rsa_cube(n: int, side: float, rng: np.random.Generator) -> np.ndarray:
    """Random sequential addition of n points in [0, side)^3."""
    from scipy.spatial import cKDTree

    accepted = np.zeros((0, 3))
    while accepted.shape[0] < n:
        cand = rng.uniform(0.0, side, (RSA_BLOCK, 3))
        ok = np.ones(RSA_BLOCK, dtype=bool)
        if accepted.shape[0]:
            tree = cKDTree(accepted)
            d, _ = tree.query(cand, k=1)
            ok &= d >= MIN_DIST
        # resolve clashes inside the block in draw order
        pairs = cKDTree(cand).query_pairs(MIN_DIST, output_type="ndarray")
        partners: Dict[int, List[int]] = {}
        for a, b in pairs:
            a, b = int(min(a, b)), int(max(a, b))
            if np.sum((cand[a] - cand[b]) ** 2) < MIN_DIST ** 2:
                partners.setdefault(b, []).append(a)
        keep = np.zeros(RSA_BLOCK, dtype=bool)
        for i in range(RSA_BLOCK):
            if not ok[i]:
                continue
            if any(keep[a] for a in partners.get(i, ())):
                continue
            keep[i] = True
        idx = np.nonzero(keep)[0][: n - accepted.shape[0]]
        accepted = np.concatenate([accepted, cand[idx]], axis=0)
    return accepted


def _random_rotation(rng: np.random.Generator) -> np.ndarray:
    """Uniformly random rotation matrix from a normalised Gaussian quaternion."""
    w, x, y, z = rng.standard_normal(4)
    s = np.sqrt(w * w + x * x + y * y + z * z)
    w, x, y, z = w / s, x / s, y / s, z / s
    return np.array([
        [1 - 2 * (y * y + z * z), 2 * (x * y - w * z), 2 * (x * z + w * y)],
        [2 * (x * y + w * z), 1 - 2 * (x * x + z * z), 2 * (y * z - w * x)],
        [2 * (x * z - w * y), 2 * (y * z + w * x), 1 - 2 * (x * x + y * y)],
    ])


def _water_box(rng: np.random.Generator, per_side: int = 6, spacing: float = 3.1,
               jitter: float = 0.3) -> np.ndarray:
    """216 rigid waters (O-H 0.96 Å, H-O-H 104.5°), atoms ordered O, H, H."""
    half = np.deg2rad(104.5) / 2.0
    local = np.array([[0.0, 0.0, 0.0],
                      [0.96 * np.sin(half), 0.0, 0.96 * np.cos(half)],
                      [-0.96 * np.sin(half), 0.0, 0.96 * np.cos(half)]])
    out = []
    for ix in range(per_side):
        for iy in range(per_side):
            for iz in range(per_side):
                o = spacing * (np.array([ix, iy, iz]) + 0.5)
                o = o + rng.uniform(-jitter, jitter, 3)
                rot = _random_rotation(rng)
                out.append(o + local @ rot.T)
    return np.concatenate(out, axis=0)


def positions(wl: Workload, seed: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Centred positions: (int32 grid coordinates [N,3], float32 Å [N,3]).

    The float32 array equals the grid coordinates times 2^-16 exactly.
    """
    rng = np.random.default_rng(seed)
    if wl.system == "cube":
        p = _rsa_cube(wl.n, wl.side, rng)
    elif wl.system == "water":
        p = _water_box(rng)
        assert p.shape[0] == wl.n
    else:
        raise ValueError(wl.system)
    p = p - p.mean(axis=0)
    pq = np.rint(p / GRID_QUANTUM).astype(np.int64)
    assert np.abs(pq).max() < 2 ** 24, "grid coordinates must be exact in float32"
    pq = pq.astype(np.int32)
    pf = (pq.astype(np.float64) * GRID_QUANTUM).astype(np.float32)
    return pq, pf


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest even); returns float32."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def features(wl: Workload, seed: int = 0) -> Dict[str, np.ndarray]:
    """h [N,D,C], q and k [N,H,dk], w1 and w2 [P,C]; all float32."""
    def g(tag):
        return np.random.default_rng([seed, tag])

    n, D, C, H, dk = wl.n, wl.D, wl.C, wl.H, wl.dk
    h = g(1).standard_normal((n, D, C), dtype=np.float32)
    q = g(2).standard_normal((n, H, dk), dtype=np.float32)
    k = g(3).standard_normal((n, H, dk), dtype=np.float32)
    paths = coupling_paths(wl.lmax)
    fan = {lo: sum(1 for p in paths if p[2] == lo) for lo in range(wl.lmax + 1)}
    scale = np.array([1.0 / np.sqrt(fan[p[2]]) for p in paths], dtype=np.float32)[:, None]
    w1 = g(4).standard_normal((len(paths), C), dtype=np.float32) * scale
    w2 = g(5).standard_normal((len(paths), C), dtype=np.float32) * scale
    if wl.dtype == "bf16":
        h, q, k = round_bf16(h), round_bf16(q), round_bf16(k)
    return {"h": h, "q": q, "k": k, "w1": w1.astype(np.float32), "w2": w2.astype(np.float32)}


def projection_weights(wl: Workload, seed: int = 0) -> Dict[str, np.ndarray]:
    """wq, wk float32 [C][H*dk] ~ N(0, 1/C): column h*dk + d of wq maps the
    degree-0 channels of an atom's features to component d of its head-h query
    (so q ~ N(0, 1) for h ~ N(0, 1))."""
    def g(tag):
        return np.random.default_rng([seed, tag])

    C, HD = wl.C, wl.H * wl.dk
    s = np.float32(1.0 / np.sqrt(C))
    return {"wq": g(6).standard_normal((C, HD), dtype=np.float32) * s,
            "wk": g(7).standard_normal((C, HD), dtype=np.float32) * s}


def escn_weight_count(lmax: int, mmax: int) -> int:
    """Rows of the SO(2) weight array: (lmax+1)^2 for order 0, then two blocks of
    (lmax+1-m)^2 for each order 1 <= m <= mmax (the layout is an interface fact)."""
    return (lmax + 1) ** 2 + sum(2 * (lmax + 1 - m) ** 2 for m in range(1, mmax + 1))


def escn_weights(wl: Workload, mmax: int, seed: int = 0) -> np.ndarray:
    """float32 [NW][C] ~ N(0, 1/(lmax+1)): each output degree mixes lmax+1 inputs."""
    nw = escn_weight_count(wl.lmax, mmax)
    g = np.random.default_rng([seed, 8])
    return (g.standard_normal((nw, wl.C), dtype=np.float32)
            * np.float32(1.0 / np.sqrt(wl.lmax + 1))).astype(np.float32)


def make(wl: Workload, seed: int = 0) -> Dict[str, np.ndarray]:
    """All inputs of one workload: positions plus features."""
    pq, pf = positions(wl, seed)
    out = features(wl, seed)
    out["pos_q"] = pq
    out["pos"] = pf
    return out


def small_cube(n: int, side: float, cutoff: float, K: int, lmax: int, C: int, H: int,
               dk: int, dtype: str = "f32", name: str = "") -> Workload:
    """An ad-hoc cube workload for parity tests at other sizes."""
    return Workload(name or f"uniform{n}_l{lmax}_{dtype}", "cube", n, side, cutoff, K,
                    lmax, C, H, dk, dtype)
