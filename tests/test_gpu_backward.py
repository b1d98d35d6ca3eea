"""GPU parity of the backward pass (egat_backward) against the oracle's
backward (oracle/backward.py), which finite differences of the oracle forward
pin (tests/test_oracle_backward.py).

dL/dh is compared per (atom, degree, channel) vector and block by block (the
forward's metrics, parity_util); dL/dq and dL/dk row by row over (atom, head)
and dL/dr row by row over atoms with the same relative-norm metric, with and
without the 1e-3 RMS floor.  Inputs are identical on both sides.  Bars as for
the forward: 1e-4 for float32 storage, 2e-2 for bf16 storage; the bf16 ℓmax 3
shape (the 100,000-atom workload's) is covered on ragged systems and on
sampled atoms at full size.  bf16 shapes of the tensor-core forward run the tiled
passes (tf32 gradient products); they are checked with and without the
traversal order, on ragged systems of 1 and 37 atoms (an isolated atom, an
atom at the origin, a ragged last tile) and at full size (32,768 atoms,
K = 256) on sampled atoms against the oracle evaluated at those atoms.  Also:
tiny float32 ragged systems, and bitwise determinism across calls.
"""
import functools

import numpy as np
import pytest
import torch

from oracle.attention import aggregate, source_coupling
from oracle.backward import (attention_backward_at, backward as oracle_backward, coupling_position_grad,
                             position_grad, tensor_product_adjoint)
from oracle.graph import radius_graph
from equivariant_graph_attention_b200 import synth
from tests.parity_util import (BWD_FLOOR, TOL, block_rel_error, channel_rel_error,
                               device_inputs, shape_of, vec_rel_error)

pytestmark = pytest.mark.gpu

SMALL = ["uniform64_l1_f32", "water216_l2_f32", "uniform4096_l2_bf16"]


def _egat():
    from equivariant_graph_attention_b200 import egat
    return egat


def row_rel_error(gpu: np.ndarray, ref: np.ndarray) -> float:
    """max over rows of ||gpu - ref|| / ||ref||.

    A row whose reference is exactly zero (an atom without neighbours, or a
    target with a single neighbour, whose softmax weight is 1 so that its logit
    gradient vanishes) must be negligible against the tensor's scale: at most
    1e-6 of its largest reference row.  The GPU forms dq as
    sum alpha dalpha k - Delta sum alpha k, whose two terms cancel to rounding
    there rather than to an exact zero.
    """
    g = np.asarray(gpu, dtype=np.float64).reshape(-1, gpu.shape[-1])
    r = np.asarray(ref, dtype=np.float64).reshape(-1, ref.shape[-1])
    nr = np.linalg.norm(r, axis=1)
    ne = np.linalg.norm(g - r, axis=1)
    zero = nr == 0.0
    scale = float(nr.max()) if nr.size else 0.0
    assert np.all(ne[zero] <= 1e-6 * scale), "gradient far from zero where the reference is zero"
    return float(np.max(ne[~zero] / nr[~zero])) if np.any(~zero) else 0.0


def check_grads(wl, got, ref, tol, label):
    """Every metric of the module docstring below the bar."""
    dh, dq, dk, dr = got
    rdh, rdq, rdk, rdr = ref
    floor = BWD_FLOOR[wl.dtype]
    e = {"dh block": block_rel_error(dh, rdh, wl.lmax),
         "dh channel": channel_rel_error(dh, rdh, wl.lmax, floor=floor),
         "dq": row_rel_error(dq, rdq), "dq floored": vec_rel_error(dq, rdq, floor),
         "dk": row_rel_error(dk, rdk), "dk floored": vec_rel_error(dk, rdk, floor),
         "dr": row_rel_error(dr, rdr), "dr floored": vec_rel_error(dr, rdr, floor)}
    print(f"backward {label}: " + "  ".join(f"{k} {v:.2e}" for k, v in e.items()))
    bad = {k: v for k, v in e.items() if not v < tol}
    assert not bad, bad


@functools.lru_cache(maxsize=None)
def _case(name):
    wl = synth.WORKLOADS[name]
    d = synth.make(wl)
    G = np.random.default_rng(17).standard_normal((wl.n, wl.D, wl.C)).astype(np.float32)
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    ref = oracle_backward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists, G)
    dr = position_grad(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists, G)
    return wl, d, G, ref + (dr,)


def _run(wl, d, G, use_order=True):
    egat = _egat()
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    Gd = torch.from_numpy(G).cuda()
    return egat.egat_backward(shape_of(wl), dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"],
                              g["cnt"], dev["w1"], dev["w2"], Gd,
                              order=g["order"] if use_order else None)


@pytest.mark.parametrize("name,use_order", [(n, True) for n in SMALL] + [("uniform4096_l2_bf16", False)])
def test_backward_parity(name, use_order):
    wl, d, G, (rdh, rdq, rdk, rdr) = _case(name)
    dh, dq, dk, dr = (x.cpu().numpy() for x in _run(wl, d, G, use_order))
    tol = TOL[wl.dtype]
    check_grads(wl, (dh, dq, dk, dr), (rdh, rdq, rdk, rdr), tol, name)


def test_backward_is_deterministic():
    wl, d, G, _ = _case("uniform4096_l2_bf16")
    a = _run(wl, d, G)
    b = _run(wl, d, G)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert _egat().egat_take_device_status() == _egat().EGAT_OK


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_backward_edge_cases(lmax):
    """Ragged systems with an isolated atom (all gradients zero) and atoms at the
    origin and on the z axis."""
    n = 23
    rng = np.random.default_rng(40 + lmax)
    pts = rng.uniform(-3.0, 3.0, (n, 3))
    pts[0] = 0.0
    pts[1] = [0.0, 0.0, -1.3]
    pts[2] = [60.0, 60.0, 60.0]            # isolated
    wl = synth.small_cube(n, 6.0, 3.0, 16, lmax, 32, 4, 8, "f32")
    feats = synth.features(wl, seed=n + lmax)
    pq = np.rint(pts / synth.GRID_QUANTUM).astype(np.int32)
    feats.update(pos_q=pq, pos=(pq.astype(np.float64) * synth.GRID_QUANTUM).astype(np.float32))
    G = rng.standard_normal((n, wl.D, wl.C)).astype(np.float32)
    dh, dq, dk, dr = (x.cpu().numpy() for x in _run(wl, feats, G))
    lists, _ = radius_graph(pq, wl.cutoff_q, K=wl.K)
    rdh, rdq, rdk = oracle_backward(feats["h"], feats["pos"], feats["q"], feats["k"], feats["w1"],
                                    feats["w2"], lmax, lists, G)
    rdr = position_grad(feats["h"], feats["pos"], feats["q"], feats["k"], feats["w1"],
                        feats["w2"], lmax, lists, G)
    assert not dq[2].any() and not dk[2].any() and not dh[2].any() and not dr[2].any()
    # atom 0 sits at the origin (the zero-radius branch of the position gradient)
    check_grads(wl, (dh, dq, dk, dr), (rdh, rdq, rdk, rdr), TOL["f32"], f"f32 lmax {lmax}")


@pytest.mark.parametrize("lmax", [1, 2, 3])
@pytest.mark.parametrize("n", [1, 37])
def test_tiled_backward_edge_cases(lmax, n):
    """The bf16 C = 128, H = 16, dk = 16 shapes on tiny systems: a single atom
    (empty unions), and 37 atoms (a ragged last tile) with an isolated atom,
    an atom at the origin and one on the negative z axis.  All three run the
    tiled passes; ℓmax 3 is the shape of the 100,000-atom workload (8-row
    stages, the source union swept once for dL/dk and once for dL/dh')."""
    rng = np.random.default_rng(70 + 3 * lmax + n)
    pts = rng.uniform(-3.0, 3.0, (n, 3))
    pts[0] = 0.0
    if n > 2:
        pts[1] = [0.0, 0.0, -1.3]
        pts[2] = [60.0, 60.0, 60.0]        # isolated
    wl = synth.small_cube(n, 6.0, 3.0, 16, lmax, 128, 16, 16, "bf16")
    feats = synth.features(wl, seed=n + lmax)
    pq = np.rint(pts / synth.GRID_QUANTUM).astype(np.int32)
    feats.update(pos_q=pq, pos=(pq.astype(np.float64) * synth.GRID_QUANTUM).astype(np.float32))
    G = rng.standard_normal((n, wl.D, wl.C)).astype(np.float32)
    dh, dq, dk, dr = (x.cpu().numpy() for x in _run(wl, feats, G))
    lists, _ = radius_graph(pq, wl.cutoff_q, K=wl.K)
    rdh, rdq, rdk = oracle_backward(feats["h"], feats["pos"], feats["q"], feats["k"], feats["w1"],
                                    feats["w2"], lmax, lists, G)
    rdr = position_grad(feats["h"], feats["pos"], feats["q"], feats["k"], feats["w1"],
                        feats["w2"], lmax, lists, G)
    if n == 1:
        assert not dq.any() and not dk.any() and not dh.any() and not dr.any()
        return
    assert not dq[2].any() and not dk[2].any() and not dh[2].any() and not dr[2].any()
    check_grads(wl, (dh, dq, dk, dr), (rdh, rdq, rdk, rdr), TOL["bf16"], f"bf16 lmax {lmax} n {n}")
    assert _egat().egat_take_device_status() == _egat().EGAT_OK


@pytest.mark.parametrize("name,count", [("uniform32768_K256_l2_bf16", 12),
                                        ("uniform100000_l3_bf16", 6)])
def test_backward_full_size_sampled(name, count):
    """The full-size bf16 workloads on the tiled passes (32,768 atoms, K = 256,
    ℓmax 2; 100,000 atoms, K = 96, ℓmax 3): dL/dq, dL/dk, dL/dh and dL/dr of sampled
    atoms (random ones, the highest-degree ones, the last atom) against the
    oracle evaluated at those atoms."""
    from tests.test_gpu_parity import _full_degree
    from tests.parity_util import sample_targets
    wl = synth.WORKLOADS[name]
    d = synth.make(wl)
    G = np.random.default_rng(17).standard_normal((wl.n, wl.D, wl.C)).astype(np.float32)
    dh, dq, dk, dr = (x.cpu().numpy() for x in _run(wl, d, G))
    atoms = sample_targets(wl, _full_degree(name), count=count, seed=9)
    # every target whose list may hold a sampled atom lies within the cutoff of it
    first, _ = radius_graph(d["pos_q"], wl.cutoff_q, rows=atoms)
    cand = sorted(set(atoms) | {int(j) for js in first for j in js})
    rows, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K, rows=cand)
    nbrs = dict(zip(cand, rows))
    touched = np.array(sorted(set(cand) | {int(j) for js in rows for j in js}))
    hp = np.zeros((wl.n, wl.D, wl.C))
    dm = np.zeros((wl.n, wl.D, wl.C))
    hp[touched] = source_coupling(d["h"][touched], d["pos"][touched], d["w1"], wl.lmax)
    dm[cand] = tensor_product_adjoint(G[cand], d["pos"][cand], d["w2"], wl.lmax)
    rdhp, rdq, rdk = attention_backward_at(d["q"], d["k"], hp, dm, nbrs, atoms)
    rdh = tensor_product_adjoint(rdhp, d["pos"][atoms], d["w1"], wl.lmax)
    # dL/dr: the target coupling's part (G, m) plus the source coupling's (dh', h)
    a_idx = np.array(atoms)
    m = aggregate(d["q"], d["k"], hp, [nbrs[a] for a in atoms], targets=atoms)
    rdr = (coupling_position_grad(G[a_idx], m, d["pos"][a_idx], d["w2"], wl.lmax)
           + coupling_position_grad(rdhp, d["h"][a_idx], d["pos"][a_idx], d["w1"], wl.lmax))
    check_grads(wl, (dh[a_idx], dq[a_idx], dk[a_idx], dr[a_idx]), (rdh, rdq, rdk, rdr),
                TOL["bf16"], f"{name} sampled")


def test_tiled_backward_random_order():
    """A random permutation as the traversal order: tiles of scattered atoms, so
    both plans hold large unions (the source plan's per-tile capacities near
    the sum of in-degrees).  Gradients are independent of the order up to
    rounding: compared with the oracle at the bf16 bar, and with the
    cell-ordered run."""
    egat = _egat()
    wl, d, G, (rdh, rdq, rdk, rdr) = _case("uniform4096_l2_bf16")
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    perm = torch.from_numpy(np.random.default_rng(23).permutation(wl.n).astype(np.int32)).cuda()
    Gd = torch.from_numpy(G).cuda()
    outs = egat.egat_backward(shape_of(wl), dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"],
                              g["cnt"], dev["w1"], dev["w2"], Gd, order=perm)
    dh, dq, dk, dr = (x.cpu().numpy() for x in outs)
    check_grads(wl, (dh, dq, dk, dr), (rdh, rdq, rdk, rdr), TOL[wl.dtype], "random order")
    assert egat.egat_take_device_status() == egat.EGAT_OK


def test_tiled_backward_without_positions():
    """No dL/dr buffer: the statistics pass skips m and streams key rows alone.
    dL/dh, dL/dq and dL/dk are bitwise those of the call with dL/dr (the
    log-sum-exp does not depend on m) and meet the bf16 bar."""
    egat = _egat()
    wl, d, G, (rdh, rdq, rdk, rdr) = _case("uniform4096_l2_bf16")
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    Gd = torch.from_numpy(G).cuda()
    args = (shape_of(wl), dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"], g["cnt"], dev["w1"],
            dev["w2"], Gd)
    full = egat.egat_backward(*args, order=g["order"])
    lean = egat.egat_backward(*args, positions=False, order=g["order"])
    assert lean[3] is None
    for a, b in zip(full[:3], lean[:3]):
        assert torch.equal(a, b)
    tol = TOL[wl.dtype]
    assert block_rel_error(lean[0].cpu().numpy(), rdh, wl.lmax) < tol
    assert channel_rel_error(lean[0].cpu().numpy(), rdh, wl.lmax,
                             floor=BWD_FLOOR[wl.dtype]) < tol
    assert row_rel_error(lean[1].cpu().numpy(), rdq) < tol
    assert row_rel_error(lean[2].cpu().numpy(), rdk) < tol
    assert egat.egat_take_device_status() == egat.EGAT_OK
