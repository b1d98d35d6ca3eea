"""GPU parity of the edge-centric eSCN convolution (egat_escn_conv) against
the oracle (oracle/escn.py), which its own pins fix (identity weights, the
m = 0 projector's closed form, roll independence, rotation equivariance).

"EquiformerV3: Scaling Efficient, Expressive, and General SE(3)-Equivariant Graph Attention Transformers", section "eSCN卷积与SO(2)线性层"; the comparison
workload of the node-centric factorisation in
"E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §3.1.

Both sides read identical inputs (bf16 features exactly as stored), so the
per-(atom, degree, channel) metric applies with the identical-input floors
of parity_util, at the float32 bar on float32 workloads and the bf16 bar on
bf16 ones.  Every workload (sampled targets where the per-edge oracle would
take minutes), each truncation order M_max, ragged systems with an isolated
atom, coincident atoms (r_ij = 0) and edges along +z and -z.
"""
import functools

import numpy as np
import pytest
import torch

from oracle.escn import escn_conv
from oracle.graph import radius_graph
from equivariant_graph_attention_b200 import synth
from tests.parity_util import FLOOR, TOL, channel_rel_error, device_inputs, sample_targets, shape_of

pytestmark = pytest.mark.gpu


def _egat():
    from equivariant_graph_attention_b200 import egat
    return egat


@functools.lru_cache(maxsize=None)
def _data(name):
    wl = synth.WORKLOADS[name]
    return wl, synth.make(wl)


def _run(wl, d, mmax, w):
    egat = _egat()
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    out = egat.egat_escn_conv(shape_of(wl), mmax, dev["h"], dev["pos"], g["nbr"], g["cnt"],
                              torch.from_numpy(w).cuda(), order=g["order"])
    torch.cuda.synchronize()
    return out.cpu().numpy(), g


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_escn_parity(name):
    wl, d = _data(name)
    mmax = wl.lmax
    w = synth.escn_weights(wl, mmax)
    out, g = _run(wl, d, mmax, w)
    if wl.n <= 700:
        rows = list(range(wl.n))
    else:
        rows = sample_targets(wl, g["cnt"].cpu().numpy(), count=60 if wl.n <= 4096 else 24)
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K, rows=rows)
    ref = escn_conv(d["h"], d["pos"], w, wl.lmax, mmax, lists, targets=rows)
    e = channel_rel_error(out[rows], ref, wl.lmax, FLOOR[wl.dtype])
    print(f"escn {name}: per-channel {e:.2e}")
    assert e < TOL[wl.dtype]


@pytest.mark.parametrize("mmax", [0, 1, 2])
def test_escn_truncation_orders(mmax):
    wl, d = _data("water216_l2_f32")
    w = synth.escn_weights(wl, mmax, seed=mmax)
    out, _ = _run(wl, d, mmax, w)
    rows = list(range(0, wl.n, 3))
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K, rows=rows)
    ref = escn_conv(d["h"], d["pos"], w, wl.lmax, mmax, lists, targets=rows)
    assert channel_rel_error(out[rows], ref, wl.lmax, FLOOR["f32"]) < TOL["f32"]


@pytest.mark.parametrize("lmax,C,dtype", [(1, 16, "f32"), (2, 64, "f32"), (3, 128, "bf16"),
                                          (3, 32, "f32")])
def test_escn_edge_cases(lmax, C, dtype):
    """Ragged system: an isolated atom (zero output), two coincident atoms
    (r_ij = 0, identity frame), neighbours straight above and below an atom
    (edges along +z and -z)."""
    pts = np.array([[0, 0, 0], [0, 0, 1.5], [0, 0, -1.2], [0.9, 0.3, -0.4], [0.9, 0.3, -0.4],
                    [-1.1, 0.8, 0.6], [50, 50, 50], [0.2, -1.3, 0.9]], dtype=np.float64)
    n = len(pts)
    wl = synth.small_cube(n, 4.0, 2.5, 8, lmax, C, 1, 8, dtype)
    feats = synth.features(wl, seed=lmax)
    pq = np.rint(pts / synth.GRID_QUANTUM).astype(np.int32)
    feats.update(pos_q=pq, pos=(pq.astype(np.float64) * synth.GRID_QUANTUM).astype(np.float32))
    w = synth.escn_weights(wl, lmax, seed=3)
    out, _ = _run(wl, feats, lmax, w)
    lists, _ = radius_graph(pq, wl.cutoff_q, K=wl.K)
    assert len(lists[6]) == 0 and np.all(out[6] == 0.0)
    assert 4 in lists[3]                                  # the coincident pair
    ref = escn_conv(feats["h"], feats["pos"], w, lmax, lmax, lists)
    assert channel_rel_error(out, ref, lmax, FLOOR[dtype]) < TOL[dtype]
