"""GPU parity of the invariant query/key projection (egat_qk_projection)
against the oracle (oracle/projection.py).

"E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation Memory"
§2.2, Eq. 6: queries and keys are SO(3)-invariant scalar projections of the
node features (reading: a linear map of each atom's degree-0 channels).

* q and k of every atom against the oracle's float64 product, per
  (atom, head) row: e = ||v_gpu - v_ref|| / max(||v_ref||, floor RMS) with
  the storage bars and floors of parity_util; bf16 outputs are one rounding
  of a float32-accurate product: within one bf16 unit of the oracle's own
  rounding plus the float32 accumulation error, 2^-19 of the sum of the
  terms' magnitudes.
* The tensor-core path (bf16, C = 128, H*dk = 256) on every bf16 workload,
  ragged tails (1, 63, 65, 127, 129 and 1,000 atoms: partial 128-atom
  tiles) and the plain path (float32 workloads, other channel counts).
* Rotating every degree block of h by its Wigner-D matrix leaves the GPU's
  q and k bitwise unchanged (only degree 0 is read).
* The projected queries and keys drive the fused forward: egat_qk_projection
  then egat_forward against the oracle forward on the oracle's projected
  (and, for bf16 workloads, bf16-stored) q and k.
"""
import functools

import numpy as np
import pytest
import torch

from oracle import so3
from oracle.attention import forward as oracle_forward
from oracle.graph import radius_graph
from oracle.projection import invariant_projection
from oracle.storage import round_bf16
from equivariant_graph_attention_b200 import synth
from tests.parity_util import (FLOOR, TOL, block_rel_error, channel_rel_error, device_inputs,
                               vec_rel_error, shape_of)

pytestmark = pytest.mark.gpu


def _egat():
    from equivariant_graph_attention_b200 import egat
    return egat


@functools.lru_cache(maxsize=None)
def _data(name):
    wl = synth.WORKLOADS[name]
    return wl, synth.make(wl), synth.projection_weights(wl)


def _project(wl, h, w):
    egat = _egat()
    st = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    hd = torch.from_numpy(np.ascontiguousarray(h)).to("cuda", dtype=st)
    wq = torch.from_numpy(w["wq"]).cuda()
    wk = torch.from_numpy(w["wk"]).cuda()
    q, k = egat.egat_qk_projection(shape_of(wl), hd, wq, wk)
    torch.cuda.synchronize()
    return q.float().cpu().numpy(), k.float().cpu().numpy()


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_projection_parity(name):
    wl, d, w = _data(name)
    q, k = _project(wl, d["h"], w)
    rq, rk = invariant_projection(d["h"], w["wq"], w["wk"], wl.H, wl.dk)
    eq, ek = vec_rel_error(q, rq, FLOOR[wl.dtype]), vec_rel_error(k, rk, FLOOR[wl.dtype])
    print(f"projection {name}: q {eq:.2e}  k {ek:.2e}")
    assert eq < TOL[wl.dtype] and ek < TOL[wl.dtype]
    if wl.dtype == "bf16":
        # one rounding of a float32-accurate product: within one bf16 unit of
        # the oracle's own rounding (boundaries may fall either way), plus
        # the float32 accumulation error, bounded by 2^-19 of the terms' sum
        h0 = np.abs(np.asarray(d["h"], np.float64)[:, 0, :])
        for got, ref, wm in ((q, rq, w["wq"]), (k, rk, w["wk"])):
            terms = (h0 @ np.abs(np.asarray(wm, np.float64))).reshape(ref.shape)
            ulp = np.abs(round_bf16(ref)) * 2.0 ** -7
            assert np.all(np.abs(got - round_bf16(ref)) <= ulp + terms * 2.0 ** -19)
    assert _egat().egat_take_device_status() == _egat().EGAT_OK


@pytest.mark.parametrize("n", [1, 63, 65, 127, 129, 1000])
@pytest.mark.parametrize("dtype,C,H,dk", [("bf16", 128, 16, 16), ("f32", 64, 4, 16),
                                          ("bf16", 32, 4, 8)])
def test_projection_ragged(n, dtype, C, H, dk):
    wl = synth.small_cube(n, max(3.0, (n / 0.1) ** (1 / 3)), 4.0, 16, 2, C, H, dk, dtype)
    d = synth.features(wl, seed=n)
    w = synth.projection_weights(wl, seed=n)
    q, k = _project(wl, d["h"], w)
    rq, rk = invariant_projection(d["h"], w["wq"], w["wk"], H, dk)
    f = FLOOR[dtype]
    assert vec_rel_error(q, rq, f) < TOL[dtype] and vec_rel_error(k, rk, f) < TOL[dtype]


def test_projection_ignores_higher_degrees():
    wl, d, w = _data("uniform4096_l2_bf16")
    G = so3.alignment_rotation(np.array([0.3, -1.1, 0.7])) @ so3.rot_z(0.9)
    h = np.array(d["h"], dtype=np.float64)
    for l in range(1, wl.lmax + 1):
        h[:, l * l:(l + 1) ** 2] = np.einsum("ab,nbc->nac", so3.wigner_D(l, G),
                                             h[:, l * l:(l + 1) ** 2])
    h = synth.round_bf16(h.astype(np.float32))
    q0, k0 = _project(wl, d["h"], w)
    q1, k1 = _project(wl, h, w)
    assert np.array_equal(q0, q1) and np.array_equal(k0, k1)


@pytest.mark.parametrize("name", ["uniform64_l1_f32", "water216_l2_f32", "uniform4096_l2_bf16"])
def test_projected_forward(name):
    """egat_qk_projection -> egat_forward against the oracle forward with the
    oracle's projected queries and keys (stored as bf16 on bf16 workloads)."""
    egat = _egat()
    wl, d, w = _data(name)
    dev = device_inputs(wl, d)
    q, k = egat.egat_qk_projection(shape_of(wl), dev["h"], torch.from_numpy(w["wq"]).cuda(),
                                   torch.from_numpy(w["wk"]).cuda())
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    out = egat.egat_forward(shape_of(wl), dev["h"], dev["pos"], q, k, g["nbr"], g["cnt"],
                            dev["w1"], dev["w2"], order=g["order"]).cpu().numpy()
    rq, rk = invariant_projection(d["h"], w["wq"], w["wk"], wl.H, wl.dk)
    if wl.dtype == "bf16":
        rq, rk = round_bf16(rq), round_bf16(rk)
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    ref = oracle_forward(d["h"], d["pos"], rq, rk, d["w1"], d["w2"], wl.lmax, lists)
    e_block = block_rel_error(out, ref, wl.lmax)
    print(f"projected forward {name}: block {e_block:.2e}")
    assert e_block < TOL[wl.dtype]
    if wl.dtype == "f32":
        assert channel_rel_error(out, ref, wl.lmax, FLOOR["f32"]) < TOL["f32"]


def test_projection_weights_at_any_float_offset():
    """Weights that are only 4-byte aligned (an offset view) give q and k within
    the bf16 bar of the oracle: the kernels read them as single floats."""
    wl, d, w = _data("uniform4096_l2_bf16")
    egat = _egat()
    hd = torch.from_numpy(np.ascontiguousarray(d["h"])).to("cuda", dtype=torch.bfloat16)
    buf = torch.zeros(2 * wl.C * wl.H * wl.dk + 2, dtype=torch.float32, device="cuda")
    n = wl.C * wl.H * wl.dk
    wq = buf[1:1 + n].view(wl.C, wl.H * wl.dk)
    wk = buf[1 + n:1 + 2 * n].view(wl.C, wl.H * wl.dk)
    wq.copy_(torch.from_numpy(w["wq"]))
    wk.copy_(torch.from_numpy(w["wk"]))
    assert wq.data_ptr() % 16 != 0
    q, k = egat.egat_qk_projection(shape_of(wl), hd, wq, wk)
    rq, rk = invariant_projection(d["h"], w["wq"], w["wk"], wl.H, wl.dk)
    f = FLOOR["bf16"]
    assert vec_rel_error(q.float().cpu().numpy(), rq, f) < TOL["bf16"]
    assert vec_rel_error(k.float().cpu().numpy(), rk, f) < TOL["bf16"]


def test_projection_outputs_at_a_float_offset():
    """q and k buffers that are only 4-byte aligned (offset views) take the
    plain kernel (the tensor-core kernel stores 16-byte row segments) and
    give the same values within the bf16 bar of the oracle."""
    wl, d, w = _data("uniform4096_l2_bf16")
    egat = _egat()
    hd = torch.from_numpy(np.ascontiguousarray(d["h"])).to("cuda", dtype=torch.bfloat16)
    wq = torch.from_numpy(w["wq"]).cuda()
    wk = torch.from_numpy(w["wk"]).cuda()
    m = wl.n * wl.H * wl.dk
    buf = torch.zeros(2 * m + 4, dtype=torch.bfloat16, device="cuda")
    q = buf[2:2 + m].view(wl.n, wl.H, wl.dk)
    k = buf[2 + m + 2:2 + 2 * m + 2].view(wl.n, wl.H, wl.dk)
    assert q.data_ptr() % 16 != 0 and q.data_ptr() % 4 == 0 and k.data_ptr() % 4 == 0
    egat.egat_qk_projection(shape_of(wl), hd, wq, wk, q=q, k=k)
    torch.cuda.synchronize()
    rq, rk = invariant_projection(d["h"], w["wq"], w["wk"], wl.H, wl.dk)
    f = FLOOR["bf16"]
    assert vec_rel_error(q.float().cpu().numpy(), rq, f) < TOL["bf16"]
    assert vec_rel_error(k.float().cpu().numpy(), rk, f) < TOL["bf16"]
