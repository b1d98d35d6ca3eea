"""Pins of the oracle's invariant query/key projection (oracle/projection.py).

"E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation Memory"
§2.2, Eq. 6: queries and keys are SO(3)-invariant scalar projections of the
node features.  The reading pinned here: a linear map, without bias, of each
atom's degree-0 channels to every head.  A plausible mistake (the wrong degree
block, transposed weights, a head/component index swapped) fails one of:

* a one-hot weight places one input channel into one (head, component) slot;
* a pure-Python triple loop on tiny inputs;
* q, k and the logits are unchanged when every degree block of h is rotated
  by its Wigner-D matrix (a projection that read any degree > 0 would change);
* the composed forward with projected queries and keys is rotation-equivariant;
* the bf16 storage rounding equals torch's float32 -> bfloat16 conversion
  (round half to even), ties included.
"""
import numpy as np
import torch

from oracle import so3
from oracle.attention import forward, logits
from oracle.graph import radius_graph
from oracle.projection import invariant_projection
from oracle.storage import round_bf16
from equivariant_graph_attention_b200 import synth

RNG = np.random.default_rng(61)


def _feats(n=7, lmax=2, C=6, H=2, dk=3, seed=2):
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((n, (lmax + 1) ** 2, C))
    wq = rng.standard_normal((C, H * dk))
    wk = rng.standard_normal((C, H * dk))
    return h, wq, wk


def test_one_hot_weight_selects_one_channel():
    h, wq, wk = _feats()
    H, dk = 2, 3
    for c0, h0, d0 in [(0, 0, 0), (5, 1, 2), (3, 0, 1)]:
        w = np.zeros_like(wq)
        w[c0, h0 * dk + d0] = 1.0
        q, k = invariant_projection(h, w, 2.0 * w, H, dk)
        want = np.zeros((h.shape[0], H, dk))
        want[:, h0, d0] = h[:, 0, c0]
        assert np.array_equal(q, want)
        assert np.array_equal(k, 2.0 * want)


def test_matches_a_plain_loop():
    h, wq, wk = _feats(n=3, C=4, H=2, dk=2)
    q, k = invariant_projection(h, wq, wk, 2, 2)
    for i in range(3):
        for hh in range(2):
            for d in range(2):
                sq = sk = 0.0
                for c in range(4):
                    sq += h[i][0][c] * wq[c][hh * 2 + d]
                    sk += h[i][0][c] * wk[c][hh * 2 + d]
                assert abs(q[i, hh, d] - sq) < 1e-12 and abs(k[i, hh, d] - sk) < 1e-12


def _rotate_blocks(h, G, lmax):
    out = np.array(h, dtype=np.float64)
    for l in range(lmax + 1):
        D = so3.wigner_D(l, G)
        out[:, l * l:(l + 1) ** 2] = np.einsum("ab,nbc->nac", D, out[:, l * l:(l + 1) ** 2])
    return out


def test_queries_keys_and_logits_are_invariant():
    lmax = 3
    h, wq, wk = _feats(n=9, lmax=lmax, C=5, H=3, dk=4)
    G = so3.alignment_rotation(RNG.standard_normal(3)) @ so3.rot_z(1.3)
    q, k = invariant_projection(h, wq, wk, 3, 4)
    qr, kr = invariant_projection(_rotate_blocks(h, G, lmax), wq, wk, 3, 4)
    assert np.max(np.abs(qr - q)) < 1e-12 and np.max(np.abs(kr - k)) < 1e-12
    assert np.max(np.abs(logits(qr[0], kr) - logits(q[0], k))) < 1e-12
    # reading a degree-1 block instead breaks the invariance (the pin has teeth)
    bad = lambda x: x[:, 1, :] @ wq
    assert np.max(np.abs(bad(_rotate_blocks(h, G, lmax)) - bad(h))) > 1e-3


def test_projected_forward_is_rotation_equivariant():
    lmax, C, H, dk = 2, 8, 2, 4
    wl = synth.small_cube(24, 6.0, 3.5, 16, lmax, C, H, dk, "f32")
    d = synth.make(wl, seed=3)
    w = synth.projection_weights(wl, seed=3)
    nbrs, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    q, k = invariant_projection(d["h"], w["wq"], w["wk"], H, dk)
    out = forward(d["h"], d["pos"], q, k, d["w1"], d["w2"], lmax, nbrs)
    G = so3.alignment_rotation(RNG.standard_normal(3)) @ so3.rot_z(0.4)
    h_rot = _rotate_blocks(d["h"], G, lmax)
    qr, kr = invariant_projection(h_rot, w["wq"], w["wk"], H, dk)
    out_rot = forward(h_rot, d["pos"].astype(np.float64) @ G.T, qr, kr, d["w1"], d["w2"], lmax,
                      nbrs)
    exp = _rotate_blocks(out, G, lmax)
    assert np.max(np.abs(out_rot - exp)) < 1e-10 * np.max(np.abs(exp))


def test_bf16_rounding_matches_torch():
    x = RNG.standard_normal(20000).astype(np.float32) * np.float32(37.0)
    # exact ties: low 16 bits 0x8000 on both even and odd upper halves
    bits = (RNG.integers(0x3f00, 0x4400, 2000, dtype=np.uint32) << 16) | np.uint32(0x8000)
    ties = bits.view(np.float32)
    for v in (x, ties, -ties):
        want = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
        assert np.array_equal(round_bf16(v), want)
