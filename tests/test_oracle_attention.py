"""Pins for the oracle's attention and the composed forward pass (CPU only).

Pages: [EX] "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §3.1-§3.2;
[TS] "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
Memory" §2.2.  Checks: scipy's softmax; weights summing to one; q = 0 giving
the neighbour mean; ℓ_max = 0 reducing to masked scaled-dot-product
attention (torch's CPU routine); invariance to neighbour order; the empty
neighbourhood; identity paths; rotation and permutation equivariance of the
whole forward pass.
"""
import numpy as np
import pytest
import scipy.special
import torch

from oracle import so3
from oracle.attention import (aggregate, forward, logits, softmax_two_pass,
                              source_coupling, head_of_channel)
from oracle.graph import radius_graph
from equivariant_graph_attention_b200 import synth

RNG = np.random.default_rng(99)


def _system(n=24, side=6.0, lmax=2, C=8, H=2, dk=4, cutoff=3.5, seed=3):
    wl = synth.small_cube(n, side, cutoff, 64, lmax, C, H, dk)
    d = synth.make(wl, seed)
    nbrs, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    return wl, d, nbrs


def test_softmax_matches_scipy():
    s = RNG.standard_normal((13, 4)) * 30
    assert np.allclose(softmax_two_pass(s), scipy.special.softmax(s, axis=0), atol=1e-15)


def test_weights_sum_to_one_even_for_large_logits():
    s = RNG.standard_normal((50, 3)) * 800.0
    a = softmax_two_pass(s)
    assert np.all(np.isfinite(a))
    assert np.max(np.abs(a.sum(0) - 1.0)) < 1e-12


def test_zero_query_gives_neighbour_mean():
    wl, d, nbrs = _system()
    q0 = np.zeros_like(d["q"])
    hp = RNG.standard_normal(d["h"].shape)
    m = aggregate(q0, d["k"], hp, nbrs)
    for i, js in enumerate(nbrs):
        if len(js):
            assert np.allclose(m[i], hp[js].mean(0), atol=1e-13)


def test_lmax0_reduces_to_masked_sdpa():
    n, C, H, dk = 30, 12, 3, 5
    wl, d, nbrs = _system(n=n, lmax=0, C=C, H=H, dk=dk, cutoff=3.0)
    assert all(len(js) for js in nbrs)
    w1 = np.ones((1, C))
    w2 = np.ones((1, C))
    out = forward(d["h"], d["pos"], d["q"], d["k"], w1, w2, 0, nbrs)[:, 0, :]
    mask = np.zeros((n, n), dtype=bool)
    for i, js in enumerate(nbrs):
        mask[i, js] = True
    Ch = C // H
    q = torch.tensor(d["q"], dtype=torch.float64).permute(1, 0, 2)[None]   # [1,H,N,dk]
    k = torch.tensor(d["k"], dtype=torch.float64).permute(1, 0, 2)[None]
    v = torch.tensor(d["h"][:, 0, :].reshape(n, H, Ch), dtype=torch.float64).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=torch.tensor(mask)[None, None])
    ref = ref[0].permute(1, 0, 2).reshape(n, C).numpy()
    assert np.max(np.abs(out - ref)) < 1e-12


def test_neighbour_order_does_not_matter_and_empty_is_zero():
    wl, d, nbrs = _system()
    hp = RNG.standard_normal(d["h"].shape)
    m1 = aggregate(d["q"], d["k"], hp, nbrs)
    shuffled = [RNG.permutation(js) for js in nbrs]
    m2 = aggregate(d["q"], d["k"], hp, shuffled)
    assert np.allclose(m1, m2, atol=1e-13)
    empty = [np.zeros(0, dtype=np.int64)] + list(nbrs[1:])
    assert np.array_equal(aggregate(d["q"], d["k"], hp, empty)[0], np.zeros(hp.shape[1:]))


def test_logit_scale_and_head_blocks():
    # channel c belongs to head floor(c*H/C): contiguous blocks of C/H
    assert head_of_channel(16, 2).tolist() == [0] * 8 + [1] * 8
    assert head_of_channel(128, 16).tolist() == list(np.repeat(np.arange(16), 8))
    q = np.zeros((2, 4)); q[1, :] = 1.0
    k = np.zeros((1, 2, 4)); k[0, 1, :] = 2.0
    assert np.allclose(logits(q, k), [[0.0, 8.0 / 2.0]])


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_identity_paths(lmax):
    # paths (l, 0, l) with unit weight return the input ([EX] §3.1 with R^0 = 1)
    plist = so3.paths(lmax)
    C = 6
    w = np.zeros((len(plist), C))
    for p, (li, lf, lo) in enumerate(plist):
        if lf == 0:
            w[p] = 1.0
    x = RNG.standard_normal((5, (lmax + 1) ** 2, C))
    pos = RNG.standard_normal((5, 3)) * 3
    assert np.allclose(source_coupling(x, pos, w, lmax), x, atol=1e-13)


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_forward_rotation_equivariance(lmax):
    wl, d, nbrs = _system(lmax=lmax)
    G = so3.alignment_rotation(RNG.standard_normal(3)) @ so3.rot_z(0.77)
    out = forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], lmax, nbrs)
    h_rot = np.array(d["h"], dtype=np.float64)
    Ds = [so3.wigner_D(l, G) for l in range(lmax + 1)]
    for l in range(lmax + 1):
        h_rot[:, l * l:(l + 1) ** 2] = np.einsum("ab,nbc->nac", Ds[l], h_rot[:, l * l:(l + 1) ** 2])
    pos_rot = d["pos"].astype(np.float64) @ G.T
    out_rot = forward(h_rot, pos_rot, d["q"], d["k"], d["w1"], d["w2"], lmax, nbrs)
    exp = np.array(out)
    for l in range(lmax + 1):
        exp[:, l * l:(l + 1) ** 2] = np.einsum("ab,nbc->nac", Ds[l], exp[:, l * l:(l + 1) ** 2])
    assert np.max(np.abs(out_rot - exp)) < 1e-10 * np.max(np.abs(exp))


def test_forward_permutation_equivariance():
    wl, d, nbrs = _system()
    out = forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, nbrs)
    perm = RNG.permutation(wl.n)
    inv = np.argsort(perm)
    nbrs_p = [inv[nbrs[perm[t]]] for t in range(wl.n)]
    out_p = forward(d["h"][perm], d["pos"][perm], d["q"][perm], d["k"][perm],
                    d["w1"], d["w2"], wl.lmax, nbrs_p)
    assert np.max(np.abs(out_p - out[perm])) < 1e-12 * np.max(np.abs(out))


def test_forward_target_subset_matches_full():
    wl, d, nbrs = _system()
    full = forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, nbrs)
    rows = [3, 0, 17]
    sub = forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax,
                  [nbrs[i] for i in rows], targets=rows)
    assert np.allclose(sub, full[rows], rtol=1e-13, atol=1e-13)
