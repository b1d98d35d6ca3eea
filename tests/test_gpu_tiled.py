"""GPU parity of the tensor-core (tiled) attention path.

Pages: "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §3.1-§3.2.

* The attention plan (per tile of 16 targets: the sorted union of their
  neighbour lists and the membership bitmask) is rebuilt here with numpy and
  must match bit for bit.
* The tiled kernel's m (step 3) and ^h (steps 3+4) must match the oracle
  within the bf16 bar on every bf16 workload (sampled targets at full size),
  and on tiny ragged systems with isolated atoms, an atom at the origin and
  atoms on the z axis.
"""
import functools

import numpy as np
import pytest
import torch

from oracle.attention import aggregate, forward as oracle_forward
from oracle import so3
from oracle.graph import radius_graph
from equivariant_graph_attention_b200 import synth
from oracle.storage import round_bf16
from tests.parity_util import (FLOOR, ROUNDING_FLOOR, TOL, block_rel_error, channel_rel_error,
                               device_inputs, sample_targets, shape_of)

pytestmark = pytest.mark.gpu

BF16 = ["uniform4096_l2_bf16", "uniform32768_K256_l2_bf16", "uniform100000_l3_bf16"]
TILE = 16


def _egat():
    from equivariant_graph_attention_b200 import egat
    return egat


@functools.lru_cache(maxsize=None)
def _data(name):
    wl = synth.WORKLOADS[name]
    return wl, synth.make(wl)


def _plan_views(plan: torch.Tensor, n: int, K: int, lmax: int):
    tiles = (n + TILE - 1) // TILE
    cap = 32
    while cap < TILE * K:
        cap *= 2
    a256 = lambda x: (x + 255) // 256 * 256
    raw = plan.cpu().numpy().view(np.uint8)
    ulen = raw[:tiles * 4].view(np.int32)
    o = a256(tiles * 4)
    uni = raw[o:o + tiles * cap * 4].view(np.int32).reshape(tiles, cap)
    o += a256(tiles * cap * 4)
    mask = raw[o:o + tiles * TILE * (cap // 32) * 4].view(np.uint32).reshape(tiles, cap // 32, TILE)
    o += a256(tiles * TILE * (cap // 32) * 4)
    ws = sum((2 * l + 1) ** 2 for l in range(lmax + 1))
    rw = 4 + TILE * (1 + (lmax + 1) + ws)
    rec = raw[o:o + tiles * rw * 4].view(np.float32).reshape(tiles, rw)
    return ulen, uni, mask, rec


@pytest.mark.parametrize("name", ["uniform4096_l2_bf16", "uniform32768_K256_l2_bf16"])
def test_plan_matches_numpy(name):
    """Union, padding and membership bits rebuilt with numpy (bit for bit), and
    the tile records: target ids exactly, |r|^l and the Wigner-D blocks of the
    targets' alignment rotations against the oracle's (least-squares) D."""
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    shape = shape_of(wl)
    plan = egat.egat_build_attention_plan(shape, g["nbr"], g["cnt"], g["order"], dev["pos"])
    ulen, uni, mask, rec = _plan_views(plan, wl.n, wl.K, wl.lmax)
    nbr, cnt, order = g["nbr"].cpu().numpy(), g["cnt"].cpu().numpy(), g["order"].cpu().numpy()
    pos = dev["pos"].cpu().numpy().astype(np.float64)
    tiles = (wl.n + TILE - 1) // TILE
    ws = sum((2 * l + 1) ** 2 for l in range(wl.lmax + 1))
    pick = range(tiles) if tiles <= 256 else np.random.default_rng(3).choice(tiles, 64, replace=False)
    for t in pick:
        rows = order[t * TILE:(t + 1) * TILE]
        lists = [nbr[i, :cnt[i]] for i in rows]
        ref = np.unique(np.concatenate(lists)) if lists else np.zeros(0, np.int32)
        U = int(ulen[t])
        assert U == len(ref)
        assert np.array_equal(uni[t, :U], ref)
        upad = max(32, (U + 31) // 32 * 32)
        assert np.all(uni[t, U:upad] == (ref[0] if U else 0))
        for r, js in enumerate(lists):
            bits = np.zeros(upad, dtype=bool)
            bits[np.searchsorted(ref, js)] = True
            u = np.arange(upad)
            got = ((mask[t, u // 32, r] >> (u % 32).astype(np.uint32)) & 1).astype(bool)
            assert np.array_equal(got, bits), (t, r)
        # tile record: header (union length, zeros), ids, |r|^l, Wigner-D
        hdr = rec[t, :4].view(np.int32)
        assert hdr[0] == U and not hdr[1:].any()
        ids = rec[t, 4:4 + TILE].view(np.int32)
        want = np.full(TILE, -1, np.int32)
        want[:len(rows)] = rows
        assert np.array_equal(ids, want)
        rp = rec[t, 4 + TILE:4 + TILE * (wl.lmax + 2)].reshape(TILE, wl.lmax + 1)
        Dr = rec[t, 4 + TILE * (wl.lmax + 2):].reshape(TILE, ws)
        for r, a in enumerate(rows[:4]):
            rr = float(np.linalg.norm(pos[a]))
            assert np.allclose(rp[r], [rr ** l for l in range(wl.lmax + 1)], rtol=1e-5, atol=0)
            Q = so3.alignment_rotation(pos[a])
            off = 0
            for l in range(wl.lmax + 1):
                w = 2 * l + 1
                got = Dr[r, off:off + w * w].reshape(w, w)
                assert np.allclose(got, so3.wigner_D(l, Q), atol=2e-5), (t, r, l)
                off += w * w


@pytest.mark.parametrize("name", BF16)
def test_tiled_attention_parity(name):
    """Step 3 alone on a drawn value array (the same values on both sides)."""
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    vals = synth.round_bf16(np.random.default_rng(8).standard_normal((wl.n, wl.D, wl.C)).astype(np.float32))
    hp = torch.from_numpy(vals).to("cuda", dtype=torch.bfloat16)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    shape = shape_of(wl)
    plan = egat.egat_build_attention_plan(shape, g["nbr"], g["cnt"], g["order"], dev["pos"])
    m = egat.egat_otf_attention_tiled(shape, dev["q"], dev["k"], hp, plan, fused=False)
    rows = list(range(wl.n)) if wl.n <= 4096 else sample_targets(
        wl, np.minimum(g["cnt"].cpu().numpy(), wl.K))
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K, rows=rows)
    ref = aggregate(d["q"], d["k"], vals, lists, rows)
    got = m[torch.tensor(rows).cuda()].cpu().numpy()
    err = block_rel_error(got, ref, wl.lmax)
    e = channel_rel_error(got, ref, wl.lmax, FLOOR["bf16"])
    print(f"tiled m {name}: max block error {err:.2e}, per-channel {e:.2e}")
    assert err < TOL["bf16"] and e < TOL["bf16"]


@pytest.mark.parametrize("name", ["uniform4096_l2_bf16", "uniform32768_K256_l2_bf16"])
def test_tiled_relaunch_on_one_plan(name):
    """The kernel's CTAs claim tiles at run time from a counter kept in the
    plan (its last 256-byte block): repeated launches on one plan (m, then ^h
    twice, then m again) give bit-identical results, and each launch leaves
    the counter at zero."""
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    shape = shape_of(wl)
    hp = egat.egat_eaas_couple(shape, dev["h"], dev["pos"], dev["w1"])
    plan = egat.egat_build_attention_plan(shape, g["nbr"], g["cnt"], g["order"], dev["pos"])
    nb = egat.egat_attention_plan_bytes(shape)
    counter = lambda: int(plan[nb - 256:nb - 252].cpu().numpy().view(np.int32)[0])
    assert counter() == 0
    m0 = egat.egat_otf_attention_tiled(shape, dev["q"], dev["k"], hp, plan, fused=False)
    assert counter() == 0
    f0 = egat.egat_otf_attention_tiled(shape, dev["q"], dev["k"], hp, plan, w2=dev["w2"], fused=True)
    f1 = egat.egat_otf_attention_tiled(shape, dev["q"], dev["k"], hp, plan, w2=dev["w2"], fused=True)
    m1 = egat.egat_otf_attention_tiled(shape, dev["q"], dev["k"], hp, plan, fused=False)
    assert counter() == 0
    assert torch.equal(m0, m1) and torch.equal(f0, f1)
    assert egat.egat_take_device_status() == 0


@pytest.mark.parametrize("name", BF16)
def test_tiled_fused_matches_per_target_kernel(name):
    """^h from the tiled kernel and from the per-target kernel agree (both
    within the bf16 bar of the oracle, which test_forward_parity checks)."""
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    shape = shape_of(wl)
    hp = egat.egat_eaas_couple(shape, dev["h"], dev["pos"], dev["w1"])
    plan = egat.egat_build_attention_plan(shape, g["nbr"], g["cnt"], g["order"], dev["pos"])
    a = egat.egat_otf_attention_tiled(shape, dev["q"], dev["k"], hp, plan, w2=dev["w2"], fused=True)
    b = egat.egat_otf_attention_coupled(shape, dev["q"], dev["k"], hp, g["nbr"], g["cnt"],
                                        dev["pos"], dev["w2"], order=g["order"])
    err = block_rel_error(a.cpu().numpy(), b.cpu().numpy(), wl.lmax)
    print(f"tiled vs per-target ^h {name}: max block difference {err:.2e}")
    assert err < TOL["bf16"]


def test_per_target_fused_kernel_parity_bf16():
    """The per-target fused kernel (the path for shapes without tensor-core
    support) against the oracle on the 4,096-atom bf16 system."""
    egat = _egat()
    wl, d = _data("uniform4096_l2_bf16")
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    shape = shape_of(wl)
    hp = egat.egat_eaas_couple(shape, dev["h"], dev["pos"], dev["w1"])
    out = egat.egat_otf_attention_coupled(shape, dev["q"], dev["k"], hp, g["nbr"], g["cnt"],
                                          dev["pos"], dev["w2"], order=g["order"]).cpu().numpy()
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    ref = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists)
    assert block_rel_error(out, ref, wl.lmax) < TOL["bf16"]
    refs = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists,
                          store=round_bf16)
    assert channel_rel_error(out, refs, wl.lmax, floor=ROUNDING_FLOOR) < TOL["bf16"]


@pytest.mark.parametrize("lmax", [1, 2, 3])
@pytest.mark.parametrize("n", [1, 7, 37])
def test_tiled_edge_cases(lmax, n):
    """Ragged tiles, an isolated atom (zero output), an atom at the origin and
    atoms on both poles of the z axis, through egat_forward's tensor path."""
    egat = _egat()
    rng = np.random.default_rng(n + 10 * lmax)
    pts = rng.uniform(-3.0, 3.0, (n, 3))
    if n >= 4:
        pts[0] = 0.0
        pts[1] = [0.0, 0.0, -1.3]
        pts[2] = [0.0, 0.0, 1.1]
        pts[3] = [60.0, 60.0, 60.0]          # isolated
    wl = synth.small_cube(n, 6.0, 3.0, 16, lmax, 128, 16, 16, "bf16")
    feats = synth.features(wl, seed=n)
    pq = np.rint(pts / synth.GRID_QUANTUM).astype(np.int32)
    feats.update(pos_q=pq, pos=(pq.astype(np.float64) * synth.GRID_QUANTUM).astype(np.float32))
    dev = device_inputs(wl, feats)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    out = egat.egat_forward(shape_of(wl), dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"],
                            g["cnt"], dev["w1"], dev["w2"], order=g["order"]).cpu().numpy()
    lists, _ = radius_graph(feats["pos_q"], wl.cutoff_q, K=wl.K)
    ref = oracle_forward(feats["h"], feats["pos"], feats["q"], feats["k"], feats["w1"],
                         feats["w2"], lmax, lists)
    if n >= 4:
        assert np.all(out[3] == 0.0)
    assert block_rel_error(out, ref, lmax) < TOL["bf16"]
    refs = oracle_forward(feats["h"], feats["pos"], feats["q"], feats["k"], feats["w1"],
                          feats["w2"], lmax, lists, store=round_bf16)
    assert channel_rel_error(out, refs, lmax, floor=ROUNDING_FLOOR) < TOL["bf16"]
