"""The attention plan of a system past the bitmap builder's size (hash-set
builder, cost per tile independent of n), on a GPU.

175,616 atoms on a jittered simple-cubic lattice (2.2 Å spacing, jitter
U(±0.3 Å), seed 0), cutoff 3.0 Å, K = 16, lmax 2, bf16, C = 128, H = 16,
dk = 16: the union and membership mask of sampled tiles must equal numpy's
bit for bit (sorted union, padding, mask words), and the tiled forward must
match the oracle on sampled atoms within the bf16 bar (block and per-channel
metrics).
"""
import numpy as np
import pytest
import torch

from oracle.attention import forward as oracle_forward
from oracle.graph import radius_graph
from oracle.storage import round_bf16
from equivariant_graph_attention_b200 import synth
from tests.parity_util import (ROUNDING_FLOOR, TOL, block_rel_error, channel_rel_error,
                               device_inputs, shape_of)
from tests.test_gpu_tiled import TILE, _plan_views

pytestmark = pytest.mark.gpu

SIDE = 56            # atoms per lattice edge: 56^3 = 175,616 > 2^17


def _system():
    rng = np.random.default_rng(0)
    g = np.arange(SIDE, dtype=np.float64) * 2.2
    p = np.stack(np.meshgrid(g, g, g, indexing="ij"), axis=-1).reshape(-1, 3)
    p += rng.uniform(-0.3, 0.3, p.shape)
    p -= p.mean(axis=0)
    wl = synth.small_cube(len(p), SIDE * 2.2, 3.0, 16, 2, 128, 16, 16, "bf16", name="lattice175616")
    d = synth.features(wl, seed=0)
    pq = np.rint(p / synth.GRID_QUANTUM).astype(np.int32)
    d.update(pos_q=pq, pos=(pq.astype(np.float64) * synth.GRID_QUANTUM).astype(np.float32))
    return wl, d


def test_large_plan_matches_numpy_and_forward_matches_oracle():
    from equivariant_graph_attention_b200 import egat
    wl, d = _system()
    assert wl.n > 1 << 17
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    assert int(g["overflow"].item()) == 0
    shape = shape_of(wl)
    plan = egat.egat_build_attention_plan(shape, g["nbr"], g["cnt"], g["order"], dev["pos"])
    ulen, uni, mask, _ = _plan_views(plan, wl.n, wl.K, wl.lmax)
    nbr, cnt, order = g["nbr"].cpu().numpy(), g["cnt"].cpu().numpy(), g["order"].cpu().numpy()
    tiles = (wl.n + TILE - 1) // TILE
    pick = np.concatenate([np.random.default_rng(3).choice(tiles, 200, replace=False), [tiles - 1]])
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
    hp = egat.egat_eaas_couple_planned(shape, dev["h"], plan, dev["w1"])
    out = egat.egat_otf_attention_tiled(shape, dev["q"], dev["k"], hp, plan, dev["w2"], fused=True)
    rows = sorted(set(np.random.default_rng(5).choice(wl.n, 60, replace=False).tolist()) | {wl.n - 1})
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K, rows=rows)
    got = out[torch.tensor(rows).cuda()].cpu().numpy()
    ref = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists,
                         targets=rows)
    refs = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists,
                          targets=rows, store=round_bf16)
    e_block = block_rel_error(got, ref, wl.lmax)
    e_chan = channel_rel_error(got, refs, wl.lmax, ROUNDING_FLOOR)
    print(f"lattice {wl.n}: block {e_block:.2e} per-channel {e_chan:.2e}")
    assert e_block < TOL["bf16"] and e_chan < TOL["bf16"]
    assert egat.egat_take_device_status() == egat.EGAT_OK
