"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Pages: [EX] "E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §2-§3, §5;
[TS] "E2Former-V2: On-the-Fly Equivariant Attention with Linear Activation
Memory" §2.

* Neighbour lists must match the oracle's brute force bit for bit after
  sorting each row (the library lists a row in cell-sweep order, the oracle
  by distance; the sets, the counts and the truncation set are unique), and
  two builds must give identical arrays (determinism).
* Floating-point outputs must match within the bars (1e-4 float32 storage,
  2e-2 bf16 storage) under the per-(atom, degree, channel) metric of
  ``parity_util`` (floor 1e-3 of the degree's RMS wherever both sides read
  identical inputs: step 2 alone, step 3 alone, steps 3+4 on a drawn value
  array), and under the per-(atom, degree) block metric.  The composed bf16
  forward is compared per channel with the oracle that stores h' in bf16 as
  the workload specifies, at the floor the bf16 rounding of h' allows.
* Small workloads are compared on every atom; the 32,768- and 100,000-atom
  workloads on a sample of targets that includes the truncated rows, in the
  same launch configuration the benchmark times (graph -> fused forward with
  the cell traversal order).
"""
import functools

import numpy as np
import pytest
import torch
from scipy.spatial import cKDTree

from oracle.attention import aggregate, forward as oracle_forward, source_coupling, target_coupling
from oracle.graph import radius_graph
from oracle.storage import round_bf16
from equivariant_graph_attention_b200 import synth
from tests.parity_util import (FLOOR, ROUNDING_FLOOR, TOL, block_rel_error, channel_rel_error,
                               device_inputs, sample_targets, shape_of)

pytestmark = pytest.mark.gpu

SMALL = ["uniform64_l1_f32", "water216_l2_f32", "uniform4096_l2_bf16"]
LARGE = ["uniform32768_K256_l2_bf16", "uniform100000_l3_bf16"]


@functools.lru_cache(maxsize=None)
def _data(name):
    wl = synth.WORKLOADS[name]
    return wl, synth.make(wl)


@functools.lru_cache(maxsize=None)
def _full_degree(name):
    wl, d = _data(name)
    tree = cKDTree(d["pos_q"].astype(np.float64))
    return np.array([len(x) - 1 for x in tree.query_ball_point(d["pos_q"].astype(np.float64),
                                                               wl.cutoff_q)])


def _egat():
    from equivariant_graph_attention_b200 import egat
    return egat


# --------------------------------------------------------------------------- graph
@pytest.mark.parametrize("name", SMALL)
def test_graph_padded_bit_exact(name):
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    nbr = g["nbr"].cpu().numpy()
    cnt = g["cnt"].cpu().numpy()
    lists, full = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    for i, ref in enumerate(lists):
        assert cnt[i] == len(ref)
        assert np.array_equal(np.sort(nbr[i, :cnt[i]]), np.sort(ref)), i
        assert np.all(nbr[i, cnt[i]:] == -1)
        if full[i] > wl.K:
            # a truncated row is listed nearest first, ties to the smaller index
            assert np.array_equal(nbr[i], ref), i
    assert int(g["overflow"].item()) == int(np.maximum(full - wl.K, 0).sum())
    order = g["order"].cpu().numpy()
    assert np.array_equal(np.sort(order), np.arange(wl.n))
    g2 = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    assert torch.equal(g["nbr"], g2["nbr"]) and torch.equal(g["order"], g2["order"])


@pytest.mark.parametrize("name", SMALL)
def test_graph_csr_bit_exact(name):
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    lists, full = radius_graph(d["pos_q"], wl.cutoff_q)
    E = int(full.sum())
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, mode="csr", col_capacity=E)
    rowptr = g["rowptr"].cpu().numpy()
    col = g["col"].cpu().numpy()
    assert rowptr[0] == 0 and rowptr[-1] == E
    for i, ref in enumerate(lists):
        assert np.array_equal(np.sort(col[rowptr[i]:rowptr[i + 1]]), np.sort(ref)), i
    assert int(g["overflow"].item()) == 0
    # a short column buffer reports exactly the entries it could not hold
    g2 = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, mode="csr", col_capacity=E - 5)
    assert int(g2["overflow"].item()) == 5
    assert np.array_equal(g2["col"].cpu().numpy(), col[:E - 5])


@pytest.mark.parametrize("name", LARGE)
def test_graph_full_size_sampled_rows(name):
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    nbr = g["nbr"].cpu().numpy()
    cnt = g["cnt"].cpu().numpy()
    full = _full_degree(name)
    assert np.array_equal(cnt, np.minimum(full, wl.K))
    assert int(g["overflow"].item()) == int(np.maximum(full - wl.K, 0).sum())
    rows = sample_targets(wl, full)
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K, rows=rows)
    for i, ref in zip(rows, lists):
        assert np.array_equal(np.sort(nbr[i, :cnt[i]]), np.sort(ref)), i
        if full[i] > wl.K:
            # a truncated row is listed nearest first, ties to the smaller index
            assert np.array_equal(nbr[i], ref), i
    # the sample covers truncated rows where there are any
    assert any(full[i] > wl.K for i in rows) or not np.any(full > wl.K)


@pytest.mark.parametrize("n", [300, 800, 1500])
def test_graph_dense_cluster_truncation(n):
    """Every atom within the cutoff of every other: each row keeps its K = 64
    nearest of n - 1, nearest first, ties (repeated positions) to the smaller
    index.  The three sizes put the rows' key counts in the three selection
    regimes of the padded builder: within the fill kernel's own key buffer,
    in the block-wide sort, and above the sort's capacity (bisection)."""
    egat = _egat()
    rng = np.random.default_rng(11)
    cutoff_q = 100_000
    pos = rng.integers(0, 50_000, size=(n, 3)).astype(np.int32)   # diameter < 86,603
    pos[n // 2:n // 2 + 20] = pos[:20]                              # repeated positions
    pos[-5:] = pos[7]
    K = 64
    g = egat.egat_build_graph(torch.from_numpy(pos).cuda(), cutoff_q, K=K)
    nbr = g["nbr"].cpu().numpy()
    cnt = g["cnt"].cpu().numpy()
    lists, full = radius_graph(pos, cutoff_q, K=K)
    assert np.all(full == n - 1) and np.all(cnt == K)
    for i, ref in enumerate(lists):
        assert np.array_equal(nbr[i], ref), i
    assert int(g["overflow"].item()) == n * (n - 1 - K)


# --------------------------------------------------------------------------- steps 2, 3
@pytest.mark.parametrize("name", SMALL + LARGE)
def test_eaas_couple_planned_parity(name):
    """Step 2 with the rotations taken from the attention plan's tile records
    (egat_eaas_couple_planned), against the oracle on every atom the sample
    covers; every atom of the system is written exactly once."""
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    shape = shape_of(wl)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    plan = egat.egat_build_attention_plan(shape, g["nbr"], g["cnt"], g["order"], dev["pos"])
    hp = torch.full_like(dev["h"], float("nan"))
    egat.egat_eaas_couple_planned(shape, dev["h"], plan, dev["w1"], out=hp)
    assert not torch.isnan(hp.float()).any()
    rows = np.arange(wl.n) if wl.n <= 4096 else np.array(sample_targets(wl, _full_degree(name), 300))
    ref = source_coupling(d["h"][rows], d["pos"][rows], d["w1"], wl.lmax)
    got = hp[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    assert block_rel_error(got, ref, wl.lmax) < TOL[wl.dtype]
    e = channel_rel_error(got, ref, wl.lmax, FLOOR[wl.dtype])
    print(f"eaas_couple_planned {name}: per-channel {e:.2e}")
    assert e < TOL[wl.dtype]


@pytest.mark.parametrize("name", SMALL + LARGE)
def test_eaas_couple_parity(name):
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    hp = egat.egat_eaas_couple(shape_of(wl), dev["h"], dev["pos"], dev["w1"])
    rows = np.arange(wl.n) if wl.n <= 4096 else np.array(sample_targets(wl, _full_degree(name), 300))
    ref = source_coupling(d["h"][rows], d["pos"][rows], d["w1"], wl.lmax)
    got = hp[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    assert block_rel_error(got, ref, wl.lmax) < TOL[wl.dtype]
    e = channel_rel_error(got, ref, wl.lmax, FLOOR[wl.dtype])
    print(f"eaas_couple {name}: per-channel {e:.2e}")
    assert e < TOL[wl.dtype]


@pytest.mark.parametrize("name", SMALL + LARGE)
def test_otf_attention_parity(name):
    """Step 3 alone, on a value array drawn directly (the same values on both sides)."""
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    rng = np.random.default_rng(8)
    vals = rng.standard_normal((wl.n, wl.D, wl.C)).astype(np.float32)
    if wl.dtype == "bf16":
        vals = synth.round_bf16(vals)
    hp = torch.from_numpy(vals).to("cuda", dtype=dev["h"].dtype)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    m = egat.egat_otf_attention(shape_of(wl), dev["q"], dev["k"], hp, g["nbr"], g["cnt"],
                                order=g["order"])
    rows = list(range(wl.n)) if wl.n <= 4096 else sample_targets(wl, _full_degree(name))
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K, rows=rows)
    ref = aggregate(d["q"], d["k"], vals, lists, rows)
    got = m[torch.tensor(rows).cuda()].cpu().numpy()
    # inputs identical on both sides: only float32 accumulation differs
    assert block_rel_error(got, ref, wl.lmax) < 1e-4
    e = channel_rel_error(got, ref, wl.lmax, FLOOR["f32"])
    print(f"otf_attention {name}: per-channel {e:.2e}")
    assert e < 1e-4


@pytest.mark.parametrize("name", SMALL + LARGE)
def test_fused_attention_parity(name):
    """Steps 3+4 alone (the per-target kernel with the target coupling fused,
    and on bf16 shapes the tiled tensor-core kernel) on a value array drawn
    directly: identical inputs on both sides, so the per-channel metric at the
    identical-input floor applies.  The per-target kernel keeps float32
    throughout; the tiled kernel multiplies the softmax weights as bf16 pairs
    hi + lo.  Both at the workload's bar."""
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    vals = np.random.default_rng(8).standard_normal((wl.n, wl.D, wl.C)).astype(np.float32)
    if wl.dtype == "bf16":
        vals = synth.round_bf16(vals)
    hp = torch.from_numpy(vals).to("cuda", dtype=dev["h"].dtype)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    shape = shape_of(wl)
    outs = {"per-target": egat.egat_otf_attention_coupled(shape, dev["q"], dev["k"], hp, g["nbr"],
                                                          g["cnt"], dev["pos"], dev["w2"],
                                                          order=g["order"])}
    if egat.tc_attention_shape(shape):
        plan = egat.egat_build_attention_plan(shape, g["nbr"], g["cnt"], g["order"], dev["pos"])
        outs["tiled"] = egat.egat_otf_attention_tiled(shape, dev["q"], dev["k"], hp, plan,
                                                      dev["w2"], fused=True)
    rows = list(range(wl.n)) if wl.n <= 4096 else sample_targets(wl, _full_degree(name))
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K, rows=rows)
    ref = target_coupling(aggregate(d["q"], d["k"], vals, lists, rows), d["pos"][rows], d["w2"],
                          wl.lmax)
    idx = torch.tensor(rows).cuda()
    for kind, out in outs.items():
        got = out[idx].cpu().numpy()
        e = channel_rel_error(got, ref, wl.lmax, FLOOR[wl.dtype])
        print(f"fused attention {name} {kind}: per-channel {e:.2e}")
        assert e < TOL[wl.dtype]
    assert egat.egat_take_device_status() == egat.EGAT_OK


# --------------------------------------------------------------------------- fused forward
def _forward_case(name, mode="padded", use_order=True):
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    if mode == "padded":
        g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
        shape = shape_of(wl)
        a, b = g["nbr"], g["cnt"]
    else:
        E = int(_full_degree(name).sum()) if wl.n > 4096 else int(
            radius_graph(d["pos_q"], wl.cutoff_q)[1].sum())
        g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, mode="csr", col_capacity=E)
        shape = shape_of(wl, mode="csr", n_edges=E)
        a, b = g["rowptr"], g["col"]
    out = egat.egat_forward(shape, dev["h"], dev["pos"], dev["q"], dev["k"], a, b,
                            dev["w1"], dev["w2"], order=g["order"] if use_order else None)
    torch.cuda.synchronize()
    return wl, d, out


@pytest.mark.parametrize("name", SMALL + LARGE)
def test_forward_parity(name):
    wl, d, out = _forward_case(name)
    if wl.n <= 4096:
        rows = list(range(wl.n))
    else:
        rows = sample_targets(wl, _full_degree(name))
    K = wl.K
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=K, rows=rows)
    ref = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists,
                         targets=rows)
    got = out[torch.tensor(rows).cuda()].cpu().numpy()
    err = block_rel_error(got, ref, wl.lmax)
    assert err < TOL[wl.dtype], err
    e = composed_channel_error(wl, d, got, lists, rows)
    print(f"forward {name}: block {err:.2e} per-channel {e:.2e}")
    assert e < TOL[wl.dtype]


def composed_channel_error(wl, d, got, lists, rows):
    """Per-channel error of the composed forward: float32 storage against the
    float64 oracle at the float32 floor; bf16 storage against the oracle that
    stores h' in bf16, at the rounding floor (parity_util)."""
    if wl.dtype == "f32":
        ref = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists,
                             targets=rows)
        return channel_rel_error(got, ref, wl.lmax, FLOOR["f32"])
    ref = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists,
                         targets=rows, store=round_bf16)
    return channel_rel_error(got, ref, wl.lmax, ROUNDING_FLOOR)


@pytest.mark.parametrize("name", ["water216_l2_f32", "uniform4096_l2_bf16"])
def test_csr_matches_padded_without_truncation(name):
    """The per-target kernel gives bit-identical results from a CSR list and a
    padded list of the same rows; the forward pass (which may take the
    tensor-core path for the padded list) agrees within the storage bar."""
    egat = _egat()
    wl, d = _data(name)
    dev = device_inputs(wl, d)
    full = radius_graph(d["pos_q"], wl.cutoff_q)[1]
    E = int(full.sum())
    gp = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    gc = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, mode="csr", col_capacity=E)
    hp = egat.egat_eaas_couple(shape_of(wl), dev["h"], dev["pos"], dev["w1"])
    a = egat.egat_otf_attention_coupled(shape_of(wl), dev["q"], dev["k"], hp, gp["nbr"],
                                        gp["cnt"], dev["pos"], dev["w2"], order=gp["order"])
    b = egat.egat_otf_attention_coupled(shape_of(wl, mode="csr", n_edges=E), dev["q"], dev["k"],
                                        hp, gc["rowptr"], gc["col"], dev["pos"], dev["w2"],
                                        order=gc["order"])
    keep = full <= wl.K     # rows the padded list did not truncate
    assert np.array_equal(a.cpu().numpy()[keep], b.cpu().numpy()[keep])
    _, _, out_p = _forward_case(name, "padded")
    _, _, out_c = _forward_case(name, "csr")
    assert block_rel_error(out_p.cpu().numpy()[keep], out_c.cpu().numpy()[keep], wl.lmax) < TOL[wl.dtype]


def test_traversal_order_does_not_change_per_target_results():
    """Per-target kernel: the traversal order only schedules work (bitwise
    identical results).  Tiled kernel: the order decides which targets share a
    tile, which changes rounding only (agreement within the bf16 bar)."""
    egat = _egat()
    wl, d = _data("uniform4096_l2_bf16")
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    hp = egat.egat_eaas_couple(shape_of(wl), dev["h"], dev["pos"], dev["w1"])
    a = egat.egat_otf_attention_coupled(shape_of(wl), dev["q"], dev["k"], hp, g["nbr"], g["cnt"],
                                        dev["pos"], dev["w2"], order=g["order"])
    b = egat.egat_otf_attention_coupled(shape_of(wl), dev["q"], dev["k"], hp, g["nbr"], g["cnt"],
                                        dev["pos"], dev["w2"], order=None)
    assert torch.equal(a, b)
    _, _, x = _forward_case("uniform4096_l2_bf16", use_order=True)
    _, _, y = _forward_case("uniform4096_l2_bf16", use_order=False)
    assert block_rel_error(x.cpu().numpy(), y.cpu().numpy(), wl.lmax) < TOL[wl.dtype]


# --------------------------------------------------------------------------- edge cases
def _tiny_problem(pos_list, lmax=2, C=16, H=2, dk=8, K=8, dtype="f32", cutoff=3.0, seed=4):
    wl = synth.small_cube(len(pos_list), 1.0, cutoff, K, lmax, C, H, dk, dtype)
    feats = synth.features(wl, seed)
    pq = np.rint(np.asarray(pos_list, dtype=np.float64) / synth.GRID_QUANTUM).astype(np.int32)
    pf = (pq.astype(np.float64) * synth.GRID_QUANTUM).astype(np.float32)
    feats.update(pos_q=pq, pos=pf)
    return wl, feats


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_special_geometry_and_isolated_atoms(lmax, dtype):
    """Atoms at the origin (r = 0), on the -z and +z axes, an isolated atom
    (no neighbours -> exactly zero output), and a ragged count of atoms."""
    egat = _egat()
    pts = [[0, 0, 0], [0, 0, -1.2], [0, 0, 1.1], [0.7, -0.4, 0.2], [-0.5, 0.9, -0.8],
           [40.0, 40.0, 40.0], [1.3, 0.2, -0.1]]
    wl, d = _tiny_problem(pts, lmax=lmax, dtype=dtype)
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    out = egat.egat_forward(shape_of(wl), dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"],
                            g["cnt"], dev["w1"], dev["w2"], order=g["order"]).cpu().numpy()
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    assert len(lists[5]) == 0
    ref = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], lmax, lists)
    assert np.all(out[5] == 0.0)
    assert block_rel_error(out, ref, lmax) < TOL[dtype]
    assert composed_channel_error(wl, d, out, lists, list(range(wl.n))) < TOL[dtype]


@pytest.mark.parametrize("n", [1, 5, 37, 301])
def test_ragged_sizes_and_no_count_array(n):
    """Sizes that leave partial warps/tiles; the padded list scanned without
    the count array (slots marked -1 are skipped)."""
    egat = _egat()
    wl = synth.small_cube(n, max(3.0, (n / 0.1) ** (1 / 3)), 4.0, 32, 2, 32, 4, 8, "f32")
    d = synth.make(wl, seed=n)
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    shape = shape_of(wl)
    out = egat.egat_forward(shape, dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"], None,
                            dev["w1"], dev["w2"]).cpu().numpy()
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    ref = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists)
    assert block_rel_error(out, ref, wl.lmax) < 1e-4
    assert channel_rel_error(out, ref, wl.lmax, FLOOR["f32"]) < 1e-4


def test_golden_tiny_forward():
    """The stored oracle output for the tiny seeded system (tests/golden)."""
    import json
    import os
    from tests.golden.make_golden import SPEC
    egat = _egat()
    with open(os.path.join(os.path.dirname(__file__), "golden", "forward_tiny.json")) as f:
        rec = json.load(f)
    s = SPEC
    wl = synth.small_cube(s["n"], s["side"], s["cutoff"], s["K"], s["lmax"], s["C"], s["H"],
                          s["dk"], s["dtype"])
    d = synth.make(wl, s["seed"])
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    cnt = g["cnt"].cpu().numpy()
    nbr = g["nbr"].cpu().numpy()
    assert [sorted(nbr[i, :cnt[i]].tolist()) for i in range(wl.n)] == [
        sorted(r) for r in rec["neighbours"]]
    out = egat.egat_forward(shape_of(wl), dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"],
                            g["cnt"], dev["w1"], dev["w2"], order=g["order"]).cpu().numpy()
    assert block_rel_error(out, np.array(rec["out"]), wl.lmax) < 1e-4
    assert channel_rel_error(out, np.array(rec["out"]), wl.lmax, FLOOR["f32"]) < 1e-4


def test_empty_input_is_a_noop():
    egat = _egat()
    wl = synth.small_cube(0, 1.0, 1.0, 4, 1, 16, 2, 8)
    shape = shape_of(wl, n=0)
    z = torch.zeros(16, device="cuda")
    pos_q = torch.zeros((0, 3), dtype=torch.int32, device="cuda")
    g = egat.egat_build_graph(pos_q, wl.cutoff_q, K=4)
    assert int(g["overflow"].item()) == 0
    out = egat.egat_forward(shape, z, z, z, z, z.int(), z.int(), z, z, workspace=torch.zeros(
        256, dtype=torch.uint8, device="cuda"))
    assert out.shape == (0, 4, 16)


def test_error_codes_from_the_device_path():
    egat = _egat()
    wl, d = _data("uniform64_l1_f32")
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    with pytest.raises(egat.EgatError) as e:
        egat.egat_forward(shape_of(wl), dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"], g["cnt"],
                          dev["w1"], dev["w2"], workspace=torch.zeros(256, dtype=torch.uint8,
                                                                      device="cuda"))
    assert e.value.code == egat.EGAT_ERR_WORKSPACE
    with pytest.raises(egat.EgatError) as e:
        egat.egat_forward(shape_of(wl), dev["h"].reshape(-1)[1:], dev["pos"], dev["q"], dev["k"],
                          g["nbr"], g["cnt"], dev["w1"], dev["w2"])
    assert e.value.code == egat.EGAT_ERR_ARG     # misaligned feature pointer
    torch.cuda.synchronize()
