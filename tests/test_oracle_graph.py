"""Pins for the oracle's brute-force radius graph (CPU only).

"E2Former-V2：突破等变图神经网络计算瓶颈的创新架构" §5.1 (edge_cutoff) and
§5.2 (verify the neighbour list).  Checked against scipy's k-d tree (a
library routine), hand-built cases for the inclusive cutoff and the
(distance, index) tie rule, and the symmetry of an untruncated graph.
"""
import numpy as np
from scipy.spatial import cKDTree

from oracle.graph import radius_graph, neighbours_of
from equivariant_graph_attention_b200 import synth


def test_matches_kdtree_on_small_workloads():
    for name in ["uniform64_l1_f32", "water216_l2_f32"]:
        wl = synth.WORKLOADS[name]
        pq, _ = synth.positions(wl)
        lists, full = radius_graph(pq, wl.cutoff_q)
        tree = cKDTree(pq.astype(np.float64))
        ref = tree.query_ball_point(pq.astype(np.float64), wl.cutoff_q)
        for i, (got, exp) in enumerate(zip(lists, ref)):
            assert sorted(got.tolist()) == sorted(j for j in exp if j != i)
        # untruncated graph is symmetric
        adj = {(i, int(j)) for i, js in enumerate(lists) for j in js}
        assert all((j, i) in adj for (i, j) in adj)


def test_degree_statistics_uniform4096():
    wl = synth.WORKLOADS["uniform4096_l2_bf16"]
    pq, _ = synth.positions(wl)
    rows = np.arange(0, wl.n, 7)
    lists, full = radius_graph(pq, wl.cutoff_q, K=wl.K, rows=rows)
    tree = cKDTree(pq.astype(np.float64))
    cnt = np.array([len(x) - 1 for x in tree.query_ball_point(pq[rows].astype(np.float64),
                                                               wl.cutoff_q)])
    assert np.array_equal(full, cnt)
    assert all(len(l) == min(f, wl.K) for l, f in zip(lists, full))


def test_cutoff_is_inclusive_and_self_excluded():
    rc = 1000
    p = np.array([[0, 0, 0], [rc, 0, 0], [0, rc + 1, 0], [0, 0, -rc]], dtype=np.int32)
    assert neighbours_of(p, rc, 0).tolist() == [1, 3]
    # 3-4-5 triangle: exact integer distance at the cutoff
    p = np.array([[0, 0, 0], [600, 800, 0], [600, 801, 0]], dtype=np.int32)
    assert neighbours_of(p, rc, 0).tolist() == [1]


def test_truncation_keeps_nearest_then_smaller_index():
    a = 100
    p = np.array([[0, 0, 0],          # 0 centre
                  [0, 0, 3 * a],      # 1 far
                  [a, 0, 0],          # 2 d = a
                  [0, -a, 0],         # 3 d = a
                  [0, 0, 2 * a],      # 4 mid
                  [-a, 0, 0],         # 5 d = a
                  [0, a // 2, 0]],    # 6 nearest
                 dtype=np.int32)
    lists, full = radius_graph(p, 10 * a, K=3, rows=[0])
    assert full.tolist() == [6]
    assert lists[0].tolist() == [6, 2, 3]
    lists, _ = radius_graph(p, 10 * a, K=None, rows=[0])
    assert lists[0].tolist() == [6, 2, 3, 5, 4, 1]


def test_empty_and_isolated():
    p = np.array([[0, 0, 0], [10 ** 6, 0, 0]], dtype=np.int32)
    lists, full = radius_graph(p, 10, K=4)
    assert [l.tolist() for l in lists] == [[], []] and full.tolist() == [0, 0]
