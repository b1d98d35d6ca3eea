"""The spatial domain decomposition's host logic (equivariant_graph_attention_b200/halo.py)
on CPU ranks.

* Plan invariants on random systems and rank counts: every atom is owned
  once; a rank's halo is exactly the neighbours of its atoms that it does not
  own, grouped by owner; what rank p sends rank r is what r expects from p,
  in r's order; local neighbour lists map back to the global ones.
* The whole decomposed forward on two and three `gloo` ranks over 127.0.0.1:
  each rank couples its own atoms (oracle source coupling), exchanges the h'
  and k rows of its boundary atoms with `halo.exchange` (one all-to-all per
  array), and runs the oracle attention and target coupling on its local
  arrays.  The owned outputs equal the oracle forward of the whole system
  (fp64, 1e-12): the decomposition loses and duplicates nothing.
The per-rank kernels are the library's (tested on the GPU); here the oracle
stands in for them, so only the plan and the exchange protocol are under
test.
"""
import multiprocessing as mp
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _system(seed=0, n=90):
    sys.path.insert(0, ROOT)
    from equivariant_graph_attention_b200 import synth
    from oracle.graph import radius_graph
    wl = synth.small_cube(n, 9.0, 3.5, 12, 1, 16, 2, 8, "f32", name=f"halo{n}")
    d = synth.make(wl, seed=seed)
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    nbr = np.full((n, wl.K), -1, dtype=np.int32)
    cnt = np.zeros(n, dtype=np.int32)
    for i, js in enumerate(lists):
        nbr[i, :len(js)] = js
        cnt[i] = len(js)
    # a traversal order with spatial locality: cells of the cutoff, lexicographic
    cell = np.floor(d["pos"] / 3.5).astype(np.int64)
    order = np.lexsort((cell[:, 2], cell[:, 1], cell[:, 0])).astype(np.int64)
    return wl, d, lists, nbr, cnt, order


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_plan_invariants(world):
    from equivariant_graph_attention_b200 import halo
    wl, d, lists, nbr, cnt, order = _system(seed=world)
    n = wl.n
    plans = [halo.build_plan(nbr, cnt, order, world, r) for r in range(world)]
    owned = np.concatenate([p.owned for p in plans])
    assert np.array_equal(np.sort(owned), np.arange(n))
    owner = halo.owners(order, world)
    for p in plans:
        need = set()
        for i in p.owned:
            need |= set(int(j) for j in lists[i])
        expect = sorted(need - set(int(a) for a in p.owned))
        assert sorted(p.halo.tolist()) == expect
        assert np.all(np.diff(owner[p.halo]) >= 0)           # grouped by owner
        assert p.recv_counts == [int(np.sum(owner[p.halo] == r)) for r in range(world)]
        assert p.recv_counts[p.rank] == 0
        loc = np.concatenate([p.owned, p.halo])
        for t, i in enumerate(p.owned):
            row = p.local_nbr[t, :p.local_cnt[t]]
            assert np.array_equal(loc[row], np.asarray(lists[i]))
        assert not p.local_cnt[p.n_owned:].any()
    for r, pr in enumerate(plans):
        for s, ps in enumerate(plans):
            got = plans[s].owned[ps.send[r]] if r != s else np.zeros(0, dtype=np.int64)
            want = pr.halo[owner[pr.halo] == s]
            assert np.array_equal(got, want)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, ws: int, port: int, out):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from equivariant_graph_attention_b200 import halo
    from oracle.attention import aggregate, forward, source_coupling, tensor_product
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=ws, timeout=timedelta(seconds=60))
    try:
        wl, d, lists, nbr, cnt, order = _system(seed=7)
        plan = halo.build_plan(nbr, cnt, order, ws, rank)
        own = plan.owned
        pack = lambda rows, idx: rows.index_select(0, idx.long())
        hp_own = torch.from_numpy(source_coupling(d["h"][own], d["pos"][own], d["w1"], wl.lmax))
        k_own = torch.from_numpy(np.asarray(d["k"][own], dtype=np.float64))
        hp_loc = torch.cat([hp_own, halo.exchange(plan, hp_own, pack=pack)]).numpy()
        k_loc = torch.cat([k_own, halo.exchange(plan, k_own, pack=pack)]).numpy()
        q_loc = np.zeros((plan.n_local,) + d["q"].shape[1:])
        q_loc[:plan.n_owned] = d["q"][own]
        local_lists = [plan.local_nbr[t, :plan.local_cnt[t]] for t in range(plan.n_owned)]
        m = aggregate(q_loc, k_loc, hp_loc, local_lists, list(range(plan.n_owned)))
        got = tensor_product(m, d["pos"][own], d["w2"], wl.lmax)
        ref = forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax,
                      [lists[i] for i in own], targets=list(own))
        err = float(np.max(np.abs(got - ref))) if own.size else 0.0
        scale = float(np.max(np.abs(ref))) if own.size else 1.0
        dist.barrier()
        out.put((rank, (err, scale, int(plan.halo.size), int(plan.n_owned))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_decomposed_forward_on_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sum(v[3] for v in results.values()) == 90
    for r in range(world):
        err, scale, nh, _ = results[r]
        assert nh > 0                                  # the ranks do exchange rows
        assert err <= 1e-12 * max(1.0, scale)


def test_plan_edge_cases():
    """More ranks than atoms (empty blocks), no count array, isolated atoms."""
    from equivariant_graph_attention_b200 import halo
    nbr = np.array([[1, 2, -1], [0, -1, -1], [0, -1, -1], [-1, -1, -1], [3, -1, -1]], dtype=np.int32)
    cnt = np.array([2, 1, 1, 0, 1], dtype=np.int32)
    order = np.array([4, 3, 0, 1, 2])
    plans = [halo.build_plan(nbr, cnt, order, 8, r) for r in range(8)]
    assert sorted(np.concatenate([p.owned for p in plans]).tolist()) == [0, 1, 2, 3, 4]
    assert sum(p.n_owned == 0 for p in plans) == 3
    for p in plans:
        assert len(p.send) == 8 and len(p.recv_counts) == 8
        assert p.local_nbr.shape == (p.n_local, 3)
    # without a count array every slot is scanned and -1 entries are skipped:
    # rank 0 of 2 owns atoms 4 and 3 (slots 0, 1); atom 4 lists atom 3 (local 1)
    full = halo.build_plan(nbr, None, order, 2, 0)
    assert full.owned.tolist() == [4, 3] and full.halo.size == 0
    assert full.local_cnt.tolist() == [3, 3]
    assert full.local_nbr.tolist() == [[1, -1, -1], [-1, -1, -1]]
    # rank 1 owns atoms 0, 1, 2, which list only one another
    other = halo.build_plan(nbr, None, order, 2, 1)
    assert other.owned.tolist() == [0, 1, 2] and other.halo.size == 0
    assert other.send[0].size == 0 and other.recv_counts == [0, 0]
