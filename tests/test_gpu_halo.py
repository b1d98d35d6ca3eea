"""The spatial domain decomposition on one GPU (equivariant_graph_attention_b200/halo.py).

* egat_gather_rows against torch indexing, out-of-range indices giving zero
  rows.
* forward_rank whole (couple -> exchange -> attend) in a world-size-1 NCCL
  group: the NCCL all-to-all path with empty halos; equal to the oracle
  forward of the whole system on sampled atoms.
* Two and three ranks emulated one after the other on one GPU: every rank's
  couple_rank, then each rank's attend_rank with the halo rows its owners'
  exchange() packed for it (the same packing as between GPUs; only the
  all-to-all transport is replaced by slicing the owners' send buffers).
  The stitched outputs equal the ORACLE forward of the whole system: the
  per-target path (float32) and the tensor-core path (bf16) on local arrays.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch

from oracle.attention import forward as oracle_forward
from oracle.graph import radius_graph
from oracle.storage import round_bf16
from equivariant_graph_attention_b200 import synth
from tests.parity_util import (FLOOR, ROUNDING_FLOOR, TOL, block_rel_error,
                               channel_rel_error, device_inputs, sample_targets, shape_of)

pytestmark = pytest.mark.gpu


def test_gather_rows():
    from equivariant_graph_attention_b200 import egat
    src = torch.randn((50, 9, 16), device="cuda")
    idx = torch.tensor([3, 0, 49, 50, -1, 7, 7], dtype=torch.int32, device="cuda")
    out = egat.egat_gather_rows(src, idx)
    want = torch.zeros_like(out)
    ok = (idx >= 0) & (idx < 50)
    want[ok] = src[idx[ok].long()]
    assert torch.equal(out, want)


def _oracle_check(wl, d, got, rows):
    """got [len(rows), D, C] against the oracle forward at those atoms."""
    lists, _ = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K, rows=rows)
    ref = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists,
                         targets=rows)
    e_block = block_rel_error(got, ref, wl.lmax)
    if wl.dtype == "bf16":
        refs = oracle_forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, lists,
                              targets=rows, store=round_bf16)
        e_chan = channel_rel_error(got, refs, wl.lmax, floor=ROUNDING_FLOOR)
    else:
        e_chan = channel_rel_error(got, ref, wl.lmax, floor=FLOOR["f32"])
    return e_block, e_chan


def _setup(name):
    from equivariant_graph_attention_b200 import egat
    wl = synth.WORKLOADS[name]
    d = synth.make(wl)
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    nbr, cnt, order = (g[x].cpu().numpy() for x in ("nbr", "cnt", "order"))
    return wl, d, dev, nbr, cnt, order


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("name", ["water216_l2_f32", "uniform4096_l2_bf16"])
def test_forward_rank_in_a_one_rank_nccl_group(name):
    import torch.distributed as dist
    from equivariant_graph_attention_b200 import egat, halo
    wl, d, dev, nbr, cnt, order = _setup(name)
    plan = halo.build_plan(nbr, cnt, order, 1, 0)
    assert plan.halo.size == 0 and plan.n_owned == wl.n
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        out = halo.forward_rank(plan, shape_of(wl), dev["h"], dev["pos"], dev["q"], dev["k"],
                                dev["w1"], dev["w2"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    got = np.zeros((wl.n, wl.D, wl.C), dtype=np.float32)
    got[plan.owned] = out.cpu().numpy()
    rows = list(range(0, wl.n, max(1, wl.n // 300)))
    e_block, e_chan = _oracle_check(wl, d, got[rows], rows)
    print(f"forward_rank world 1 {name}: block {e_block:.2e} channel {e_chan:.2e}")
    assert e_block < TOL[wl.dtype] and e_chan < TOL[wl.dtype]
    assert egat.egat_take_device_status() == egat.EGAT_OK


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("name", ["water216_l2_f32", "uniform4096_l2_bf16"])
def test_decomposed_forward_matches_oracle(world, name):
    from equivariant_graph_attention_b200 import egat, halo
    wl, d, dev, nbr, cnt, order = _setup(name)
    shape = shape_of(wl)
    plans = [halo.build_plan(nbr, cnt, order, world, r) for r in range(world)]
    states = [halo.couple_rank(p, shape, dev["h"], dev["pos"], dev["q"], dev["k"], dev["w1"])
              for p in plans]

    # each owner's send buffers as exchange() packs them, by destination rank
    def packed(field):
        bufs = []
        for p, st in zip(plans, states):
            cap = {}

            def transport(send_buf, in_splits, out_splits, cap=cap):
                cap["buf"], cap["splits"] = send_buf, in_splits
                return torch.empty((sum(out_splits),) + tuple(send_buf.shape[1:]),
                                   dtype=send_buf.dtype, device=send_buf.device)
            halo.exchange(p, getattr(st, field), transport=transport)
            offs = np.concatenate([[0], np.cumsum(cap["splits"])])
            bufs.append([cap["buf"][offs[r]:offs[r + 1]] for r in range(world)])
        return bufs

    hp_bufs, k_bufs = packed("hp_own"), packed("k_own")
    got = np.zeros((wl.n, wl.D, wl.C), dtype=np.float32)
    for r, (p, st) in enumerate(zip(plans, states)):
        # what an all-to-all delivers to rank r: the owners' chunks in rank order
        hp_halo = torch.cat([hp_bufs[s][r] for s in range(world)])
        k_halo = torch.cat([k_bufs[s][r] for s in range(world)])
        assert hp_halo.shape[0] == p.halo.size
        got[p.owned] = halo.attend_rank(p, shape, st, hp_halo, k_halo, dev["w2"]).cpu().numpy()
    assert all(p.halo.size > 0 for p in plans)
    rows = list(range(wl.n)) if wl.n <= 700 else sample_targets(wl, cnt, count=120)
    e_block, e_chan = _oracle_check(wl, d, got[rows], rows)
    print(f"decomposed {world} ranks {name}: block {e_block:.2e} channel {e_chan:.2e}")
    assert e_block < TOL[wl.dtype] and e_chan < TOL[wl.dtype]
    assert egat.egat_take_device_status() == egat.EGAT_OK
