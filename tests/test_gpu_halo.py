"""The spatial domain decomposition on one GPU (equivariant_graph_attention_b200/halo.py).

* egat_gather_rows against torch indexing, out-of-range indices giving zero
  rows.
* Two and three ranks emulated one after the other on one GPU: each rank's
  source coupling and attention run in the library on its local arrays, and
  the exchange is the same packing (egat_gather_rows of each owner's rows by
  the plan's send lists) without the all-to-all.  The owned outputs equal
  egat_forward of the whole system: the same rows and neighbour orders, so
  the float32 results agree to rounding.
"""
import numpy as np
import pytest
import torch

from equivariant_graph_attention_b200 import synth
from tests.parity_util import device_inputs, shape_of

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


@pytest.mark.parametrize("world", [2, 3])
def test_decomposed_forward_matches_single_gpu(world):
    from equivariant_graph_attention_b200 import egat, halo
    wl = synth.WORKLOADS["water216_l2_f32"]
    d = synth.make(wl)
    dev = device_inputs(wl, d)
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    shape = shape_of(wl)
    full = egat.egat_forward(shape, dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"], g["cnt"],
                             dev["w1"], dev["w2"], order=g["order"])
    nbr, cnt, order = (g[x].cpu().numpy() for x in ("nbr", "cnt", "order"))
    plans = [halo.build_plan(nbr, cnt, order, world, r) for r in range(world)]
    # every rank's coupled rows first (step 2), then each rank's local attention with
    # its halo rows packed from their owners by the plan's send lists
    hp_own, k_own = [], []
    for p in plans:
        own = torch.from_numpy(p.owned).cuda()
        s_own = egat.Shape(n=p.n_owned, lmax=wl.lmax, C=wl.C, H=wl.H, dk=wl.dk, K=wl.K, dtype=wl.dtype)
        hp_own.append(egat.egat_eaas_couple(s_own, dev["h"][own].contiguous(),
                                            dev["pos"][own].contiguous(), dev["w1"]))
        k_own.append(dev["k"][own].contiguous())
    got = torch.zeros_like(full)
    for r, p in enumerate(plans):
        halo_hp = [egat.egat_gather_rows(hp_own[s], torch.from_numpy(plans[s].send[r].astype(np.int32)).cuda())
                   for s in range(world) if s != r]
        halo_k = [egat.egat_gather_rows(k_own[s], torch.from_numpy(plans[s].send[r].astype(np.int32)).cuda())
                  for s in range(world) if s != r]
        hp_loc = torch.cat([hp_own[r]] + halo_hp)
        k_loc = torch.cat([k_own[r]] + halo_k)
        loc = torch.from_numpy(np.concatenate([p.owned, p.halo])).cuda()
        q_loc = torch.zeros((p.n_local, wl.H, wl.dk), dtype=dev["q"].dtype, device="cuda")
        q_loc[:p.n_owned] = dev["q"][loc[:p.n_owned]]
        s_loc = egat.Shape(n=p.n_local, lmax=wl.lmax, C=wl.C, H=wl.H, dk=wl.dk, K=wl.K, dtype=wl.dtype)
        out = egat.egat_otf_attention_coupled(s_loc, q_loc, k_loc, hp_loc,
                                              torch.from_numpy(p.local_nbr).cuda(),
                                              torch.from_numpy(p.local_cnt).cuda(),
                                              dev["pos"][loc].contiguous(), dev["w2"])
        got[loc[:p.n_owned]] = out[:p.n_owned]
    err = float(((got - full).norm(dim=(1, 2)) / full.norm(dim=(1, 2)).clamp_min(1e-30)).max())
    assert err < 1e-5
    assert egat.egat_take_device_status() == egat.EGAT_OK
