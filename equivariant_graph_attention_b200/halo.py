"""Spatial domain decomposition with one halo exchange per step.

One GPU reaches systems of about 10^5 atoms ("E2Former-V2：突破等变图神经网络
计算瓶颈的创新架构" §3.2).  Past that, the atoms are split into contiguous
blocks of the graph builder's traversal order (cells in Morton order, so a
block is spatially compact), one block per rank.  Each step, rank r

1. couples its own atoms at the source (step 2) with the library;
2. packs the h' and k rows that other ranks need (``egat_gather_rows``) and
   exchanges them in one all-to-all per array (NCCL over NVLink between GPUs);
3. runs steps 3+4 for its own atoms over local arrays: its own rows first,
   then the received halo rows (halo atoms appear only as sources, with empty
   neighbour lists, so their outputs are zero and discarded).

The plan (who owns what, which rows go where) is host logic computed once per
neighbour list from the global padded lists, which every rank can build from
the replicated positions (12 bytes per atom).  The only data-path collective
is the exchange of step 2; the forward needs nothing else from other ranks.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable, Dict, List, Optional

import numpy as np
import torch

from . import egat


@dataclass
class HaloPlan:
    rank: int
    world: int
    owned: np.ndarray          # int64 global ids of this rank's atoms, in traversal order
    halo: np.ndarray           # int64 global ids of the halo, grouped by owning rank, ascending within
    recv_counts: List[int]     # per rank: halo atoms owned by it (0 for this rank)
    send: List[np.ndarray]     # per rank: local indices (into owned) of the rows it receives from us
    local_nbr: np.ndarray      # int32 [n_owned + n_halo, K]: owned rows in local indices, halo rows -1
    local_cnt: np.ndarray      # int32 [n_owned + n_halo]
    _dev: Dict[str, Dict[str, torch.Tensor]] = field(default_factory=dict, repr=False)

    @property
    def n_owned(self) -> int:
        return int(self.owned.size)

    def on(self, device) -> Dict[str, torch.Tensor]:
        """The plan's index arrays on `device`, copied once and kept: owned ids
        (int32), local ids (owned then halo, int64), the concatenated send lists
        (int32), the local lists and counts, and the local traversal order."""
        key = str(device)
        if key not in self._dev:
            t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dt)
            self._dev[key] = {
                "own": t(self.owned, torch.int32),
                "loc": t(np.concatenate([self.owned, self.halo]), torch.int64),
                "send": t(np.concatenate(self.send) if self.send else np.zeros(0), torch.int32),
                "nbr": t(self.local_nbr, torch.int32),
                "cnt": t(self.local_cnt, torch.int32),
                "order": torch.arange(self.n_local, dtype=torch.int32, device=device),
            }
        return self._dev[key]

    @property
    def n_local(self) -> int:
        return int(self.owned.size + self.halo.size)


def owners(order: np.ndarray, world: int) -> np.ndarray:
    """Owning rank of every atom: rank r holds slots [r n / world, (r+1) n / world) of
    the traversal order."""
    order = np.asarray(order, dtype=np.int64)
    n = order.size
    owner = np.empty(n, dtype=np.int64)
    for r in range(world):
        owner[order[r * n // world:(r + 1) * n // world]] = r
    return owner


def _needed(nbr: np.ndarray, cnt: np.ndarray, targets: np.ndarray) -> np.ndarray:
    """Distinct neighbours (global ids) of the given targets."""
    n, K = nbr.shape
    rows = nbr[targets]
    c = np.clip(cnt[targets], 0, K)
    valid = (np.arange(K)[None, :] < c[:, None]) & (rows >= 0) & (rows < n)
    return np.unique(rows[valid].astype(np.int64))


def build_plan(nbr: np.ndarray, cnt: Optional[np.ndarray], order: np.ndarray, world: int,
               rank: int) -> HaloPlan:
    """The halo plan of `rank` from the global padded lists (nbr [n, K], cnt [n] or
    None for full rows) and the traversal order."""
    nbr = np.asarray(nbr)
    n, K = nbr.shape
    cnt = np.full(n, K, dtype=np.int64) if cnt is None else np.asarray(cnt, dtype=np.int64)
    order = np.asarray(order, dtype=np.int64)
    owner = owners(order, world)
    blocks = [order[r * n // world:(r + 1) * n // world] for r in range(world)]
    owned = blocks[rank]

    def halo_of(r: int) -> np.ndarray:
        need = _needed(nbr, cnt, blocks[r])
        need = need[owner[need] != r]
        return need[np.lexsort((need, owner[need]))]      # by owning rank, then id

    halo = halo_of(rank)
    local_of = np.full(n, -1, dtype=np.int64)
    local_of[owned] = np.arange(owned.size)
    local_of[halo] = owned.size + np.arange(halo.size)
    rows = nbr[owned].astype(np.int64)
    c = np.clip(cnt[owned], 0, K)
    valid = (np.arange(K)[None, :] < c[:, None]) & (rows >= 0) & (rows < n)
    local_nbr = np.full((owned.size + halo.size, K), -1, dtype=np.int32)
    local_nbr[:owned.size] = np.where(valid, local_of[np.where(valid, rows, 0)], -1)
    local_cnt = np.zeros(owned.size + halo.size, dtype=np.int32)
    local_cnt[:owned.size] = c
    recv_counts = [int(np.sum(owner[halo] == p)) for p in range(world)]
    send = []
    for p in range(world):
        if p == rank:
            send.append(np.zeros(0, dtype=np.int64))
            continue
        theirs = halo_of(p)
        mine = theirs[owner[theirs] == rank]               # ascending id: their receive order
        send.append(local_of[mine])
    return HaloPlan(rank, world, owned, halo, recv_counts, send, local_nbr, local_cnt)


def exchange(plan: HaloPlan, own_rows: torch.Tensor, group=None,
             pack: Optional[Callable[[torch.Tensor, torch.Tensor], torch.Tensor]] = None,
             transport: Optional[Callable] = None) -> torch.Tensor:
    """Rows of the halo atoms (in plan.halo order) from their owners, given this
    rank's own rows [n_owned, ...]: the send buffer is packed on the device
    (egat_gather_rows, grouped by destination rank) and one all-to-all moves it.
    `pack(rows, idx)` replaces the device packing (tests on CPU ranks);
    `transport(send_buf, in_splits, out_splits)` replaces the all-to-all (one
    GPU standing in for several ranks, one after the other)."""
    dev = own_rows.device
    if own_rows.is_cuda:
        send_idx = plan.on(dev)["send"]
    else:
        send_idx = torch.from_numpy(np.concatenate(plan.send).astype(np.int32))
    if pack is None:
        if not own_rows.is_cuda:
            raise RuntimeError("exchange packs rows on the GPU; pass `pack` for CPU tensors")
        send_buf = egat.egat_gather_rows(own_rows.contiguous(), send_idx)
    else:
        send_buf = pack(own_rows, send_idx)
    in_splits = [int(s.size) for s in plan.send]
    out_splits = list(plan.recv_counts)
    if transport is not None:
        return transport(send_buf, in_splits, out_splits)
    import torch.distributed as dist
    recv = torch.empty((sum(out_splits),) + tuple(own_rows.shape[1:]), dtype=own_rows.dtype,
                       device=dev)
    dist.all_to_all_single(recv, send_buf, output_split_sizes=out_splits,
                           input_split_sizes=in_splits, group=group)
    return recv


@dataclass
class RankState:
    """One rank's device arrays for a step: its own coupled rows and keys, its
    own queries, and the positions of its local atoms (owned, then halo)."""
    hp_own: torch.Tensor
    k_own: torch.Tensor
    q_own: torch.Tensor
    pos_loc: torch.Tensor


def _local_shape(shape: "egat.Shape", n: int) -> "egat.Shape":
    return egat.Shape(n=n, lmax=shape.lmax, C=shape.C, H=shape.H, dk=shape.dk, K=shape.K,
                      dtype=shape.dtype)


def couple_rank(plan: HaloPlan, shape: "egat.Shape", h: torch.Tensor, pos: torch.Tensor,
                q: torch.Tensor, k: torch.Tensor, w1: torch.Tensor,
                own_rows: bool = False) -> RankState:
    """Step 2 for this rank's own atoms (egat_eaas_couple on its rows of h); each
    rank reads only its own rows of h, q and k and the positions of its local
    atoms.  h, q, k are the whole system's arrays, or (own_rows) already this
    rank's rows in plan.owned order; pos is always the whole system's."""
    a = plan.on(h.device)
    own_i32, loc = a["own"], a["loc"]
    if own_rows:
        h_own, q_own, k_own = h.contiguous(), q.contiguous(), k.contiguous()
    else:
        h_own = egat.egat_gather_rows(h.contiguous(), own_i32)
        q_own = egat.egat_gather_rows(q.contiguous(), own_i32)
        k_own = egat.egat_gather_rows(k.contiguous(), own_i32)
    pos_loc = pos.index_select(0, loc).contiguous()
    hp_own = egat.egat_eaas_couple(_local_shape(shape, plan.n_owned), h_own,
                                   pos_loc[:plan.n_owned].contiguous(), w1)
    return RankState(hp_own, k_own, q_own, pos_loc)


def attend_rank(plan: HaloPlan, shape: "egat.Shape", st: RankState, hp_halo: torch.Tensor,
                k_halo: torch.Tensor, w2: torch.Tensor) -> torch.Tensor:
    """Steps 3+4 for this rank's own atoms over its local arrays (own rows, then
    the halo rows received): ^h float32 [n_owned, D, C] in plan.owned order.

    The local system lists the owned atoms first, in the global traversal
    order (a spatially compact block), then the halo atoms, which appear only
    as sources (empty lists).  Shapes of the tensor-core path build the
    attention plan over the local arrays and run the tiled kernel; its tiles of
    halo slots have empty unions and only write zero rows, which are dropped.
    Other shapes run the per-target kernel."""
    dev = st.hp_own.device
    n_loc = plan.n_local
    hp_loc = torch.cat([st.hp_own, hp_halo])
    k_loc = torch.cat([st.k_own, k_halo])
    q_loc = torch.cat([st.q_own, torch.zeros((n_loc - plan.n_owned,) + tuple(st.q_own.shape[1:]),
                                             dtype=st.q_own.dtype, device=dev)])
    a = plan.on(dev)
    nbr, cnt = a["nbr"], a["cnt"]
    s_loc = _local_shape(shape, n_loc)
    if n_loc == 0:
        return torch.zeros((0, s_loc.D, shape.C), dtype=torch.float32, device=dev)
    if egat.tc_attention_shape(s_loc):
        try:
            ap = egat.egat_build_attention_plan(s_loc, nbr, cnt, a["order"], st.pos_loc)
            out = egat.egat_otf_attention_tiled(s_loc, q_loc, k_loc, hp_loc, ap, w2, fused=True)
            return out[:plan.n_owned]
        except egat.EgatError as e:   # a local system past the plan builder's size limit
            if e.code != egat.EGAT_ERR_UNSUPPORTED:
                raise
    out = egat.egat_otf_attention_coupled(s_loc, q_loc, k_loc, hp_loc, nbr, cnt, st.pos_loc, w2)
    return out[:plan.n_owned]


def forward_rank(plan: HaloPlan, shape: "egat.Shape", h: torch.Tensor, pos: torch.Tensor,
                 q: torch.Tensor, k: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor,
                 group=None, own_rows: bool = False) -> torch.Tensor:
    """^h of this rank's atoms (float32 [n_owned, D, C], in plan.owned order) for the
    inputs h, pos, q, k of the `shape` system (whole arrays, or with own_rows
    this rank's rows of h, q, k): step 2 on the owned atoms, one exchange of the
    boundary atoms' h' and k rows (NCCL all-to-all in `group`), then steps 3+4
    over the local arrays."""
    st = couple_rank(plan, shape, h, pos, q, k, w1, own_rows=own_rows)
    hp_halo = exchange(plan, st.hp_own, group)
    k_halo = exchange(plan, st.k_own, group)
    return attend_rank(plan, shape, st, hp_halo, k_halo, w2)
