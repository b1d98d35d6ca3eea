"""Host-side model of the copy / wait protocol of the tile-staged source
coupling (`eaas_tile_kernel`, csrc/coupling.cu).

A CTA of 8 warps takes the plan's tiles j = 0, 1, ... in turn.  Bulk copies
fill two row buffers (tile j in rows[j % 2], completing rowbar[j % 2]) and
three record buffers (tile j in recs[j % 3], completing recbar[j % 3]).
Thread 0 issues tile 0's record and rows and tile 1's record; at tile j,
warp 0 issues tile j + 1's rows and tile j + 2's record, after waiting on
donebar[(j - 1) % 2] for the phase in which all 8 warps said they were done
with tile j - 1 (the last reader of both buffers).  Every warp waits on
tile j's record and rows, reads them, and arrives on donebar[j % 2].  There
is no block-wide barrier, so warps drift apart.

The model runs the 8 warps as independent programs under many random
schedules (one warp steps at a time, a wait blocks until its phase has
completed) and checks:

* every wait names the parity of the phase that carries its tile: the fill
  (or the all-warps-done phase) it needs, never one a full cycle earlier or
  later;
* no copy overwrites a buffer while any warp may still read the tile it
  holds;
* every schedule finishes (no deadlock), and every warp reads every tile's
  own record and rows.
No GPU is involved.
"""
import random

import pytest

WARPS = 8


class Barrier:
    """An mbarrier: phases complete in order; `arrivals` per phase."""

    def __init__(self, count):
        self.count = count
        self.pending = 0
        self.completed = 0          # phases completed
        self.log = []               # payload tag of each completed phase

    def arrive(self, tag):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.completed += 1
            self.log.append(tag)

    def ready(self, parity, want_phase):
        # try_wait.parity(p) succeeds when the current phase's parity differs
        # from p, so the wait means phase `want_phase` only while the barrier
        # is at that phase or one past it; two phases behind or ahead, the
        # parity would name another phase
        assert parity == want_phase & 1
        assert want_phase <= self.completed <= want_phase + 1, (want_phase, self.completed)
        return self.completed == want_phase + 1


def run(tiles: int, seed: int):
    rng = random.Random(seed)
    rowbar = [Barrier(1), Barrier(1)]
    recbar = [Barrier(1), Barrier(1), Barrier(1)]
    donebar = [Barrier(WARPS), Barrier(WARPS)]
    rows = [None, None]                  # tile whose rows the buffer holds
    recs = [None, None, None]
    readers = {}                         # (kind, buffer) -> set of warps still to read the held tile

    def fill(kind, buf, tile):
        held = rows[buf] if kind == "rows" else recs[buf]
        if held is not None:
            assert not readers.get((kind, buf)), (kind, buf, held, tile)   # nobody still needs it
        (rows if kind == "rows" else recs)[buf] = tile
        readers[(kind, buf)] = set(range(WARPS))
        (rowbar if kind == "rows" else recbar)[buf].arrive(tile)

    # thread 0 before the loop (the first record is waited on at once)
    fill("recs", 0, 0)
    fill("rows", 0, 0)
    if tiles > 1:
        fill("recs", 1, 1)

    def program(w):
        for j in range(tiles):
            rb, wb = j % 3, j % 2
            while not recbar[rb].ready((j // 3) & 1, j // 3):
                yield
            while not rowbar[wb].ready((j >> 1) & 1, j >> 1):
                yield
            if w == 0 and j + 1 < tiles:
                if j >= 1:
                    b = (j + 1) % 2
                    while not donebar[b].ready(((j - 1) >> 1) & 1, (j - 1) >> 1):
                        yield
                nb = (j + 1) % 3
                while not recbar[nb].ready(((j + 1) // 3) & 1, (j + 1) // 3):
                    yield
                assert recs[nb] == j + 1
                fill("rows", (j + 1) % 2, j + 1)
                if j + 2 < tiles:
                    fill("recs", (j + 2) % 3, j + 2)
            # the tile's compute reads its record and rows
            assert recs[rb] == j and rows[wb] == j, (w, j, recs, rows)
            yield
            readers[("recs", rb)].discard(w)
            readers[("rows", wb)].discard(w)
            donebar[wb].arrive(j)

    progs = {w: program(w) for w in range(WARPS)}
    live = set(progs)
    steps = 0
    while live:
        w = rng.choice(sorted(live))
        try:
            next(progs[w])
        except StopIteration:
            live.discard(w)
        steps += 1
        assert steps < 200000, "no progress: a wait can never be satisfied"
    assert donebar[0].completed + donebar[1].completed == tiles
    assert donebar[0].log == list(range(0, tiles, 2)) and donebar[1].log == list(range(1, tiles, 2))


@pytest.mark.parametrize("tiles", [1, 2, 3, 4, 5, 7, 16, 33])
@pytest.mark.parametrize("seed", range(6))
def test_tile_coupling_protocol(tiles, seed):
    run(tiles, seed * 101 + tiles)
