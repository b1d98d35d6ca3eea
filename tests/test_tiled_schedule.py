"""Host-side model of the copy / wait protocol of the tensor-core attention
kernel (`otf_attention_tc_kernel`, csrc/attention_tc.cu).

A CTA walks the tiles it claims, in claim order (the claims themselves are
modelled by test_tile_claims below).  Bulk copies fill shared-memory
buffers and complete mbarrier phases: the stage buffers (rows), two tile
record buffers (alternating), the tile's union indices + query rows, and its
membership mask.  This model replays the kernel's control flow (tile
prologue, stage loop with its barrier, the prefetch of the next tile's record,
indices, mask and first rows, the epilogue) as a sequence of events in
barrier-separated phases, and checks for random union lengths (empty tiles
and one-stage tiles included), for every stage shape the kernel uses:

* every wait names the parity of the phase whose fill it needs, and no
  barrier is filled again before every thread has waited on its last phase;
* every read of a buffer happens after the reader waited on the fill that
  delivered its contents;
* no copy overwrites a buffer while a read of its previous contents in the
  same or a later phase is still due (reads of the old contents all lie in
  earlier phases, or precede the issue in the issuing thread).
No GPU is involved.
"""
import random

import pytest

SHAPES = {1: (3, 32), 2: (2, 32), 3: (2, 16)}    # lmax -> (STAGES, RS)
SM_COUNT = 148


class Model:
    def __init__(self):
        self.phase = 0
        self.fills = {}      # barrier -> number of fills issued
        self.waited = {}     # barrier -> set of (fill index) every thread has waited
        self.content = {}    # buffer -> (payload, barrier, fill index, phase of issue)
        self.last_read = {}  # buffer -> (payload, phase) of the latest read by all threads

    def barrier(self):
        self.phase += 1

    def fill(self, bar, buf, payload):
        n = self.fills.get(bar, 0)
        if n > 0:
            assert (n - 1) in self.waited.get(bar, set()), f"{bar} refilled before phase {n - 1} was waited"
        old = self.content.get(buf)
        if old is not None:
            lr = self.last_read.get(buf)
            if lr is not None and lr[0] == old[0]:
                assert lr[1] < self.phase, f"{buf} overwritten in the phase of a read of {old[0]}"
        self.content[buf] = (payload, bar, n, self.phase)
        self.fills[bar] = n + 1

    def wait(self, bar, parity, expect_fill):
        assert expect_fill < self.fills.get(bar, 0), f"{bar}: waiting on a fill never issued"
        assert parity == (expect_fill & 1), f"{bar}: parity {parity} for fill {expect_fill}"
        self.waited.setdefault(bar, set()).add(expect_fill)

    def read(self, buf, payload, by_all=True):
        cur = self.content.get(buf)
        assert cur is not None and cur[0] == payload, f"{buf} holds {cur and cur[0]}, wanted {payload}"
        assert cur[2] in self.waited.get(cur[1], set()), f"{buf} read before its fill was waited"
        if by_all:
            self.last_read[buf] = (payload, self.phase)


def replay(S, RS, ulen_of_tiles):
    """One CTA over its tiles (union lengths given); mirrors the kernel."""
    m = Model()
    stages_of = lambda U: (U + RS - 1) // RS
    K = len(ulen_of_tiles)
    stage_bar = lambda gs: f"full{gs % S}"
    stage_fill = {}      # global stage -> fill index of its buffer's barrier
    gbase = 0

    def issue_rows(k, s, gs):
        # row-issuing threads (several, not only thread 0) read the indices:
        # a copy over them must wait for a later phase
        m.read("su", ("idx", k))
        m.fill(stage_bar(gs), f"stage{gs % S}", ("rows", k, s))
        stage_fill[gs] = m.fills[stage_bar(gs)] - 1

    rec_fill = {}
    def issue_record(k):
        m.fill(f"rec{k & 1}", f"recbuf{k & 1}", ("rec", k))
        rec_fill[k] = m.fills[f"rec{k & 1}"] - 1

    def wait_rec(k):
        m.wait(f"rec{k & 1}", (k >> 1) & 1, rec_fill[k])

    # first tile
    issue_record(0)
    wait_rec(0)
    m.fill("idx", "su", ("idx", 0)); m.content["sq"] = (("q", 0), "idx", m.fills["idx"] - 1, m.phase)
    m.fill("msk", "smask", ("msk", 0))
    m.wait("idx", 0, 0)
    for s in range(min(S - 1, stages_of(ulen_of_tiles[0]))):
        issue_rows(0, s, s)
    for k in range(K):
        has_next = k + 1 < K
        wait_rec(k)
        m.wait("idx", k & 1, k)
        m.wait("msk", k & 1, k)
        m.read(f"recbuf{k & 1}", ("rec", k))
        ns = stages_of(ulen_of_tiles[k])
        m.read("sq", ("q", k))
        trig = max(0, ns - S + 1)
        take_st = trig - 1 if trig > 1 else 0    # the claimed next tile's record is copied here
        for st in range(ns):
            m.barrier()
            if st + S - 1 < ns:
                issue_rows(k, st + S - 1, gbase + st + S - 1)
            if st == take_st and has_next:
                issue_record(k + 1)
            if st == trig and has_next:
                wait_rec(k + 1)
                m.fill("idx", "su", ("idx", k + 1))
                m.content["sq"] = (("q", k + 1), "idx", m.fills["idx"] - 1, m.phase)
                assert m.last_read["sq"][1] < m.phase
            gs = gbase + st
            m.wait(stage_bar(gs), (gs // S) & 1, stage_fill[gs])
            m.read(f"stage{gs % S}", ("rows", k, st))
            m.read("smask", ("msk", k))
        if ns == 0 and has_next:
            issue_record(k + 1)
        m.barrier()
        gbase += ns
        if has_next:
            if ns == 0:
                wait_rec(k + 1)
                m.fill("idx", "su", ("idx", k + 1))
                m.content["sq"] = (("q", k + 1), "idx", m.fills["idx"] - 1, m.phase)
            m.fill("msk", "smask", ("msk", k + 1))
            wait_rec(k + 1)
            m.wait("idx", (k + 1) & 1, k + 1)
            m.read(f"recbuf{(k + 1) & 1}", ("rec", k + 1))
            for s in range(min(S - 1, stages_of(ulen_of_tiles[k + 1]))):
                issue_rows(k + 1, s, gbase + s)
        m.read(f"recbuf{k & 1}", ("rec", k))      # epilogue
        m.barrier()


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_copy_wait_protocol(lmax):
    S, RS = SHAPES[lmax]
    rng = random.Random(100 + lmax)
    for _ in range(300):
        tiles = rng.choice([1, 2, 3, 4, 7, 15])
        short = rng.random() < 0.5
        ulen = [rng.choice([0, 1, 16, 17, 31, 32, 33, 64, 65]) if short else rng.randint(0, 1500)
                for _ in range(tiles)]
        replay(S, RS, ulen)


def test_model_catches_a_missing_wait():
    """The model rejects a read before the wait on its fill."""
    m = Model()
    m.fill("idx", "su", ("idx", 0))
    with pytest.raises(AssertionError):
        m.read("su", ("idx", 0), by_all=False)


def test_model_catches_an_early_index_prefetch():
    """The model rejects prefetching the next tile's indices one stage too
    early (while the last rows of the current tile still read them)."""
    src = open(__file__).read().replace("trig = max(0, ns - S + 1)", "trig = max(0, ns - S)")
    ns = {}
    exec(compile(src.split("@pytest.mark.parametrize")[0], "mutant", "exec"), ns)
    with pytest.raises(AssertionError):
        for seed in range(50):
            rng = random.Random(seed)
            ns["replay"](2, 32, [rng.randint(33, 400) for _ in range(4)])


def claims(tiles: int, grid: int, seed: int):
    """The run-time tile claims of `grid` CTAs, in a random interleaving.

    A CTA's first tile is its block index; once per tile (near its end) its
    thread 0 takes a ticket c = atomicAdd(counter, 1), and a while later it
    takes the claim: the next tile is grid + c, past the last tile meaning
    done, and the holder of ticket tiles - 1 sets the counter to zero.
    Returns the tiles each CTA processed and the counter after the launch."""
    rng = random.Random(seed)
    box = [0]
    got = {b: [] for b in range(grid)}
    handed = []

    def cta(b):
        tile = b
        while tile < tiles:
            got[b].append(tile)
            yield                            # the tile's work, up to the claim
            c = box[0]                       # atomicAdd returns the old value
            box[0] += 1
            handed.append(c)
            yield                            # a stage later: take the claim
            if c == tiles - 1:
                assert sorted(handed) == list(range(tiles)), "reset before the last claim"
                box[0] = 0
            yield                            # the rest of the tile
            tile = grid + c

    progs = {b: cta(b) for b in range(grid)}
    live = set(progs)
    while live:
        b = rng.choice(sorted(live))
        try:
            next(progs[b])
        except StopIteration:
            live.discard(b)
    assert handed == list(range(tiles))      # tickets are handed out in order
    return got, box[0]


@pytest.mark.parametrize("tiles", [1, 2, 147, 148, 149, 300, 2048])
@pytest.mark.parametrize("seed", range(3))
def test_tile_claims(tiles, seed):
    """Every tile is processed exactly once, whatever the interleaving, and
    the counter is zero again after each launch (three launches in a row on
    one plan)."""
    grid = min(tiles, SM_COUNT)
    for launch in range(3):
        got, after = claims(tiles, grid, seed * 10 + launch)
        assert sorted(t for ts in got.values() for t in ts) == list(range(tiles))
        assert all(ts and ts[0] == b for b, ts in got.items())
        assert after == 0
