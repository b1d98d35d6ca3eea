"""Host-side model of the copy / product / read-back protocol of the
tensor-core query/key projection (`qk_projection_umma_kernel`,
csrc/projection.cu).

A CTA walks its tiles slot, slot + stride, ... (J of them; sequence numbers
j = 0 .. J-1).  Two A buffers in shared memory receive the tiles' degree-0
slices by tensor copies, tile j into buffer j % 2, completing mbarrier
abar[j % 2]; two float32 accumulators in tensor memory receive the products,
tile j into accumulator j % 2, and the products' commit completes mbarrier
bar[j % 2].  Thread 0 issues the copies of tiles 0 and 1 before the loop and
the products of tile 0.  Iteration j:
  1. issues tile j + 1's products (after a CTA barrier, which orders them
     after every warp's read-back of tile j - 1 from the same accumulator,
     and after waiting on abar[(j + 1) % 2] for tile j + 1's copies);
  2. waits on bar[j % 2] for tile j's products;
  3. issues tile j + 2's copies into buffer j % 2 (freed by step 2);
  4. reads accumulator j % 2 back and stores tile j.
Copies complete in any order; the products of one thread complete in issue
order.  This model runs the asynchronous engines under many random
schedules and checks:

* every wait names the parity of the phase that carries its tile;
* products read a buffer only after its copy completed and while no copy
  into it is in flight, and a copy never lands in a buffer whose products
  are still pending;
* products never write an accumulator that a read-back still needs, and a
  read-back sees exactly its own tile's products;
* every tile of the CTA is stored once, and nothing is in flight when the
  CTA exits (so tensor memory and shared memory may be released).
It also checks the grid's partition of the tiles for several sizes.
No GPU is involved.
"""
import random

import pytest

K_UM = 128          # the kernel's kUM: atoms per tile


class Barrier:
    """An mbarrier with one arrival per phase."""

    def __init__(self):
        self.completed = 0
        self.log = []

    def complete(self, tag):
        self.completed += 1
        self.log.append(tag)

    def ready(self, parity, want_phase):
        # try_wait.parity names phase `want_phase` only while the barrier is at
        # that phase or one past it
        assert parity == want_phase & 1
        assert want_phase <= self.completed <= want_phase + 1, (want_phase, self.completed)
        return self.completed == want_phase + 1


def replay(tiles: int, slot: int, stride: int, seed: int):
    rng = random.Random(seed)
    abar, bar = [Barrier(), Barrier()], [Barrier(), Barrier()]
    abuf = [None, None]          # tile whose slices the buffer holds (after its copy completes)
    acc = [None, None]           # tile whose products the accumulator holds
    copies = []                  # in flight: (buffer, tile)
    products = []                # in flight, in issue order: (buffer, accumulator, tile)
    reading = [None, None]       # accumulator -> tile being read back
    stored = []

    def step_engines():
        """complete one asynchronous operation, chosen at random"""
        kinds = []
        if copies:
            kinds.append("copy")
        if products:
            kinds.append("mma")
        if not kinds:
            return False
        if rng.choice(kinds) == "copy":
            b, t = copies.pop(rng.randrange(len(copies)))
            assert not any(pb == b for pb, _, _ in products), "a copy lands under pending products"
            abuf[b] = t
            abar[b].complete(t)
        else:
            b, a, t = products.pop(0)
            assert abuf[b] == t, "products read a buffer that does not hold their tile"
            assert not any(cb == b for cb, _ in copies), "products read a buffer under a copy"
            assert reading[a] is None, "products overwrite an accumulator being read"
            acc[a] = t
            bar[a].complete(t)
        return True

    def wait(barrier, parity, phase):
        while not barrier.ready(parity, phase):
            assert step_engines(), "a wait with nothing in flight never completes"

    def load_tile(jj, b):
        tl = slot + jj * stride
        if tl < tiles:
            assert not any(cb == b for cb, _ in copies)
            copies.append((b, tl))

    def issue(jj):
        # the CTA barrier: every read-back of an earlier tile has finished
        assert reading == [None, None]
        b = jj & 1
        wait(abar[b], (jj >> 1) & 1, jj >> 1)
        products.append((b, b, slot + jj * stride))

    J = (tiles - slot + stride - 1) // stride if slot < tiles else 0
    load_tile(0, 0)
    load_tile(1, 1)
    if J > 0:
        issue(0)
    for j in range(J):
        tile = slot + j * stride
        b = j & 1
        if j + 1 < J:
            issue(j + 1)
        # the engines run on while the CTA works
        for _ in range(rng.randrange(3)):
            step_engines()
        wait(bar[b], (j >> 1) & 1, j >> 1)
        load_tile(j + 2, b)
        reading[b] = tile
        for _ in range(rng.randrange(3)):
            step_engines()
        assert acc[b] == tile, "the read-back sees another tile's products"
        stored.append(tile)
        reading[b] = None
    assert not copies and not products, "work in flight at exit"
    for a in range(2):
        assert bar[a].log == [slot + jj * stride for jj in range(a, J, 2)]
    return stored


@pytest.mark.parametrize("n", [1, 127, 128, 129, 1000, 4096, 32768, 100000, 175616])
@pytest.mark.parametrize("sms", [148, 8])
def test_projection_copy_product_protocol(n, sms):
    tiles = (n + K_UM - 1) // K_UM
    pairs = min(tiles, sms // 2)
    seen = []
    for slot in range(pairs):
        seen += replay(tiles, slot, pairs, seed=n * 7 + slot)
    assert sorted(seen) == list(range(tiles))   # every tile once per matrix (q or k)


@pytest.mark.parametrize("seed", range(40))
def test_projection_protocol_random_schedules(seed):
    rng = random.Random(seed)
    tiles = rng.randrange(1, 40)
    stride = rng.randrange(1, 6)
    for slot in range(min(stride, tiles)):
        assert replay(tiles, slot, stride, seed * 31 + slot) == list(range(slot, tiles, stride))
