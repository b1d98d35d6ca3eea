"""Host-side check of the source plan's sizing (csrc/backward_tc.cu).

The tiled backward builds, per tile of 16 source atoms (slots of the
traversal order), the union of the targets whose neighbour lists hold one of
its sources.  Its capacity is the sum of the sources' in-degrees rounded up to
a multiple of 32 (at least 32), and tiles are laid end to end by an exclusive
scan of the capacities.  The workspace reserves n*K + 32*tiles union entries
and half as many mask words, sized on the host before any in-degree is known.

This model recomputes capacities, offsets and unions with numpy for random
padded graphs, including skewed ones (every atom listing the same few atoms,
in-degrees far above K), and checks that every tile's union and mask words
fit its slice and that the slices fit the reservation.  No GPU is involved.
"""
import numpy as np
import pytest

TILE = 16
PAD = 32


def plan_sizes(nbr, cnt, order):
    n, K = nbr.shape
    tiles = (n + TILE - 1) // TILE
    indeg = np.zeros(n, dtype=np.int64)
    holders = [[] for _ in range(n)]
    for i in range(n):
        for j in nbr[i, :cnt[i]]:
            if 0 <= j < n:
                indeg[j] += 1
                holders[j].append(i)
    caps, unions = [], []
    for t in range(tiles):
        srcs = [order[s] for s in range(t * TILE, min((t + 1) * TILE, n))]
        s_t = int(sum(indeg[a] for a in srcs))
        caps.append(max(PAD, -(-s_t // PAD) * PAD))
        unions.append(len(set(i for a in srcs for i in holders[a])))
    offs = np.concatenate([[0], np.cumsum(caps)])
    return n, K, tiles, caps, offs, unions


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("skew", [False, True])
def test_source_plan_fits_its_reservation(seed, skew):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 200))
    K = int(rng.integers(1, 40))
    cnt = rng.integers(0, K + 1, size=n)
    if skew:
        hubs = rng.integers(0, n, size=3)
        nbr = rng.choice(hubs, size=(n, K))
    else:
        nbr = rng.integers(-1, n, size=(n, K))
    order = rng.permutation(n)
    n, K, tiles, caps, offs, unions = plan_sizes(nbr, cnt, order)
    reserve = n * K + PAD * tiles
    assert offs[-1] <= reserve
    for t in range(tiles):
        upad = max(PAD, -(-unions[t] // PAD) * PAD)
        assert upad <= caps[t]                     # the padded union fits the slice
        assert caps[t] % PAD == 0 and offs[t] % PAD == 0
        # mask words: cap/32 chunks of 16 words at offs/2, inside the half-size reservation
        assert offs[t] // 2 + caps[t] // 2 <= reserve // 2
