"""Host-side model of the copy / wait protocol of the tensor-core query/key
projection (`qk_projection_tc_kernel`, csrc/projection.cu).

A CTA walks its tiles slot, slot + stride, ... .  Bulk copies fill a ring of
kPBuf shared-memory tiles, each completing its own mbarrier; the ring starts
with the first kPBuf - 1 tiles in flight, iteration j waits on buffer
j % kPBuf (phase parity (j / kPBuf) & 1), then issues the tile kPBuf - 1
ahead into the buffer iteration j - 1 read, and ends with a block barrier.
After a wait gives up, the drain waits on the last issued phase of every
buffer.  This model replays that control flow for many tile counts and grid
sizes and checks:

* every wait names the parity of the fill that delivers the tile it reads;
* no buffer is refilled before the barrier that ends the iteration reading
  its previous contents;
* every issued fill is waited on, in the loop or by the drain, and the drain
  waits exactly the last issued fill of each buffer.
No GPU is involved.
"""
import pytest

K_PBUF = 4          # the kernel's kPBuf
K_PM = 64           # atoms per tile


def replay(tiles: int, slot: int, stride: int):
    fills = {b: [] for b in range(K_PBUF)}       # buffer -> tile sequence numbers issued
    waited = set()                               # (buffer, fill index)
    barriers = 0
    issued_at = {}                               # (buffer, fill index) -> barrier count at issue

    def issue(seq):
        b = seq % K_PBUF
        if fills[b]:
            prev = fills[b][-1]
            # the previous contents are read by iteration prev, which must have
            # ended with its barrier (one barrier per iteration, from 0)
            assert barriers >= prev + 1, (seq, prev, barriers)
            assert prev < seq
        fills[b].append(seq)
        issued_at[(b, len(fills[b]) - 1)] = barriers

    for q in range(K_PBUF - 1):
        if slot + q * stride < tiles:
            issue(q)
    j = 0
    tile = slot
    while tile < tiles:
        b = j % K_PBUF
        parity = (j // K_PBUF) & 1
        k = fills[b].index(j)                   # the fill that carries tile j
        assert k % 2 == parity
        waited.add((b, k))
        if tile + (K_PBUF - 1) * stride < tiles:
            issue(j + K_PBUF - 1)
        barriers += 1                           # __syncthreads ends iteration j
        tile += stride
        j += 1
    # the kernel's drain after a give-up: the last issued sequence number of
    # each buffer among 0 .. j + kPBuf - 2 (those that exist)
    drain = {}
    for b in range(K_PBUF):
        last = -1
        for q in range(j + K_PBUF - 1):
            if q % K_PBUF == b and slot + q * stride < tiles:
                last = q
        if last >= 0:
            drain[b] = (last // K_PBUF) & 1
    for b, seqs in fills.items():
        if seqs:
            assert b in drain and drain[b] == ((len(seqs) - 1) % 2), (b, seqs)
            for k in range(len(seqs)):
                assert (b, k) in waited or k == len(seqs) - 1
        else:
            assert b not in drain
    return j


@pytest.mark.parametrize("n", [1, 63, 64, 65, 1000, 4096, 32768, 100000, 175616])
@pytest.mark.parametrize("sms", [148, 8])
def test_projection_ring_protocol(n, sms):
    tiles = (n + K_PM - 1) // K_PM
    pairs = min(tiles, sms // 2)
    stride = pairs
    done = 0
    for slot in range(pairs):
        done += replay(tiles, slot, stride)
    assert done == tiles                         # every tile is processed by exactly one CTA of a pair
