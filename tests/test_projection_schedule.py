"""Host-side model of the copy / product protocol of the tensor-core
query/key projection (`qk_projection_umma_kernel`, csrc/projection.cu).

A CTA walks its tiles slot, slot + stride, ... .  Its threads fill two
shared-memory A buffers with cp.async copies, one commit group per tile
sequence number (an empty group past the last tile): groups 0 and 1 before
the loop, group j + 2 in iteration j once the products of tile j are done.
Iteration j waits until at most one group is pending (cp.async.wait_group 1),
issues tile j's products from buffer j % 2, and waits on the mbarrier phase
of parity j % 2 that their commit completes.  This model replays that
control flow for many tile counts and grid sizes and checks:

* the group that fills tile j's buffer is complete when its products are
  issued, and it carries tile j;
* no buffer is refilled before the products that read its previous tile
  have completed;
* one commit per tile, so the mbarrier has at most one phase pending and
  tile j waits on parity j % 2;
* every tile of the CTA is multiplied exactly once, and every group is
  complete when the CTA exits (cp.async.wait_group 0).
No GPU is involved.
"""
import pytest

K_UM = 128          # the kernel's kUM: atoms per tile


def replay(tiles: int, slot: int, stride: int):
    groups = []                      # committed groups: (sequence number, buffer, tile or None)
    complete = 0                     # groups complete so far (they complete in order)
    buffer_busy = {0: None, 1: None}  # buffer -> sequence number whose products still read it
    done_products = set()
    phases = 0                       # mbarrier phases completed

    def load(seq, b):
        tile = slot + seq * stride
        assert buffer_busy[b] is None, (seq, b, buffer_busy[b])
        groups.append((seq, b, tile if tile < tiles else None))

    load(0, 0)
    load(1, 1)
    j = 0
    tile = slot
    multiplied = []
    while tile < tiles:
        b = j % 2
        # cp.async.wait_group 1: every group but the newest is complete
        complete = max(complete, len(groups) - 1)
        seq, gb, gtile = groups[j]
        assert j < complete and seq == j and gb == b and gtile == tile
        buffer_busy[b] = j                       # the products read buffer b
        parity = phases & 1
        assert parity == j % 2
        phases += 1                              # the commit completes the phase
        done_products.add(j)
        buffer_busy[b] = None                    # products done: buffer b is free
        multiplied.append(tile)
        load(j + 2, b)
        tile += stride
        j += 1
    complete = len(groups)                       # cp.async.wait_group 0 before exit
    assert all(i < complete for i in range(len(groups)))
    assert len(groups) == j + 2
    return multiplied


@pytest.mark.parametrize("n", [1, 127, 128, 129, 1000, 4096, 32768, 100000, 175616])
@pytest.mark.parametrize("sms", [148, 8])
def test_projection_copy_product_protocol(n, sms):
    tiles = (n + K_UM - 1) // K_UM
    pairs = min(tiles, sms // 2)
    seen = []
    for slot in range(pairs):
        seen += replay(tiles, slot, pairs)
    assert sorted(seen) == list(range(tiles))   # every tile once per matrix (q or k)
