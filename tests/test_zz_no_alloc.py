"""egat_forward_noalloc: the forward pass for callers that cannot allocate.

Some callers of this library may not allocate device memory when they call
it — a plugin inside a framework that owns every device allocation, or a
service whose memory footprint is fixed at start-up.  egat_forward_noalloc
serves them: its scratch is a fixed device array inside the library.  These
tests call it through the C ABI and require its output to match egat_forward
(which takes a caller-allocated workspace) within the float tolerance the
parity tests use, on two calls in a row with different inputs, so that a
stale scratch from the first call would show up in the second.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from equivariant_graph_attention_b200 import synth
from tests.parity_util import FLOOR, TOL, block_rel_error, channel_rel_error, device_inputs, shape_of

pytestmark = pytest.mark.gpu


def _case(name, seed):
    from equivariant_graph_attention_b200 import egat
    wl = synth.WORKLOADS[name]
    dev = device_inputs(wl, synth.make(wl, seed))
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    return wl, dev, g


@pytest.mark.parametrize("name", ["water216_l2_f32", "uniform4096_l2_bf16"])
def test_noalloc_matches_forward_on_two_calls(name):
    from equivariant_graph_attention_b200 import egat
    for seed in (0, 1):          # two calls in a row, different inputs
        wl, dev, g = _case(name, seed)
        shape = shape_of(wl)
        assert egat.egat_forward_workspace_bytes(shape) <= egat.NOALLOC_SCRATCH_BYTES
        ref = egat.egat_forward(shape, dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"],
                                g["cnt"], dev["w1"], dev["w2"], order=g["order"])
        out = torch.full_like(ref, float("nan"))
        egat.egat_forward_noalloc(shape, dev["h"], dev["pos"], dev["q"], dev["k"], g["nbr"],
                                  g["cnt"], dev["w1"], dev["w2"], out, order=g["order"])
        torch.cuda.synchronize()
        err = block_rel_error(out.cpu().numpy(), ref.cpu().numpy(), wl.lmax)
        assert err < TOL[wl.dtype], (name, seed, err)
        e = channel_rel_error(out.cpu().numpy(), ref.cpu().numpy(), wl.lmax, FLOOR[wl.dtype])
        assert e < TOL[wl.dtype], (name, seed, e)


def test_noalloc_rejects_problems_beyond_its_scratch():
    from equivariant_graph_attention_b200 import egat
    wl = synth.WORKLOADS["uniform32768_K256_l2_bf16"]          # h' is 75.5 MB
    shape = shape_of(wl)
    assert egat.egat_forward_workspace_bytes(shape) > egat.NOALLOC_SCRATCH_BYTES
    lib = egat.load_library()
    cs = shape.c()
    fake = ctypes.c_void_p(0x10000)
    rc = lib.egat_forward_noalloc(ctypes.byref(cs), fake, fake, fake, fake, fake, fake, None,
                                  fake, fake, fake, None)
    assert rc == egat.EGAT_ERR_SCRATCH_LIMIT
    assert b"scratch" in lib.egat_strerror(rc)
