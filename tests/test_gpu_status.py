"""GPU tests of the library's failure report (egat_take_device_status).

The tensor-core attention kernel waits on mbarriers for its bulk copies and
bounds every wait; a wait that gives up is counted on the device and reported
as EGAT_ERR_TIMEOUT.  The failure is made by a self-test kernel whose wait
cannot succeed (an mbarrier that expects bytes no copy delivers), with a short
poll limit: nothing faults and nothing hangs.
"""
import numpy as np
import pytest

from equivariant_graph_attention_b200 import synth
from tests.parity_util import device_inputs, shape_of

pytestmark = pytest.mark.gpu


def _egat():
    from equivariant_graph_attention_b200 import egat
    return egat


def test_wait_timeout_is_reported_and_cleared():
    egat = _egat()
    egat.egat_take_device_status()                       # start from a clean count
    assert egat.egat_take_device_status() == egat.EGAT_OK
    egat.egat_selftest_wait_timeout(polls=1000)
    assert egat.egat_take_device_status() == egat.EGAT_ERR_TIMEOUT
    assert egat.egat_take_device_status() == egat.EGAT_OK


def test_tiled_attention_reports_no_timeout():
    egat = _egat()
    wl = synth.WORKLOADS["uniform4096_l2_bf16"]
    d = synth.make(wl)
    dev = device_inputs(wl, d)
    shape = shape_of(wl)
    egat.egat_take_device_status()
    g = egat.egat_build_graph(dev["pos_q"], wl.cutoff_q, K=wl.K)
    plan = egat.egat_build_attention_plan(shape, g["nbr"], g["cnt"], g["order"], dev["pos"])
    hp = egat.egat_eaas_couple_planned(shape, dev["h"], plan, dev["w1"])
    out = egat.egat_otf_attention_tiled(shape, dev["q"], dev["k"], hp, plan, w2=dev["w2"])
    assert egat.egat_take_device_status() == egat.EGAT_OK
    assert np.isfinite(out.cpu().numpy()).all()
