"""Write the oracle's output for a tiny seeded system to forward_tiny.json, and
its gradients for a seeded upstream gradient to backward_tiny.json.

Calls only the oracle and the seeded input generator.  The stored values lock
the oracle against unintended change (regression fixtures, not pins: the
pages print no worked example of either pass; the backward's pins are finite
differences of the forward) and give the CUDA parity tests one fixed case.
Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle.attention import forward          # noqa: E402
from oracle.graph import radius_graph         # noqa: E402
from equivariant_graph_attention_b200 import synth   # noqa: E402

SPEC = dict(n=12, side=5.0, cutoff=3.0, K=6, lmax=2, C=16, H=2, dk=8, dtype="f32", seed=11)


def build():
    s = SPEC
    wl = synth.small_cube(s["n"], s["side"], s["cutoff"], s["K"], s["lmax"], s["C"], s["H"],
                          s["dk"], s["dtype"])
    d = synth.make(wl, s["seed"])
    nbrs, full = radius_graph(d["pos_q"], wl.cutoff_q, K=wl.K)
    out = forward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, nbrs)
    return wl, d, nbrs, full, out


def build_backward():
    """(G, dh, dq, dk, dr) of L = <G, ^h> for the tiny system, G ~ N(0, 1) seeded."""
    from oracle.backward import backward, position_grad
    wl, d, nbrs, _, _ = build()
    G = np.random.default_rng([SPEC["seed"], 99]).standard_normal((wl.n, wl.D, wl.C))
    dh, dq, dk = backward(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, nbrs, G)
    dr = position_grad(d["h"], d["pos"], d["q"], d["k"], d["w1"], d["w2"], wl.lmax, nbrs, G)
    return G, dh, dq, dk, dr


def main():
    wl, d, nbrs, full, out = build()
    rec = {"spec": SPEC, "cutoff_q": wl.cutoff_q,
           "neighbours": [n.tolist() for n in nbrs], "full_degree": full.tolist(),
           "out": np.round(out, 15).tolist()}
    with open(os.path.join(HERE, "forward_tiny.json"), "w") as f:
        json.dump(rec, f)
    G, dh, dq, dk, dr = build_backward()
    rec = {"spec": SPEC, "upstream_seed": [SPEC["seed"], 99],
           "dh": np.round(dh, 15).tolist(), "dq": np.round(dq, 15).tolist(),
           "dk": np.round(dk, 15).tolist(), "dr": np.round(dr, 15).tolist()}
    with open(os.path.join(HERE, "backward_tiny.json"), "w") as f:
        json.dump(rec, f)


if __name__ == "__main__":
    main()
