"""Write the oracle's output for a tiny seeded system to forward_tiny.json.

Calls only the oracle and the seeded input generator.  The stored values lock
the oracle against unintended change (a regression fixture, not a pin: the
pages print no worked example of the forward pass) and give the CUDA parity
tests one fixed case.  Run from the repository root:

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


def main():
    wl, d, nbrs, full, out = build()
    rec = {"spec": SPEC, "cutoff_q": wl.cutoff_q,
           "neighbours": [n.tolist() for n in nbrs], "full_degree": full.tolist(),
           "out": np.round(out, 15).tolist()}
    with open(os.path.join(HERE, "forward_tiny.json"), "w") as f:
        json.dump(rec, f)


if __name__ == "__main__":
    main()
