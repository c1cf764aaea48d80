"""Writes tests/golden/tiny_oracle.json from the oracle alone.

The pages print no worked numeric example, so this fixture is a regression
record of the float64 oracle on the seed-0 "tiny" workload (1 request, 16 heads,
L = 256, 8 tree nodes): visibility words, depths, accept result, every lse value
and per-node sums of the output.  Regenerate with
    python tests/golden/make_golden.py
only when a change to the oracle's arithmetic is justified by the pages.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from tree_speculative_decoding_kd_b200 import workload as W  # noqa: E402


def compute():
    wl = W.make_workload("tiny")
    st = wl.step
    res = oracle.verify_step(wl.c_kv, wl.k_rope, wl.cache_lens, st.parents, st.tokens,
                             st.argmax, st.q_abs, st.q_rope, wl.cfg.scale)
    return {
        "workload": "tiny (B=1, H=16, n=8, L=256, seed 0)",
        "parents": st.parents[0].tolist(),
        "vis_words": res["vis"][0, :, 0].tolist(),
        "depths": oracle.depths(st.parents[0]).tolist(),
        "accept_path": res["path"][0, :res["len"][0]].tolist(),
        "accept_len": int(res["len"][0]),
        "bonus": int(res["bonus"][0]),
        "lse": [[float(x) for x in row] for row in res["lse"][0]],
        "out_node_sums": [float(x) for x in res["out"][0].sum(axis=(1, 2))],
        "out_00_first8": [float(x) for x in res["out"][0, 0, 0, :8]],
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(compute(), f, indent=1)
    print("wrote tiny_oracle.json")
