"""Writes c0_oracle.json: a frozen digest of the float64 oracle on the tiny
workload (1 layer, 2 heads x 64, 8 warmup chunks of 64 rows, seed 0).

The pages print no worked example with numbers, so this file does not pin the
oracle to the pages; it freezes the oracle so that any later change to its
arithmetic shows up as a failing test (tests/test_golden.py) and has to be
justified. It calls only ``oracle`` and the seeded input generator.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from ispa_synth import C0, layer_streams  # noqa: E402


def digest():
    st = layer_streams(C0, 0, seed=0)
    out = oracle.warmup_layer([st.chunk(c) for c in range(C0.n_chunks)], st.w)
    idx = [(0, 0), (5, 77), (127, 3), (64, 64)]
    rows = [0, 100, 511]
    return {
        "workload": "tiny: 1 layer, H=2, hd=64, sink 16, local 64, history 256, 8 chunks, seed 0",
        "lam": out["lam"],
        "eps": out["eps"],
        "err2": out["err2"],
        "G_fro": float(np.linalg.norm(out["G"])),
        "R_fro": float(np.linalg.norm(out["R"])),
        "S_fro": float(np.linalg.norm(out["S"])),
        "dW_fro": float(np.linalg.norm(out["dW"])),
        "G_entries": [float(out["G"][i, j]) for i, j in idx],
        "R_entries": [float(out["R"][i, j]) for i, j in idx],
        "dW_entries": [float(out["dW"][i, j]) for i, j in idx],
        "a_loc_rows": [[float(x) for x in out["a_loc"][r, :4]] for r in rows],
        "a_full_rows": [[float(x) for x in out["a_full"][r, :4]] for r in rows],
        "lse_full_chunk0": [float(x) for x in out["chunks"][0]["lse_full"][:, :4].ravel()],
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "c0_oracle.json"), "w") as f:
        json.dump(digest(), f, indent=1)
    print("wrote", os.path.join(HERE, "c0_oracle.json"))
