"""Writes the stored expected actions under tests/golden/ from the fp64 oracle.

The pages print no worked numeric example for the action expert, so these fixtures are
the oracle's own output on seeded synthetic inputs: they freeze the oracle against
accidental drift and give GPU tests an expected value without recomputation. Only
``oracle`` and the input generator are called here.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O  # noqa: E402
from vla_inputs import get, make_inputs  # noqa: E402

NAMES = ["tiny", "mid_pi0_b3", "mid_ada_b2", "mid_d128"]


def expected_actions(name):
    wl = get(name)
    inp = make_inputs(wl)
    st = None if inp["state"] is None else inp["state"].astype(np.float64)
    return O.denoise(wl.expert, O.decode_params(inp["params"]), inp["noise"].astype(np.float64),
                     st, O.bf16_to_f64(inp["prefix_k"]), O.bf16_to_f64(inp["prefix_v"]), wl.steps)


def main():
    for name in NAMES:
        a = expected_actions(name)
        path = os.path.join(HERE, f"{name}_actions.json")
        with open(path, "w") as f:
            json.dump({"workload": name, "source": "oracle.denoise (fp64), seeded inputs",
                       "shape": list(a.shape), "actions": [float(v) for v in a.ravel()]}, f)
            f.write("\n")
        print("wrote", path, a.shape)


if __name__ == "__main__":
    main()
