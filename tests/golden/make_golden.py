"""Writes tests/golden/tiny_recurrence.json from the fp64 oracle only.

The fixture is a regression pin: it freezes the oracle's output on one tiny
seeded case (T=12, H=2, G=1, P=2, N=3, with initial state) so that any later
change to the oracle's arithmetic shows up in ``test_golden_fixture``.
Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from ssd_inputs import make_inputs  # noqa: E402


def main():
    inp = make_inputs(batch=1, seqlen=12, nheads=2, headdim=2, ngroups=1, dstate=3,
                      dtype="f32", dt_dist="loguniform", initial_states=True, seed=42)
    y, final, _ = oracle.recurrence(**inp)
    out = {
        "what": "SSD recurrence, fp64 oracle output on seeded fp32 inputs (seed 42)",
        "inputs": {k: v.double().numpy().tolist() for k, v in inp.items()},
        "y": y.tolist(),
        "final_states": final.tolist(),
    }
    with open(os.path.join(HERE, "tiny_recurrence.json"), "w") as fh:
        json.dump(out, fh)


if __name__ == "__main__":
    main()
