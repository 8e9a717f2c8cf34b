"""Writes tests/golden/oracle_tiny_step.json: an oracle regression fixture.

The pages print no worked numeric example, so this file holds no published value.
It records the CPU oracle's own output on the seeded tiny workload (fp32, 1
request, ctx 64, K=8, one Mamba-2 and one attention layer) so that any later change
to the oracle's arithmetic or to the input generators is visible.  It calls only
the oracle and the seeded input generators.  Regenerate with
    python tests/golden/make_golden.py
and name, in the commit, the passage of the H-Spec pages (or its reading) that
justifies the change.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from hybrid_mamba_attention_b200 import inputs as I  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_step.json")


def compute():
    wl = I.WORKLOADS["tiny"]
    st = I.make_step_inputs(wl)
    res = oracle.draft_step(wl.shapes, st["weights"], st["kv"], st["h_last"], st["ctx_lens"],
                            x_in=st["x_in"])
    h = res["hidden"]
    idx = [(0, 0, 0), (0, 3, 17), (0, 7, 255), (0, 5, 128)]
    return {
        "workload": wl.description,
        "source": "CPU oracle regression fixture (no published values exist on the pages)",
        "hidden_shape": list(h.shape),
        "hidden_sum": float(h.sum()),
        "hidden_sumsq": float((h ** 2).sum()),
        "samples": [{"index": list(i), "value": float(h[i])} for i in idx],
    }


if __name__ == "__main__":
    with open(OUT, "w") as f:
        json.dump(compute(), f, indent=1)
    print(OUT)
