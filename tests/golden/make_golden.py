"""Write tests/golden/tiny_regression.json from the oracle alone.

The pages print no worked example, so this fixture is a regression snapshot
of the pinned oracle on a tiny seeded workload (prefill, 40 tokens, H_I=4,
H=8, k=8): it fails if the oracle's arithmetic drifts.  It imports only the
oracle and the seeded input generator.  Run from the repository root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from sparse_attention_weight_b200 import inputs  # noqa: E402
from sparse_attention_weight_b200.configs import Workload  # noqa: E402

WL = Workload("golden_tiny", 94, "prefill", k=8, h_index=4, heads=8, seq_len=40)


def compute():
    ins = inputs.make_inputs(WL)
    b = ins["batch"]
    r = oracle.forward(b.kv_offset, b.kv_len, b.q_seq, b.q_pos, ins["q_idx"], ins["k_idx"], ins["w"],
                       ins["q"], ins["kv"], WL.k, WL.sm_scale)
    return {
        "workload": {"cfg_id": WL.cfg_id, "seq_len": WL.seq_len, "h_index": WL.h_index,
                     "heads": WL.heads, "k": WL.k, "seed": 0},
        "idx": [list(map(int, r)) for r in r["idx"]],
        "scores_row39": [float(v) for v in r["scores"][39]],
        "out_row39_head0_first8": [float(v) for v in r["out"][39, 0, :8]],
        "lse_row39": [float(v) for v in r["lse"][39]],
    }


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_regression.json")
    with open(path, "w") as f:
        json.dump(compute(), f, indent=1)
    print("wrote", path)
