"""Writes tests/golden/tiny_mixed_layer.json: frozen fp64 oracle outputs on a
tiny mixed layer (one ordinary and one replaced head).  Calls only the oracle
and the seeded input generator.

The replaced head follows Eq. (3) of "When Can Attention Heads Be Statically
Defined?" (reading notes, section 二.3); the ordinary head is causal softmax
attention (section 一 of the same page).  Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from mixed_head_causal_b200.inputs import Workload, make_inputs  # noqa: E402


def main():
    w = Workload("golden_b1_h2_t6_d4", B=1, H=2, T=6, d=4, fixed_replaced=(1,))
    x = make_inputs(w, seed=0)
    o, lse = oracle.fwd(x["q"], x["k"], x["v"], x["alpha"], x["rho"], x["mask"])
    dq, dk, dv = oracle.bwd(x["q"], x["k"], x["v"], x["do"], x["alpha"], x["rho"], x["mask"])

    def lst(t):
        return t.double().numpy().tolist()

    a = x["alpha"].double().nan_to_num(nan=0.0)  # ordinary rows are never read
    r = x["rho"].double().nan_to_num(nan=0.0)
    doc = {
        "source": "fp64 oracle (oracle/saf_oracle.c) via tests/golden/make_golden.py",
        "cites": "Eq. (3) and section 一 of 'When Can Attention Heads Be Statically Defined?' reading notes",
        "shape": {"B": 1, "H": 2, "T": 6, "d": 4, "replaced": [1]},
        "inputs": {"q": lst(x["q"]), "k": lst(x["k"]), "v": lst(x["v"]), "do": lst(x["do"]),
                   "alpha": lst(a), "rho": lst(r), "mask": lst(x["mask"])},
        "outputs": {"o": o.tolist(), "lse": lse.tolist(), "dq": dq.tolist(), "dk": dk.tolist(), "dv": dv.tolist()},
    }
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_mixed_layer.json")
    with open(out, "w") as f:
        json.dump(doc, f, indent=1)
    print("wrote", out)


if __name__ == "__main__":
    main()
