"""Write tests/golden/tiny_oracle.txt from the fp64 oracle alone.

The pages print no worked example, so this fixture records what the oracle
gives on the tiny workload (T=256, d=256, E=8, top-2, f=512, seed 0 of the
seeded recipe).  It guards the oracle against unnoticed changes to its
arithmetic; the oracle's correctness itself is pinned by tests/oracle_pins.py.

Run:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle.oracle import default_oracle  # noqa: E402
from top_routing_grouped_softmax_b200.synth import make_inputs  # noqa: E402

TOKENS = [0, 1, 2, 3, 100, 255]
COLS = [0, 1, 2, 3, 127, 255]


def main(path=os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.txt")):
    inp = make_inputs("tiny")
    o = default_oracle()
    r, ex = o.forward(inp.bits("x"), inp.bits("W_router"), None, inp.bits("W_gate"),
                      inp.bits("W_up"), inp.bits("W_down"), inp.cfg.k,
                      rows=np.array(TOKENS, np.int64))
    pr = o.permute(r.ids, inp.cfg.E)
    lines = ["# fp64 oracle on the tiny workload (T=256 d=256 E=8 k=2 f=512, seed 0)",
             "# written by tests/golden/make_golden.py from oracle/ only"]
    lines.append("counts " + " ".join(str(int(c)) for c in pr.counts))
    lines.append("offsets " + " ".join(str(int(c)) for c in pr.offsets))
    for t in TOKENS:
        lines.append(f"ids {t} " + " ".join(str(int(e)) for e in r.ids[t]))
        lines.append(f"w {t} " + " ".join(f"{w:.17e}" for w in r.weights[t]))
    for i, t in enumerate(TOKENS):
        lines.append(f"out {t} " + " ".join(f"{c}:{ex.out[i, c]:.17e}" for c in COLS))
    with open(path, "w") as fh:
        fh.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
