"""The oracle still reproduces its stored tiny-workload fixture (CPU)."""
import os

import numpy as np

from top_routing_grouped_softmax_b200.synth import make_inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_oracle.txt")


def _parse():
    rec = {"ids": {}, "w": {}, "out": {}}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        tag, *rest = line.split()
        if tag in ("counts", "offsets"):
            rec[tag] = np.array([int(v) for v in rest])
        elif tag in ("ids", "w"):
            rec[tag][int(rest[0])] = np.array([float(v) for v in rest[1:]])
        elif tag == "out":
            rec[tag][int(rest[0])] = {int(c): float(v) for c, v in (p.split(":") for p in rest[1:])}
    return rec


def test_oracle_matches_golden(oracle):
    rec = _parse()
    inp = make_inputs("tiny")
    tokens = sorted(rec["out"])
    r, ex = oracle.forward(inp.bits("x"), inp.bits("W_router"), None, inp.bits("W_gate"),
                           inp.bits("W_up"), inp.bits("W_down"), 2, rows=np.array(tokens))
    pr = oracle.permute(r.ids, 8)
    assert np.array_equal(pr.counts, rec["counts"])
    assert np.array_equal(pr.offsets, rec["offsets"])
    for i, t in enumerate(tokens):
        assert np.array_equal(r.ids[t], rec["ids"][t].astype(np.int32))
        assert np.allclose(r.weights[t], rec["w"][t], rtol=1e-15, atol=0)
        for c, v in rec["out"][t].items():
            assert abs(ex.out[i, c] - v) <= 1e-15 * max(abs(v), 1e-30) + 1e-300
