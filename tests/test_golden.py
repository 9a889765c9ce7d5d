"""The oracle reproduces its stored regression fixture (tests/golden/)."""
import os

import numpy as np

import oracle
import ssta_inputs as si

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_f32_seed0.txt")


def load_golden():
    kept, lse, o = {}, {}, {}
    with open(GOLD) as f:
        lines = f.read().splitlines()
    for line in lines:
        if line.startswith("#") or not line.strip():
            continue
        parts = line.split()
        if parts[0] == "kept":
            b, h, i = map(int, parts[1:4])
            kept[(b, h, i)] = [int(t) for t in parts[5:]]
        elif parts[0] == "lse":
            lse[tuple(map(int, parts[1:4]))] = float(parts[4])
        elif parts[0] == "o":
            o[tuple(map(int, parts[1:5]))] = float(parts[5])
    return kept, lse, o


def test_oracle_matches_golden():
    kept, lse, o = load_golden()
    w = si.get_workload("tiny_f32")
    x = si.make_inputs(w, seed=0)
    r = oracle.ssta_forward(w, *[x[k].double().numpy() if x[k] is not None else None
                                 for k in ("q", "k", "v", "q_text", "k_text", "v_text")])
    for (b, h, i), ids in kept.items():
        assert list(r["kv_idx"][b, h, i, : r["kv_cnt"][b, h, i]]) == ids
    for (b, h, row), val in lse.items():
        assert abs(r["LSE"][b, h, row] - val) < 1e-12
    for (b, h, row, c), val in o.items():
        assert abs(r["O"][b, h, row, c] - val) < 1e-12
