"""Write the stored expectations under tests/golden/ from the CPU oracle only.

Run from the repository root:  python tests/golden/make_golden.py
The pages print no worked example, so these files are regression fixtures of
the pinned oracle (kept-tile lists and a few output values for the tiny fp32
workload, seed 0), not values taken from the pages.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import ssta_inputs as si  # noqa: E402


def main():
    w = si.get_workload("tiny_f32")
    x = si.make_inputs(w, seed=0)
    arrs = [x[k].double().numpy() if x[k] is not None else None
            for k in ("q", "k", "v", "q_text", "k_text", "v_text")]
    r = oracle.ssta_forward(w, *arrs)
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_f32_seed0.txt")
    with open(out, "w") as f:
        f.write("# tiny_f32 workload, seed 0: written by tests/golden/make_golden.py (CPU oracle only)\n")
        f.write("# kept b h query_tile : ascending kept key-tile ids\n")
        B, H, NQ = r["kv_cnt"].shape
        for b in range(B):
            for h in range(H):
                for i in range(NQ):
                    ids = r["kv_idx"][b, h, i, : r["kv_cnt"][b, h, i]]
                    f.write(f"kept {b} {h} {i} : {' '.join(str(int(j)) for j in ids)}\n")
        f.write("# lse b h packed_row value ; o b h packed_row channel value (float64, %.17g)\n")
        for (b, h, row) in [(0, 0, 0), (0, 0, 37), (0, 1, 100), (0, 1, 255)]:
            f.write(f"lse {b} {h} {row} {r['LSE'][b, h, row]:.17g}\n")
            for c in (0, 63, 127):
                f.write(f"o {b} {h} {row} {c} {r['O'][b, h, row, c]:.17g}\n")
    print("wrote", out)


if __name__ == "__main__":
    main()
