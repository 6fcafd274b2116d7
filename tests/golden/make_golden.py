"""Write the oracle's regression fixture for the tiny fp32 CCA workload.

The pages print no worked example, so this file stores values produced by the
CPU oracle alone (never by the CUDA path). It guards the oracle and the seeded
input generator against silent drift; the pins in test_oracle_pins.py are
what tie the oracle to the method itself.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402

ROWS = [0, 1, 3, 17, 40, 63]
COLS = [0, 5, 31, 64, 127]


def main():
    shape = workloads.WORKLOADS["tiny_cca_fp32"]
    inp = workloads.as_float64(workloads.make_inputs(shape))
    res = oracle.cca_block(inp, shape.n_q_heads, shape.n_kv_heads, shape.head_dim)
    fix = {
        "workload": shape.name,
        "source": "CPU float64 oracle (oracle/cca_oracle.py), seeded inputs from workloads.py",
        "rows": ROWS,
        "cols": COLS,
        "y": [[float(res["y"][0, r, c]) for c in COLS] for r in ROWS],
        "k_cache": [[float(res["k_cache"][0, r].reshape(-1)[c]) for c in (0, 7, 16, 31)] for r in ROWS],
        "v_cache": [[float(res["v_cache"][0, r].reshape(-1)[c]) for c in (0, 7, 16, 31)] for r in ROWS],
        "x_checksum": float(inp["x"].sum()),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_cca_fp32.json")
    with open(path, "w") as f:
        json.dump(fix, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
