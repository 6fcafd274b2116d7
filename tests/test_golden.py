"""The oracle and the seeded generator still give the stored tiny-workload values."""
import json
import os

import numpy as np

import oracle
import workloads

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_workload_matches_stored_oracle_values():
    with open(os.path.join(HERE, "golden", "tiny_cca_fp32.json")) as f:
        fix = json.load(f)
    shape = workloads.WORKLOADS[fix["workload"]]
    inp = workloads.as_float64(workloads.make_inputs(shape))
    assert abs(float(inp["x"].sum()) - fix["x_checksum"]) < 1e-9
    res = oracle.cca_block(inp, shape.n_q_heads, shape.n_kv_heads, shape.head_dim)
    rows, cols = fix["rows"], fix["cols"]
    np.testing.assert_allclose(res["y"][0][np.ix_(rows, cols)], fix["y"], rtol=1e-12, atol=1e-15)
    kc = res["k_cache"][0].reshape(shape.seq_len, -1)[np.ix_(rows, [0, 7, 16, 31])]
    np.testing.assert_allclose(kc, fix["k_cache"], rtol=1e-12, atol=1e-15)
    vc = res["v_cache"][0].reshape(shape.seq_len, -1)[np.ix_(rows, [0, 7, 16, 31])]
    np.testing.assert_allclose(vc, fix["v_cache"], rtol=1e-12, atol=1e-15)
