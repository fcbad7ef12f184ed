"""The oracle reproduces its frozen regression fixtures (tests/golden)."""
import json
import os

import numpy as np
import pytest

import workloads
from oracle import oracle as orc

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
FILES = sorted(f for f in os.listdir(HERE) if f.startswith("golden_") and f.endswith(".json"))


@pytest.mark.parametrize("fname", FILES)
def test_oracle_matches_fixture(fname, oracle_lib):
    with open(os.path.join(HERE, fname)) as f:
        doc = json.load(f)
    p = doc["workload"]
    wl = workloads.Workload(fname[:-5], p["B"], p["H"], p["d_c"], p["d_r"], p["L"], p["g"], p["w"],
                            p["dtype"], p["q_scale"], p["kv_scale"], seed=p["seed"])
    x = workloads.generate(wl, threads=1)
    res = orc.lca(x.q_c, x.q_r, x.c_kv, x.k_r, g=wl.g, w=wl.w, lib=oracle_lib)
    dense = orc.mla(x.q_c, x.q_r, x.c_kv, x.k_r, lib=oracle_lib)
    want = np.array([[float.fromhex(v) for v in row] for row in doc["lca_out"]])
    want_d = np.array([[float.fromhex(v) for v in row] for row in doc["mla_out"]])
    np.testing.assert_allclose(res.out[0], want, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(dense[0], want_d, rtol=1e-13, atol=1e-15)
    assert res.anchor[0].tolist() == doc["lca_anchor"]
