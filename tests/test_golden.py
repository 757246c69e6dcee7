"""The stored oracle outputs for the tiny float32 workload (written by
tests/golden/make_golden.py from the oracle alone) still match the generator
and the oracle; the GPU parity test reuses the same file."""
import os

import numpy as np

import oracle
from hierarchical_kv_pruning_b200 import synth
from tests._util import oracle_inputs, oracle_tree

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_fp32_10x10x10.npz")


def test_golden_tiny_fp32():
    g = np.load(GOLDEN)
    sh = synth.shape(0)
    w = synth.make_workload(sh, "cpu", 1000)
    inp = oracle_inputs(w)
    assert np.array_equal(inp["q_kg"], g["q_kg"]), "generator drifted"
    r = oracle.hikvp(oracle_tree(w), inp["q_kg"], inp["q_seq"], inp["k_seq"], inp["v_seq"], sh.keep)
    for k in ("kept_root", "kept_mid", "kept_leaf"):
        assert np.array_equal(r[k], g[k])
    assert np.max(np.abs(r["y"] - g["y"])) < 1e-13
    assert np.max(np.abs(r["lse"] - g["lse"])) < 1e-13
