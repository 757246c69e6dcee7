"""Writes tests/golden/tiny_fp32_10x10x10.npz: the oracle's kept sets and
outputs for the tiny float32 workload (10x10x10 tree, D=64, N=T=16, K=2/2/4,
seed 1000).  Inputs come from the seeded generator; every expected value comes
from ``oracle`` alone.  Run: python tests/golden/make_golden.py"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from hierarchical_kv_pruning_b200 import synth  # noqa: E402
from tests._util import oracle_inputs, oracle_tree  # noqa: E402


def main():
    sh = synth.shape(0)
    w = synth.make_workload(sh, "cpu", 1000)
    inp = oracle_inputs(w)
    r = oracle.hikvp(oracle_tree(w), inp["q_kg"], inp["q_seq"], inp["k_seq"], inp["v_seq"], sh.keep)
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_fp32_10x10x10.npz")
    np.savez(out, kept_root=r["kept_root"], kept_mid=r["kept_mid"], kept_leaf=r["kept_leaf"],
             y=r["y"], lse=r["lse"], q_kg=inp["q_kg"])
    print("wrote", out)


if __name__ == "__main__":
    main()
