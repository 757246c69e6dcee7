"""The seeded generator: tree shapes, pooling of interior keys ("Method details
/ Hierarchical clustering of KGKVs": every higher-level key pools the keys
below it), child tables, determinism."""
import numpy as np
import pytest
import torch

from hierarchical_kv_pruning_b200 import synth


@pytest.mark.parametrize("permuted", [False, True])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_interior_keys_are_subtree_means(permuted, dtype):
    sh = synth.custom(dtype=dtype, n_heads=4, n_kv_heads=2, head_dim=16, fanout=(4, 3, 5),
                      batch=3, n_tokens=2, seq_len=5, permuted=permuted)
    w = synth.make_workload(sh, "cpu", 4)
    bR, bI, bL = sh.fanout
    tol = 1e-6 if dtype == torch.float32 else 2 ** -7
    for hk in range(2):
        for r in range(bR):
            mids = [int(m) for m in (w.root_child[hk, r] if permuted else range(r * bI, (r + 1) * bI))]
            leaves_all = []
            for m in mids:
                leaves = [int(x) for x in (w.mid_child[hk, m] if permuted else range(m * bL, (m + 1) * bL))]
                leaves_all += leaves
                mean = w.leaf_keys[hk, leaves].double().mean(0)
                assert torch.allclose(w.mid_keys[hk, m].double(), mean, rtol=tol, atol=tol)
            mean = w.leaf_keys[hk, leaves_all].double().mean(0)
            assert torch.allclose(w.root_keys[hk, r].double(), mean, rtol=tol, atol=tol)


def test_child_tables_are_permutations():
    sh = synth.custom(dtype=torch.bfloat16, n_heads=2, n_kv_heads=1, head_dim=8, fanout=(5, 4, 3),
                      permuted=True)
    w = synth.make_workload(sh, "cpu", 2)
    assert sorted(w.root_child[0].flatten().tolist()) == list(range(20))
    assert sorted(w.mid_child[0].flatten().tolist()) == list(range(60))


@pytest.mark.parametrize("i", [0, 1])
def test_shapes_and_determinism(i):
    sh = synth.shape(i)
    w = synth.make_workload(sh, "cpu", 1000 + i)
    bR, bI, bL = sh.fanout
    assert w.root_keys.shape == (sh.n_kv_heads, bR, sh.head_dim)
    assert w.mid_keys.shape == (sh.n_kv_heads, bR * bI, sh.head_dim)
    assert w.leaf_keys.shape == (sh.n_kv_heads, bR * bI * bL, sh.head_dim)
    assert w.q_kg.shape == (sh.batch, sh.n_tokens, sh.n_heads, sh.head_dim)
    assert w.k_seq.shape == (sh.batch, sh.seq_len, sh.n_kv_heads, sh.head_dim)
    assert all(t.dtype == sh.dtype for t in (w.root_keys, w.leaf_values, w.q_seq, w.v_seq))
    w2 = synth.make_workload(sh, "cpu", 1000 + i)
    assert torch.equal(w.q_kg, w2.q_kg) and torch.equal(w.leaf_keys, w2.leaf_keys)


def test_queries_sit_near_their_target_leaf():
    sh = synth.shape(0)
    w = synth.make_workload(sh, "cpu", 1000)
    t = int(w.targets[0, 0])
    d = (w.q_kg[0, :, 0].double() - w.leaf_keys[0, t].double()).std()
    assert 0.05 < float(d) < 0.2


def test_benchmark_shapes_match_their_descriptions():
    s = synth.SHAPES
    assert s[0].n_leaves == 1000 and s[0].keep == (2, 2, 4) and s[0].dtype == torch.float32
    assert s[1].n_leaves == 47 ** 3 and s[1].keep == (8, 8, 32) and s[1].batch == 16
    assert s[2].n_leaves == 10 ** 6 and s[2].seq_len == 1024 and s[2].n_tokens == 64
    assert s[3].n_leaves == 215 * 215 * 216 and s[3].permuted and s[3].n_kv_heads == 1
    assert s[4].n_leaves == 125_000_000 and s[4].leaf_on_host and s[4].keep == (8, 8, 64)
