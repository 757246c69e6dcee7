"""Pins for the oracle's descent on trees of any depth with a variable number of
children per node ("Method details / Hierarchical clustering of KGKVs": the
clusters are of unequal size and the depth can be set larger).

* A uniform three-level tree written in CSR form must give exactly the kept
  sets of the three-level oracle (pinned on its own by brute force).
* Brute force on tiny variable trees of depth 2, 3 and 4: every level's kept
  set holds the K highest exact scores (Python fractions) of that level's
  candidates, which are the children of the level above's kept nodes; ties go
  to the lower row; kept sets come back ascending.
* With every node kept, the whole path equals attention over all leaves and
  the visible sequence (the rectangular-attention form).
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from hierarchical_kv_pruning_b200 import synth
from tests._util import oracle_tree, storage


def csr_tree(w) -> oracle.CsrTree:
    return oracle.CsrTree([storage(k) for k in w.keys], storage(w.leaf_values),
                          [o.cpu().numpy() for o in w.child_off],
                          [None if c is None else c.cpu().numpy() for c in w.child_id])


def uniform_as_csr(w) -> oracle.CsrTree:
    """A three-level uniform workload written as a CSR tree."""
    sh = w.shape
    bR, bI, bL = sh.fanout
    Hkv = sh.n_kv_heads
    off0 = np.tile(np.arange(bR + 1, dtype=np.int32) * bI, (Hkv, 1))
    off1 = np.tile(np.arange(bR * bI + 1, dtype=np.int32) * bL, (Hkv, 1))
    ids0 = None if w.root_child is None else w.root_child.cpu().numpy().reshape(Hkv, -1)
    ids1 = None if w.mid_child is None else w.mid_child.cpu().numpy().reshape(Hkv, -1)
    return oracle.CsrTree([storage(w.root_keys), storage(w.mid_keys), storage(w.leaf_keys)],
                          storage(w.leaf_values), [off0, off1], [ids0, ids1])


@pytest.mark.parametrize("dtype,permuted", [(torch.float32, False), (torch.bfloat16, True)])
def test_uniform_tree_in_csr_form_matches_the_three_level_oracle(dtype, permuted):
    sh = synth.custom(dtype=dtype, n_heads=4, n_kv_heads=2, head_dim=16, fanout=(5, 4, 6), keep=(1, 1, 1),
                      batch=3, n_tokens=3, seq_len=3, permuted=permuted)
    w = synth.make_workload(sh, "cpu", 51)
    t3, tc = oracle_tree(w), uniform_as_csr(w)
    q = storage(w.q_kg)
    for K in [(1, 1, 1), (2, 5, 9), (5, 20, 120), (3, 7, 30), (4, 4, 4)]:
        kr, km, kl = oracle.descend(t3, q, K)
        got = oracle.descend_csr(tc, q, K)
        assert np.array_equal(got[0], kr) and np.array_equal(got[1], km) and np.array_equal(got[2], kl), K


def _frac_scores(tree, level, q_kg, b, h, rows):
    H = q_kg.shape[2]
    hkv = h // (H // tree.n_kv_heads)
    q = oracle.widen(q_kg[b, :, h, :])
    keys = tree.keys[level]
    out = []
    for r in rows:
        k = oracle.widen(keys[hkv, r])
        out.append(sum(Fraction(float(q[n, d])) * Fraction(float(k[d]))
                       for n in range(q.shape[0]) for d in range(q.shape[1])))
    return out


def _check_level(cands, kept, scores, K):
    kept = list(kept)
    assert len(kept) == K and kept == sorted(kept) and len(set(kept)) == K
    assert set(kept) <= set(cands)
    sc = dict(zip(cands, scores))
    for i in kept:
        for j in set(cands) - set(kept):
            assert sc[i] > sc[j] or (sc[i] == sc[j] and i < j), (i, j)


def _check_descent(tree, q_kg, K, b, h, kept):
    H = q_kg.shape[2]
    hkv = h // (H // tree.n_kv_heads)
    cands = list(range(tree.rows[0]))
    for l in range(tree.n_levels):
        _check_level(cands, kept[l], _frac_scores(tree, l, q_kg, b, h, cands), K[l])
        if l + 1 < tree.n_levels:
            cands = [int(c) for p in kept[l] for c in tree.children(l, hkv, int(p))]


SHAPES = [
    # (n_roots, fan-out ranges per level, K per level, permuted)
    (6, ((2, 5),), (2, 4), False),                        # depth 2: roots and leaves
    (5, ((1, 4), (2, 5)), (2, 3, 5), True),               # depth 3, unequal clusters, permuted rows
    (4, ((2, 3), (1, 3), (2, 4)), (2, 3, 3, 6), True),    # depth 4
    (3, ((3, 3), (1, 1), (2, 2)), (1, 2, 2, 4), False),   # a level of single children
]


@pytest.mark.parametrize("case", SHAPES, ids=[str(i) for i in range(len(SHAPES))])
def test_brute_force_on_variable_trees(case):
    n_roots, ranges, K, perm = case
    sh = synth.CsrShape("tiny", torch.bfloat16, 4, 2, 8, n_roots, ranges, K, 2, 2, 3, permuted=perm)
    w = synth.make_csr_workload(sh, "cpu", 61)
    t = csr_tree(w)
    q = storage(w.q_kg)
    kept = oracle.descend_csr(t, q, K)
    for i, (b, h) in enumerate(itertools.product(range(2), range(4))):
        _check_descent(t, q, K, b, h, [k[i] for k in kept])


def test_every_level_kept_equals_attention_over_all_leaves():
    sh = synth.CsrShape("full", torch.float32, 2, 1, 8, 3, ((2, 4), (1, 3)), (1, 1, 1), 2, 3, 5)
    w = synth.make_csr_workload(sh, "cpu", 71)
    t = csr_tree(w)
    K = tuple(w.rows)     # every node is a candidate and kept at every level
    inp = dict(q_kg=storage(w.q_kg), q_seq=storage(w.q_seq), k_seq=storage(w.k_seq), v_seq=storage(w.v_seq))
    r = oracle.hikvp_csr(t, inp["q_kg"], inp["q_seq"], inp["k_seq"], inp["v_seq"], K)
    for l in range(t.n_levels):
        assert (r["kept"][l] == np.arange(w.rows[l])).all()
    # rectangular attention by hand: one softmax over all leaves and the visible sequence
    scale = 1.0 / np.sqrt(8)
    lk, lv = oracle.widen(t.leaf_keys[0]), oracle.widen(storage(w.leaf_values)[0])
    for i, (b, h) in enumerate(r["traversals"]):
        qk, qs = oracle.widen(inp["q_kg"][b, :, h]), oracle.widen(inp["q_seq"][b, :, h])
        ks, vs = oracle.widen(inp["k_seq"][b, :, 0]), oracle.widen(inp["v_seq"][b, :, 0])
        for n in range(3):
            vis = 5 - 3 + n + 1
            logits = np.concatenate([lk @ qk[n] * scale, ks[:vis] @ qs[n] * scale])
            p = np.exp(logits - logits.max())
            y = (p[:len(lk)] @ lv + p[len(lk):] @ vs[:vis]) / p.sum()
            assert np.allclose(r["y"][i, n], y, rtol=0, atol=1e-12)
            assert abs(r["lse"][i, n] - (logits.max() + np.log(p.sum()))) < 1e-12


def test_ties_go_to_lower_rows_and_too_few_candidates_rejected():
    sh = synth.CsrShape("ties", torch.float32, 1, 1, 4, 4, ((1, 3), (2, 2)), (2, 2, 3), 1, 2, 2)
    w = synth.make_csr_workload(sh, "cpu", 81)
    for k in w.keys:
        k.copy_(torch.tensor([1.0, -2.0, 0.5, 4.0]).expand_as(k))
    t = csr_tree(w)
    q = storage(w.q_kg)
    kept = oracle.descend_csr(t, q, (2, 2, 3))
    assert kept[0].tolist() == [[0, 1]]
    mids = sorted(int(c) for p in (0, 1) for c in t.children(0, 0, p))
    assert kept[1].tolist() == [mids[:2]]
    leaves = sorted(int(c) for p in kept[1][0] for c in t.children(1, 0, int(p)))
    assert kept[2].tolist() == [leaves[:3]]
    with pytest.raises(ValueError):
        oracle.descend_csr(t, q, (1, 1, 99))     # more leaves asked for than any traversal has
