"""Pins for the oracle's greedy descent ("Quick read / How it works": keep the
top-K branches at the roots, load the next level's keys, prune level by level).

Brute force on tiny trees: for every level the kept set must hold exactly the K
highest exact scores of that level's candidate set (ties to the lower row id),
the candidate set must be the children of the previous level's kept nodes, and
kept sets must come back in ascending row order.  Scores here are recomputed
with Python fractions, independently of the oracle's C accumulator.
"""
import itertools
import random
from fractions import Fraction

import pytest
import torch

import oracle
from hierarchical_kv_pruning_b200 import synth
from tests._util import oracle_tree, storage


def _frac_scores(tree, level, q_kg, b, h, rows):
    keys = [tree.root_keys, tree.mid_keys, tree.leaf_keys][level]
    H = q_kg.shape[2]
    hkv = h // (H // tree.n_kv_heads)
    q = oracle.widen(q_kg[b, :, h, :])
    out = []
    for r in rows:
        k = oracle.widen(keys[hkv, r])
        out.append(sum(Fraction(float(q[n, d])) * Fraction(float(k[d]))
                       for n in range(q.shape[0]) for d in range(q.shape[1])))
    return out


def _check_level(cands, kept, scores, K):
    cands = list(cands)
    kept = list(kept)
    assert len(kept) == K
    assert kept == sorted(kept), "kept rows must be ascending"
    assert len(set(kept)) == K
    assert set(kept) <= set(cands)
    sc = dict(zip(cands, scores))
    out = [c for c in cands if c not in set(kept)]
    for i in kept:
        for j in out:
            assert sc[i] > sc[j] or (sc[i] == sc[j] and i < j), (i, j, sc[i], sc[j])


def _check_descent(tree, q_kg, K, b, h, kr, km, kl):
    H = q_kg.shape[2]
    hkv = h // (H // tree.n_kv_heads)
    roots = list(range(tree.fanout[0]))
    _check_level(roots, kr, _frac_scores(tree, 0, q_kg, b, h, roots), K[0])
    mids = [int(c) for p in kr for c in tree.children(0, hkv, int(p))]
    _check_level(mids, km, _frac_scores(tree, 1, q_kg, b, h, mids), K[1])
    leaves = [int(c) for p in km for c in tree.children(1, hkv, int(p))]
    _check_level(leaves, kl, _frac_scores(tree, 2, q_kg, b, h, leaves), K[2])


def _tiny(fanout, dtype, permuted, seed, H=2, H_kv=1, N=2, D=8):
    sh = synth.custom(dtype=dtype, n_heads=H, n_kv_heads=H_kv, head_dim=D, fanout=fanout,
                      keep=(1, 1, 1), batch=2, n_tokens=N, seq_len=N, permuted=permuted)
    return synth.make_workload(sh, "cpu", seed)


@pytest.mark.parametrize("dtype,permuted", [(torch.float32, False), (torch.bfloat16, False),
                                            (torch.bfloat16, True)])
def test_all_k_on_3x3x3(dtype, permuted):
    w = _tiny((3, 3, 3), dtype, permuted, seed=7)
    t = oracle_tree(w)
    q = storage(w.q_kg)
    for K_R in range(1, 4):
        for K_I in range(1, 3 * K_R + 1):
            for K_L in range(1, 3 * K_I + 1, 2):
                kr, km, kl = oracle.descend(t, q, (K_R, K_I, K_L))
                for i, (b, h) in enumerate(itertools.product(range(2), range(2))):
                    _check_descent(t, q, (K_R, K_I, K_L), b, h, kr[i], km[i], kl[i])


@pytest.mark.parametrize("K", [(1, 1, 1), (2, 3, 5), (4, 16, 64), (3, 5, 11), (4, 4, 4)])
def test_4x4x4_grouped_heads(K):
    w = _tiny((4, 4, 4), torch.bfloat16, True, seed=11, H=4, H_kv=2, N=3, D=16)
    t = oracle_tree(w)
    q = storage(w.q_kg)
    kr, km, kl = oracle.descend(t, q, K)
    for i, (b, h) in enumerate(itertools.product(range(2), range(4))):
        _check_descent(t, q, K, b, h, kr[i], km[i], kl[i])


def test_ties_go_to_lower_row():
    # Every key identical: all exact scores tie, so the lowest row ids win at
    # every level (and children of the kept parents are the lowest children).
    sh = synth.custom(dtype=torch.float32, n_heads=1, n_kv_heads=1, head_dim=4, fanout=(3, 4, 5),
                      batch=1, n_tokens=2, seq_len=2)
    w = synth.make_workload(sh, "cpu", 3)
    for t in (w.root_keys, w.mid_keys, w.leaf_keys):
        t.copy_(torch.tensor([1.0, -2.0, 0.5, 4.0]).expand_as(t))
    tree = oracle_tree(w)
    kr, km, kl = oracle.descend(tree, storage(w.q_kg), (2, 3, 7))
    assert kr.tolist() == [[0, 1]]
    assert km.tolist() == [[0, 1, 2]]
    assert kl.tolist() == [[0, 1, 2, 3, 4, 5, 6]]


def test_duplicated_keys_tie_break_and_zero_query():
    sh = synth.custom(dtype=torch.bfloat16, n_heads=1, n_kv_heads=1, head_dim=8, fanout=(4, 2, 2),
                      batch=1, n_tokens=1, seq_len=1)
    w = synth.make_workload(sh, "cpu", 5)
    e = torch.eye(8)
    # root 3 duplicates root 1; the query points at them: scores (0, 1, 0, 1).
    w.root_keys[0] = torch.stack([e[0], e[1], e[2], e[1]])
    w.q_kg[0, 0, 0] = e[1]
    tree = oracle_tree(w)
    q = storage(w.q_kg)
    sc = oracle.level_scores(tree, 0, q, 0, 0, [0, 1, 2, 3])
    assert sc[1] == sc[3] > sc[0] == sc[2] == 0
    assert oracle.descend(tree, q, (1, 1, 1))[0].tolist() == [[1]]
    assert oracle.descend(tree, q, (2, 1, 1))[0].tolist() == [[1, 3]]
    assert oracle.descend(tree, q, (3, 1, 1))[0].tolist() == [[0, 1, 3]]
    # all-zero query: every score is exactly zero -> lowest rows everywhere
    w.q_kg.zero_()
    kr, km, kl = oracle.descend(oracle_tree(w), storage(w.q_kg), (2, 2, 3))
    assert kr.tolist() == [[0, 1]] and km.tolist() == [[0, 1]] and kl.tolist() == [[0, 1, 2]]


def test_known_winner_by_construction():
    # Fan-out (3, 2, 2): root r has mids 2r, 2r+1; mid m has leaves 2m, 2m+1.
    # Keys are basis directions, the query is 3 e2 + 2 e4 + e7, so by hand:
    # roots score (0, 0, 3), mids 4/5 (children of root 2) score (0, 2),
    # leaves 10/11 (children of mid 5) score (0, 1).
    D = 8
    sh = synth.custom(dtype=torch.float32, n_heads=1, n_kv_heads=1, head_dim=D, fanout=(3, 2, 2),
                      batch=1, n_tokens=1, seq_len=1)
    w = synth.make_workload(sh, "cpu", 1)
    e = torch.eye(D)
    w.root_keys[0] = e[:3]
    w.mid_keys[0] = e[5].expand(6, D)
    w.mid_keys[0, 4] = e[3]
    w.mid_keys[0, 5] = e[4]
    w.leaf_keys[0] = e[0].expand(12, D)
    w.leaf_keys[0, 10] = e[6]
    w.leaf_keys[0, 11] = e[7]
    w.q_kg[0, 0, 0] = 3 * e[2] + 2 * e[4] + e[7]
    tree = oracle_tree(w)
    q = storage(w.q_kg)
    assert [a.tolist() for a in oracle.descend(tree, q, (1, 1, 1))] == [[[2]], [[5]], [[11]]]
    # K = 2 everywhere: the zero-score ties go to the lowest row ids:
    # roots {2, 0}; mids {5} + lowest zero among children {0, 1, 4} -> 0;
    # leaves {11} + lowest zero among children of mids 0 and 5 -> 0.
    assert [a.tolist() for a in oracle.descend(tree, q, (2, 2, 2))] == [[[0, 2]], [[0, 5]], [[0, 11]]]
    # two tokens summing to the same direction give the same answer
    w2 = synth.make_workload(synth.custom(dtype=torch.float32, n_heads=1, n_kv_heads=1, head_dim=D,
                                          fanout=(3, 2, 2), batch=1, n_tokens=2, seq_len=2), "cpu", 1)
    for a, b in ((w2.root_keys, w.root_keys), (w2.mid_keys, w.mid_keys), (w2.leaf_keys, w.leaf_keys)):
        a.copy_(b)
    w2.q_kg[0, 0, 0] = 2 * e[2] + 3 * e[4] - e[7]
    w2.q_kg[0, 1, 0] = e[2] - 1 * e[4] + 2 * e[7]
    assert [a.tolist() for a in oracle.descend(oracle_tree(w2), storage(w2.q_kg), (1, 1, 1))] == [[[2]], [[5]], [[11]]]


def test_rejects_k_above_candidates():
    w = _tiny((3, 3, 3), torch.float32, False, seed=1)
    with pytest.raises(ValueError):
        oracle.descend(oracle_tree(w), storage(w.q_kg), (4, 1, 1))
    with pytest.raises(ValueError):
        oracle.descend(oracle_tree(w), storage(w.q_kg), (1, 4, 1))
    with pytest.raises(ValueError):
        oracle.descend(oracle_tree(w), storage(w.q_kg), (1, 1, 4))


# ---- randomized sweep, checked against the definition written out directly ----

def _children_from_tables(w, level, hkv, p):
    """Children of node p of `level`, read straight off the workload's child
    tables (or the implicit layout p * fan-out + j), not through the oracle."""
    fo = w.shape.fanout[level + 1]
    tab = w.root_child if level == 0 else w.mid_child
    if tab is None:
        return [p * fo + j for j in range(fo)]
    return [int(x) for x in tab[hkv, p].tolist()]


def _greedy_by_definition(w, K, b, h):
    """Kept sets of one traversal: at each level sort the candidates by exact
    score (descending) then row id, keep the first K, report them ascending.
    The exact score is (sum over tokens of q) . k, in rationals."""
    sh = w.shape
    hkv = h // (sh.n_heads // sh.n_kv_heads)
    q = w.q_kg[b, :, h, :].double()
    s = [sum(Fraction(float(q[n, d])) for n in range(q.shape[0])) for d in range(q.shape[1])]
    kept, cands = [], list(range(sh.fanout[0]))
    for level, keys in enumerate((w.root_keys, w.mid_keys, w.leaf_keys)):
        if level > 0:
            cands = [c for p in kept[-1] for c in _children_from_tables(w, level - 1, hkv, p)]
        k = keys[hkv].double()
        score = {r: sum(s[d] * Fraction(float(k[r, d])) for d in range(len(s))) for r in cands}
        ranked = sorted(cands, key=lambda r: (-score[r], r))
        kept.append(sorted(ranked[:K[level]]))
    return kept


@pytest.mark.parametrize("seed", range(24))
def test_random_trees_match_the_greedy_definition(seed):
    rng = random.Random(seed)
    fanout = tuple(rng.randint(2, 5) for _ in range(3))
    H_kv, G = rng.choice([1, 2, 2]), rng.choice([1, 2, 3])
    K_R = rng.randint(1, fanout[0])
    K_I = rng.randint(1, K_R * fanout[1])
    K_L = rng.randint(1, K_I * fanout[2])
    sh = synth.custom(dtype=rng.choice([torch.float32, torch.bfloat16]), n_heads=G * H_kv, n_kv_heads=H_kv,
                      head_dim=rng.choice([4, 8]), fanout=fanout, keep=(K_R, K_I, K_L), batch=2,
                      n_tokens=rng.randint(1, 3), seq_len=3, permuted=rng.random() < 0.7)
    w = synth.make_workload(sh, "cpu", 100 + seed)
    # exact ties: copy a few key rows onto others at every level
    for keys in (w.root_keys, w.mid_keys, w.leaf_keys):
        for _ in range(2):
            a, c = rng.randrange(keys.shape[1]), rng.randrange(keys.shape[1])
            keys[:, c] = keys[:, a]
    kr, km, kl = oracle.descend(oracle_tree(w), storage(w.q_kg), sh.keep)
    for i, (b, h) in enumerate(itertools.product(range(2), range(sh.n_heads))):
        got = [kr[i].tolist(), km[i].tolist(), kl[i].tolist()]
        assert got == _greedy_by_definition(w, sh.keep, b, h), (seed, b, h)


def test_ranking_across_a_borrow():
    # x0 = 2^a - 20 u comes from two products of opposite sign in two digits of
    # the exact accumulator (2^a at bit 0 of a digit, -20 u = -5 u 2^2 in the
    # digit below); x1 = 2^a - 16 u is one product inside the lower digit.  The
    # ranking must put x1 above x0 (u = 2^(a - 22)).
    a = (-oracle.exact_origin()) % 32
    while a < 22:
        a += 32
    u = 2.0 ** (a - 22)
    sh = synth.custom(dtype=torch.float32, n_heads=1, n_kv_heads=1, head_dim=4, fanout=(3, 1, 1),
                      batch=1, n_tokens=1, seq_len=1)
    w = synth.make_workload(sh, "cpu", 2)
    w.root_keys[0] = torch.tensor([[2.0 ** a, -20 * u, 0, 0], [2.0 ** a - 16 * u, 0, 0, 0], [0, 0, 0, 0]])
    w.q_kg[0, 0, 0] = torch.tensor([1.0, 1.0, 0, 0])
    tree, q = oracle_tree(w), storage(w.q_kg)
    assert oracle.descend(tree, q, (1, 1, 1))[0].tolist() == [[1]]
    assert oracle.descend(tree, q, (2, 1, 1))[0].tolist() == [[0, 1]]
