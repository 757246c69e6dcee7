"""The two ways of running the descent give the same results.

The fused kernel (one CTA per query, KV head and chunk of heads, every level)
and the parent-major kernels (kept parents grouped by (KV head, parent) over
the whole batch, each parent's child rows read once per group of traversals)
must produce bit-identical kept sets, outputs and LSEs, and both must match
the oracle.  The cases cover every dtype / head size, permuted and CSR trees of
depth 2 to 4, host-resident levels with one and several query chunks, parents
kept by more traversals than one work item holds, and more (KV head, parent)
keys than one scan tile.
"""
import numpy as np
import pytest
import torch

from hierarchical_kv_pruning_b200 import synth
from hierarchical_kv_pruning_b200.binding import (ATLASKV_DESCENT_FUSED, ATLASKV_DESCENT_PARENT_MAJOR, CsrHikvpTree,
                                                  HikvpTree)
from tests.test_gpu_parity import _compare_csr, _host_levels, check_structure, compare, gpu_run

pytestmark = pytest.mark.gpu
MODES = (ATLASKV_DESCENT_FUSED, ATLASKV_DESCENT_PARENT_MAJOR)


def run_mode(w, K, mode):
    with HikvpTree.from_workload(w) as tree:
        tree.set_descent(mode)
        return gpu_run(w, K, tree=tree)


def same(a, b):
    for k in ("kept_root", "kept_mid", "kept_leaf", "out", "lse"):
        assert torch.equal(a[k], b[k]), k


CASES = [
    # (dtype, H, H_kv, D, fanout, K, B, N, T, permuted)
    (torch.float32, 4, 2, 128, (6, 5, 7), (3, 4, 9), 3, 5, 11, True),          # fp32 D 128: 8 heads per warp
    (torch.float32, 2, 2, 64, (30, 30, 9), (16, 200, 1000), 1, 1, 1, False),   # K above 128, 1000 leaves
    (torch.bfloat16, 4, 1, 64, (9, 8, 7), (3, 5, 20), 2, 16, 40, False),       # bf16 D 64
    (torch.bfloat16, 6, 3, 128, (7, 9, 11), (2, 7, 33), 2, 33, 33, True),
    (torch.bfloat16, 2, 1, 128, (5, 4, 3), (5, 20, 60), 2, 3, 70, False),      # nothing pruned
    (torch.bfloat16, 32, 1, 128, (6, 12, 9), (4, 10, 40), 4, 8, 16, True),     # ~85 traversals per root: split items
    (torch.bfloat16, 8, 2, 128, (64, 40, 8), (6, 12, 30), 3, 8, 24, False),    # 2560 mids per KV head: 3 scan tiles
    (torch.bfloat16, 32, 8, 128, (20, 20, 20), (8, 8, 32), 5, 64, 130, False),
]


@pytest.mark.parametrize("case", CASES, ids=[str(i) for i in range(len(CASES))])
def test_uniform_trees_both_descents(case):
    dtype, H, H_kv, D, fanout, K, B, N, T, perm = case
    sh = synth.custom(dtype=dtype, n_heads=H, n_kv_heads=H_kv, head_dim=D, fanout=fanout, keep=K, batch=B,
                      n_tokens=N, seq_len=T, permuted=perm)
    w = synth.make_workload(sh, "cuda", 5151)
    g = [run_mode(w, K, m) for m in MODES]
    same(g[0], g[1])
    check_structure(w, K, g[1])
    compare(w, K, g[1])


CSR = [
    (torch.bfloat16, 8, 2, 128, 12, ((3, 9),), (4, 12), 3, 16, 40, False),
    (torch.bfloat16, 8, 2, 128, 20, ((2, 12), (3, 15)), (6, 10, 24), 3, 24, 50, True),
    (torch.bfloat16, 32, 1, 128, 16, ((4, 9), (2, 7), (3, 6)), (5, 9, 12, 30), 2, 8, 20, True),
    (torch.float32, 4, 2, 64, 10, ((1, 6), (2, 5)), (3, 3, 6), 2, 5, 9, False),
]


@pytest.mark.parametrize("case", CSR, ids=[str(i) for i in range(len(CSR))])
def test_csr_trees_both_descents(case):
    dtype, H, H_kv, D, n_roots, ranges, K, B, N, T, perm = case
    sh = synth.CsrShape("csr", dtype, H, H_kv, D, n_roots, ranges, K, B, N, T, permuted=perm)
    w = synth.make_csr_workload(sh, "cuda", 97)
    got = []
    for m in MODES:
        with CsrHikvpTree.from_workload(w) as tree:
            tree.set_descent(m)
            r = tree.attend(w.q_kg, w.q_seq, w.k_seq, w.v_seq, K)
            tree.sync_status()
            got.append({"out": r["out"].cpu(), "lse": r["lse"].cpu(), "kept": [k.cpu() for k in r["kept"]]})
    for l in range(len(K)):
        assert torch.equal(got[0]["kept"][l], got[1]["kept"][l]), l
    assert torch.equal(got[0]["out"], got[1]["out"]) and torch.equal(got[0]["lse"], got[1]["lse"])
    _compare_csr(w, K, got[1])


@pytest.mark.parametrize("mids", [False, True])
@pytest.mark.parametrize("batch", [3, 9])   # one query chunk; four chunks
def test_host_levels_both_descents(mids, batch):
    sh = synth.custom(dtype=torch.bfloat16, n_heads=8, n_kv_heads=2, head_dim=128, fanout=(10, 12, 14),
                      keep=(3, 5, 20), batch=batch, n_tokens=24, seq_len=48, permuted=True)
    w = synth.make_workload(sh, "cuda", 77)
    hw = _host_levels(w, mids)
    g = [run_mode(hw, sh.keep, m) for m in MODES]
    same(g[0], g[1])
    compare(w, sh.keep, g[1])


def test_parent_major_rejects_nothing_the_fused_accepts_at_benchmark_K():
    # the workspace of the parent-major plan is larger; both sizes are positive
    sh = synth.shape(1)
    small = synth.custom(dtype=sh.dtype, n_heads=sh.n_heads, n_kv_heads=sh.n_kv_heads, head_dim=sh.head_dim,
                         fanout=(12, 12, 12), keep=sh.keep, batch=2, n_tokens=4, seq_len=8)
    w = synth.make_workload(small, "cuda", 3)
    sizes = []
    for m in MODES:
        with HikvpTree.from_workload(w) as tree:
            tree.set_descent(m)
            sizes.append(tree.workspace_size(small.keep, 2, 4, sh.n_heads, 8))
    assert sizes[0] > 0 and sizes[1] > sizes[0]
    np.testing.assert_equal(len(sizes), 2)
