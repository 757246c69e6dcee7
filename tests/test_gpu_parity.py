"""Parity of the CUDA path (through the C ABI) with the oracle.

Kept node and leaf sets must be bit-exact.  Outputs: float32 within
1e-5 * max|y_ref| (max-abs), bfloat16 within 2e-2 max-abs on unit-scale
outputs; LSE within 1e-4 (float32) / 2e-3 (bfloat16, logits from bfloat16
inputs accumulated in fp32).  At the benchmark shapes the kept sets of every
traversal are compared with the oracle's descent, the outputs on 256 sampled
traversals, and every traversal is also checked by properties that hold at any
size (ascending, distinct, in range, nested).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from hierarchical_kv_pruning_b200 import synth
from hierarchical_kv_pruning_b200.binding import AtlaskvError, HikvpTree
from tests._util import oracle_inputs, oracle_tree, storage

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_fp32_10x10x10.npz")
BF16_TOL = 2e-2
LSE_TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-3}


def gpu_run(w, K, scale=0.0, tree=None, descent=0):
    own = tree is None
    if own:
        tree = HikvpTree.from_workload(w)
        tree.set_descent(descent)
    r = tree.attend(w.q_kg, w.q_seq, w.k_seq, w.v_seq, K, scale=scale)
    tree.sync_status()
    out = {k: (v.cpu() if torch.is_tensor(v) and k != "workspace" else v) for k, v in r.items()}
    if own:
        tree.close()
    return out


def to_device(w, device="cuda"):
    f = {}
    for name in ("root_keys", "mid_keys", "leaf_keys", "leaf_values", "root_child", "mid_child", "q_kg", "q_seq",
                 "k_seq", "v_seq", "targets"):
        v = getattr(w, name)
        f[name] = None if v is None else v.to(device)
    return synth.Workload(w.shape, **f)


def sample_traversals(B, H, n, seed=0):
    rng = np.random.default_rng(seed)
    pairs = {(0, 0), (B - 1, H - 1)}
    while len(pairs) < min(n, B * H):
        pairs.add((int(rng.integers(B)), int(rng.integers(H))))
    return sorted(pairs)


def compare(w, K, g, traversals=None, scale=None):
    sh = w.shape
    t = oracle_tree(w)
    inp = oracle_inputs(w)
    r = oracle.hikvp(t, inp["q_kg"], inp["q_seq"], inp["k_seq"], inp["v_seq"], K, traversals, scale)
    worst = 0.0
    for i, (b, h) in enumerate(r["traversals"]):
        assert g["kept_root"][b, h].tolist() == r["kept_root"][i].tolist(), ("root", b, h)
        assert g["kept_mid"][b, h].tolist() == r["kept_mid"][i].tolist(), ("mid", b, h)
        assert g["kept_leaf"][b, h].tolist() == r["kept_leaf"][i].tolist(), ("leaf", b, h)
        y = g["out"][b, :, h, :].double().numpy()
        err = np.max(np.abs(y - r["y"][i]))
        if sh.dtype == torch.float32:
            assert err <= 1e-5 * np.max(np.abs(r["y"][i])), (b, h, err)
        else:
            assert err <= BF16_TOL, (b, h, err)
        lerr = np.max(np.abs(g["lse"][b, :, h].double().numpy() - r["lse"][i]))
        assert lerr <= LSE_TOL[sh.dtype], (b, h, lerr)
        worst = max(worst, err)
    return worst


def check_structure(w, K, g):
    """Properties of every traversal: ascending distinct ids in range, nesting."""
    sh = w.shape
    bR, bI, bL = sh.fanout
    kr, km, kl = g["kept_root"], g["kept_mid"], g["kept_leaf"]
    for a, hi in ((kr, bR), (km, bR * bI), (kl, sh.n_leaves)):
        assert int(a.min()) >= 0 and int(a.max()) < hi
        assert bool((a[..., 1:] > a[..., :-1]).all())
    G = sh.group
    hkv = torch.arange(sh.n_heads) // G
    if w.root_child is None:
        parent_mid = km // bI
        parent_leaf = kl // bL
    else:
        inv_mid = torch.empty(sh.n_kv_heads, bR * bI, dtype=torch.int64)
        inv_leaf = torch.empty(sh.n_kv_heads, bR * bI * bL, dtype=torch.int64)
        rc, mc = w.root_child.cpu().long(), w.mid_child.cpu().long()
        for hk in range(sh.n_kv_heads):
            inv_mid[hk, rc[hk].flatten()] = torch.arange(bR).repeat_interleave(bI)
            inv_leaf[hk, mc[hk].flatten()] = torch.arange(bR * bI).repeat_interleave(bL)
        parent_mid = inv_mid[hkv[None, :, None].expand_as(km), km.long()]
        parent_leaf = inv_leaf[hkv[None, :, None].expand_as(kl), kl.long()]
    # every kept mid's parent is a kept root, every kept leaf's parent a kept mid
    assert bool((parent_mid[..., :, None] == kr[..., None, :].long()).any(-1).all())
    assert bool((parent_leaf[..., :, None] == km[..., None, :].long()).any(-1).all())
    assert torch.isfinite(g["out"].float()).all()


# ---------------------------------------------------------------------------

def test_tiny_fp32_matches_golden():
    gold = np.load(GOLDEN)
    sh = synth.shape(0)
    w = to_device(synth.make_workload(sh, "cpu", 1000))
    assert np.array_equal(storage(w.q_kg), gold["q_kg"])
    g = gpu_run(w, sh.keep)
    assert g["kept_root"][0, 0].tolist() == gold["kept_root"][0].tolist()
    assert g["kept_mid"][0, 0].tolist() == gold["kept_mid"][0].tolist()
    assert g["kept_leaf"][0, 0].tolist() == gold["kept_leaf"][0].tolist()
    y = g["out"][0, :, 0, :].double().numpy()
    assert np.max(np.abs(y - gold["y"][0])) <= 1e-5 * np.max(np.abs(gold["y"][0]))
    assert np.max(np.abs(g["lse"][0, :, 0].double().numpy() - gold["lse"][0])) <= 1e-4


SMALL = [
    # (dtype, H, H_kv, D, fanout, K, B, N, T, permuted)
    (torch.float32, 1, 1, 64, (10, 10, 10), (2, 2, 4), 1, 16, 16, False),
    (torch.float32, 4, 2, 128, (6, 5, 7), (3, 4, 9), 3, 5, 11, True),
    (torch.bfloat16, 4, 1, 64, (9, 8, 7), (3, 5, 20), 2, 16, 40, False),
    (torch.bfloat16, 8, 2, 128, (12, 11, 10), (4, 6, 17), 3, 20, 37, False),    # ragged N, T
    (torch.bfloat16, 6, 3, 128, (7, 9, 11), (2, 7, 33), 2, 33, 33, True),      # N = T, permuted
    (torch.bfloat16, 2, 1, 128, (5, 4, 3), (5, 20, 60), 2, 3, 70, False),      # full K: nothing pruned
    (torch.bfloat16, 32, 8, 128, (20, 20, 20), (8, 8, 32), 2, 128, 130, False),
    (torch.bfloat16, 32, 1, 128, (16, 16, 17), (16, 16, 64), 3, 32, 96, True),
    (torch.bfloat16, 4, 2, 128, (8, 8, 10), (3, 4, 20), 2, 200, 300, False),   # one head's rows in two row blocks
    (torch.bfloat16, 6, 2, 128, (10, 10, 12), (4, 9, 100), 2, 48, 50, True),   # row blocks cut heads; ragged leaf tile
    (torch.float32, 2, 2, 64, (30, 30, 9), (16, 200, 1000), 1, 1, 1, False),    # K above 128 and 1000 leaves
]


@pytest.mark.parametrize("case", SMALL, ids=[str(i) for i in range(len(SMALL))])
def test_small_trees(case):
    dtype, H, H_kv, D, fanout, K, B, N, T, perm = case
    sh = synth.custom(dtype=dtype, n_heads=H, n_kv_heads=H_kv, head_dim=D, fanout=fanout, keep=K, batch=B,
                      n_tokens=N, seq_len=T, permuted=perm)
    w = synth.make_workload(sh, "cuda", 4242)
    g = gpu_run(w, K)
    check_structure(w, K, g)
    compare(w, K, g)


# The bf16 tensor-core attention runs a persistent grid of two CTAs per SM over
# units of 128 query rows; these shapes have more units than a B200 has CTA
# slots (296), a ragged last round, and short units (one leaf tile, one or two
# sequence tiles), so a CTA crosses many unit boundaries: the Q switch to the
# next unit, O started afresh once the previous unit's O has been read.
PERSISTENT = [
    # (H, H_kv, N, T, B, D): N = 64 loads Q by TMA, N = 48 by cp.async (heads cut by row blocks)
    (8, 2, 64, 70, 80, 128),     # 320 units
    (6, 2, 48, 50, 100, 128),    # 400 units
    (8, 2, 64, 70, 80, 64),      # the same at D = 64 (one 64-column block per tile)
    (6, 2, 48, 50, 100, 64),
]


@pytest.mark.parametrize("case", PERSISTENT, ids=["q_tma", "q_cp_async", "q_tma_d64", "q_cp_async_d64"])
def test_persistent_attention_many_units(case):
    H, H_kv, N, T, B, D = case
    sh = synth.custom(dtype=torch.bfloat16, n_heads=H, n_kv_heads=H_kv, head_dim=D, fanout=(6, 6, 6),
                      keep=(3, 3, 9), batch=B, n_tokens=N, seq_len=T, permuted=True)
    w = synth.make_workload(sh, "cuda", 99)
    g = gpu_run(w, sh.keep)
    check_structure(w, sh.keep, g)
    compare(w, sh.keep, g, traversals=sample_traversals(B, H, 40, seed=3))
    # the same units through the host-leaf path: sequence part and knowledge
    # part as separate persistent launches, merged
    hw = synth.Workload(sh, w.root_keys, w.mid_keys, w.leaf_keys.cpu().pin_memory(),
                        w.leaf_values.cpu().pin_memory(), w.root_child, w.mid_child, w.q_kg, w.q_seq, w.k_seq,
                        w.v_seq, w.targets)
    same_as_hbm_path(g, gpu_run(hw, sh.keep))


def test_balanced_lambda_regime():
    # KG queries scaled so the KG and sequence log-sum-exps are comparable and
    # both lambda weights matter.
    sh = synth.custom(dtype=torch.bfloat16, n_heads=8, n_kv_heads=2, head_dim=128, fanout=(10, 10, 10),
                      keep=(4, 4, 16), batch=2, n_tokens=32, seq_len=64)
    w = synth.make_workload(sh, "cuda", 7)
    w.q_kg.mul_(0.15)
    g = gpu_run(w, sh.keep)
    compare(w, sh.keep, g)


def test_scale_argument():
    sh = synth.custom(dtype=torch.bfloat16, n_heads=4, n_kv_heads=1, head_dim=64, fanout=(6, 6, 6),
                      keep=(2, 3, 8), batch=2, n_tokens=16, seq_len=24)
    w = synth.make_workload(sh, "cuda", 8)
    g = gpu_run(w, sh.keep, scale=0.05)
    compare(w, sh.keep, g, scale=0.05)


DESCENTS = pytest.mark.parametrize("descent", [1, 2], ids=["fused", "parent_major"])


@DESCENTS
def test_all_keys_identical_mass_ties(descent):
    # Every score ties exactly; more ambiguous candidates than one refinement
    # chunk: the lowest row ids must win at every level (parent-major: the
    # selection's fallback and the queued exact tier).
    sh = synth.custom(dtype=torch.bfloat16, n_heads=2, n_kv_heads=1, head_dim=128, fanout=(40, 30, 20),
                      keep=(5, 70, 150), batch=2, n_tokens=4, seq_len=8, permuted=True)
    w = synth.make_workload(sh, "cuda", 9)
    for t in (w.root_keys, w.mid_keys, w.leaf_keys):
        t.copy_(w.leaf_keys[0, 0].expand_as(t))
    g = gpu_run(w, sh.keep, descent=descent)
    compare(w, sh.keep, g)
    assert g["kept_root"][0, 0].tolist() == list(range(5))


@DESCENTS
def test_zero_queries(descent):
    sh = synth.custom(dtype=torch.bfloat16, n_heads=2, n_kv_heads=1, head_dim=128, fanout=(8, 8, 8),
                      keep=(3, 5, 7), batch=2, n_tokens=4, seq_len=8)
    w = synth.make_workload(sh, "cuda", 10)
    w.q_kg.zero_()
    g = gpu_run(w, sh.keep, descent=descent)
    compare(w, sh.keep, g)
    assert g["kept_leaf"][0, 0].tolist() == list(range(7))


@DESCENTS
def test_near_ties_need_exact_arithmetic(descent):
    # Pairs of float32 keys that differ in one component by one unit in the
    # last place, and duplicated keys: the fp32 filter cannot order them,
    # exact arithmetic must.
    sh = synth.custom(dtype=torch.float32, n_heads=2, n_kv_heads=1, head_dim=64, fanout=(16, 8, 8),
                      keep=(5, 11, 23), batch=3, n_tokens=7, seq_len=9)
    w = synth.make_workload(sh, "cuda", 11)
    for keys in (w.root_keys, w.mid_keys, w.leaf_keys):
        k = keys[0]
        n = k.shape[0]
        for i in range(1, n, 2):
            k[i] = k[i - 1]
            j = i % sh.head_dim
            k[i, j] = torch.nextafter(k[i - 1, j], torch.tensor(float("inf"), device=k.device))
        for i in range(3, n, 7):
            k[i] = k[i - 3]
    g = gpu_run(w, sh.keep, descent=descent)
    compare(w, sh.keep, g)


def test_leaves_in_pinned_host_memory_small():
    sh = synth.custom(dtype=torch.bfloat16, n_heads=8, n_kv_heads=2, head_dim=128, fanout=(12, 10, 9),
                      keep=(3, 4, 16), batch=3, n_tokens=16, seq_len=48, permuted=True)
    w = synth.make_workload(sh, "cuda", 12)
    g_dev = gpu_run(w, sh.keep)
    hw = synth.Workload(sh, w.root_keys, w.mid_keys, w.leaf_keys.cpu().pin_memory(),
                        w.leaf_values.cpu().pin_memory(), w.root_child, w.mid_child, w.q_kg, w.q_seq, w.k_seq,
                        w.v_seq, w.targets)
    g_host = gpu_run(hw, sh.keep)
    same_as_hbm_path(g_dev, g_host)
    compare(w, sh.keep, g_host)


def test_leaves_in_pinned_host_memory_chunked():
    # B = 9 splits into four query chunks (2, 2, 2, 3) staged on a second stream
    # while the other chunks compute; kept sets equal the HBM-resident path's,
    # outputs to rounding.
    sh = synth.custom(dtype=torch.bfloat16, n_heads=8, n_kv_heads=2, head_dim=128, fanout=(12, 10, 9),
                      keep=(3, 4, 16), batch=9, n_tokens=16, seq_len=48, permuted=True)
    w = synth.make_workload(sh, "cuda", 15)
    g_dev = gpu_run(w, sh.keep)
    hw = synth.Workload(sh, w.root_keys, w.mid_keys, w.leaf_keys.cpu().pin_memory(),
                        w.leaf_values.cpu().pin_memory(), w.root_child, w.mid_child, w.q_kg, w.q_seq, w.k_seq,
                        w.v_seq, w.targets)
    g_host = gpu_run(hw, sh.keep)
    same_as_hbm_path(g_dev, g_host)
    compare(w, sh.keep, g_host)


def same_as_hbm_path(g_dev, g_host):
    """Host-resident leaves against the same workload in HBM: identical kept
    sets; the attention is the same softmax but runs as a sequence part merged
    with the knowledge part (host leaves) against one launch (HBM), so the
    outputs agree to rounding: within one bfloat16 ulp at unit scale."""
    for k in ("kept_root", "kept_mid", "kept_leaf"):
        assert torch.equal(g_dev[k], g_host[k]), k
    assert float((g_dev["out"].float() - g_host["out"].float()).abs().max()) <= 2 ** -7
    assert float((g_dev["lse"] - g_host["lse"]).abs().max()) <= 1e-4


def _host_levels(w, mids=True):
    """The same workload with the leaf keys and values (and the mid keys) in
    pinned host memory: only the root keys stay on the device."""
    return synth.Workload(w.shape, w.root_keys, w.mid_keys.cpu().pin_memory() if mids else w.mid_keys,
                          w.leaf_keys.cpu().pin_memory(), w.leaf_values.cpu().pin_memory(), w.root_child,
                          w.mid_child, w.q_kg, w.q_seq, w.k_seq, w.v_seq, w.targets)


@pytest.mark.parametrize("batch", [3, 9])   # one query chunk; four chunks (2, 2, 2, 3)
def test_mids_and_leaves_in_pinned_host_memory(batch):
    # Only the roots resident: the kept roots' mid blocks are staged before
    # level 1, the kept mids' leaf blocks before level 2; the kept sets equal
    # the HBM-resident path's, the outputs agree to rounding, and both match
    # the oracle.
    sh = synth.custom(dtype=torch.bfloat16, n_heads=8, n_kv_heads=2, head_dim=128, fanout=(12, 10, 9),
                      keep=(3, 4, 16), batch=batch, n_tokens=16, seq_len=48, permuted=True)
    w = synth.make_workload(sh, "cuda", 18 + batch)
    g_dev = gpu_run(w, sh.keep)
    g_host = gpu_run(_host_levels(w), sh.keep)
    same_as_hbm_path(g_dev, g_host)
    compare(w, sh.keep, g_host)


def _cached_runs(w_host, batches, blocks):
    """Run the batches in turn on one host-leaf tree with a leaf-block cache of
    `blocks` blocks (0: none); return the outputs and the cache counters."""
    outs = []
    with HikvpTree.from_workload(w_host) as tree:
        if blocks:
            tree.set_leaf_cache(blocks)
        for q in batches:
            r = tree.attend(q[0], q[1], q[2], q[3], w_host.shape.keep)
            tree.sync_status()
            outs.append({k: (v.cpu() if torch.is_tensor(v) and k != "workspace" else v) for k, v in r.items()})
        stats = tree.leaf_cache_stats() if blocks else None
    return outs, stats


@pytest.mark.parametrize("blocks", [4096, 8])   # room for every block; one set of 8 ways (evictions, bypasses)
def test_leaf_block_cache_gives_the_same_results(blocks):
    # Batches A, A, B, A on one tree: with the cache every output equals the
    # uncached path's, and the repeated batch finds its blocks in the cache.
    sh = synth.custom(dtype=torch.bfloat16, n_heads=8, n_kv_heads=2, head_dim=128, fanout=(12, 10, 9),
                      keep=(3, 4, 16), batch=9, n_tokens=16, seq_len=48, permuted=True)
    wa = synth.make_workload(sh, "cuda", 31)
    wb = synth.make_workload(sh, "cuda", 32)
    hw = _host_levels(wa, mids=False)
    qa = (wa.q_kg, wa.q_seq, wa.k_seq, wa.v_seq)
    qb = (wb.q_kg, wb.q_seq, wb.k_seq, wb.v_seq)
    plain, _ = _cached_runs(hw, [qa, qb], 0)
    got, stats = _cached_runs(hw, [qa, qa, qb, qa], blocks)
    for g, ref in zip(got, [plain[0], plain[0], plain[1], plain[0]]):
        for k in ("kept_root", "kept_mid", "kept_leaf", "out", "lse"):
            assert torch.equal(g[k], ref[k]), k
    compare(wa, sh.keep, got[1])
    assert stats["hits"] + stats["fills"] + stats["bypasses"] > 0
    if blocks == 4096:
        assert stats["hits"] > 0 and stats["hits"] >= stats["fills"]
    else:
        assert stats["bypasses"] > 0


def test_leaf_block_cache_needs_host_leaves():
    from hierarchical_kv_pruning_b200.binding import ATLASKV_EUNSUPPORTED
    sh = synth.custom(dtype=torch.bfloat16, n_heads=2, n_kv_heads=1, head_dim=128, fanout=(4, 4, 4),
                      keep=(2, 2, 2), batch=1, n_tokens=2, seq_len=2)
    w = synth.make_workload(sh, "cuda", 33)
    with HikvpTree.from_workload(w) as tree:
        with pytest.raises(AtlaskvError) as ei:
            tree.set_leaf_cache(64)
        assert ei.value.status == ATLASKV_EUNSUPPORTED


def test_host_mids_fp32_d64():
    sh = synth.custom(dtype=torch.float32, n_heads=2, n_kv_heads=1, head_dim=64, fanout=(9, 7, 5),
                      keep=(3, 5, 9), batch=2, n_tokens=5, seq_len=9)
    w = synth.make_workload(sh, "cuda", 21)
    g_host = gpu_run(_host_levels(w), sh.keep)
    compare(w, sh.keep, g_host)


def test_mids_on_host_need_leaves_on_host():
    from hierarchical_kv_pruning_b200.binding import ATLASKV_EINVAL
    sh = synth.custom(dtype=torch.bfloat16, n_heads=2, n_kv_heads=1, head_dim=128, fanout=(4, 4, 4),
                      keep=(2, 2, 2), batch=1, n_tokens=2, seq_len=2)
    w = synth.make_workload(sh, "cuda", 22)
    with pytest.raises(AtlaskvError) as ei:
        HikvpTree(w.root_keys, w.mid_keys.cpu().pin_memory(), w.leaf_keys, w.leaf_values, sh.fanout)
    assert ei.value.status == ATLASKV_EINVAL


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.bfloat16, 64), (torch.float32, 128)])
def test_decode_step_single_token(dtype, D):
    # A decode step: one query token (N = 1) attends to the T - 1 tokens
    # before it and to itself, and to its kept leaves.
    sh = synth.custom(dtype=dtype, n_heads=8, n_kv_heads=2, head_dim=D, fanout=(16, 12, 10),
                      keep=(4, 6, 24), batch=5, n_tokens=1, seq_len=77, permuted=True)
    w = synth.make_workload(sh, "cuda", 23)
    g = gpu_run(w, sh.keep)
    check_structure(w, sh.keep, g)
    compare(w, sh.keep, g)


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("n_tokens", [1, 24])
def test_layers_in_one_call_match_single_calls(n_tokens, D):
    # Several layers, each with its own tree and inputs, in one batched call:
    # every layer's results equal its own single call bit for bit and match
    # the oracle.
    from hierarchical_kv_pruning_b200.binding import attend_layers
    sh = synth.custom(dtype=torch.bfloat16, n_heads=8, n_kv_heads=2, head_dim=D, fanout=(10, 9, 8),
                      keep=(3, 5, 16), batch=6, n_tokens=n_tokens, seq_len=40)
    layers = [synth.make_workload(sh, "cuda", 30 + l) for l in range(4)]
    trees = [HikvpTree.from_workload(w) for w in layers]
    try:
        got = attend_layers(trees, [(w.q_kg, w.q_seq, w.k_seq, w.v_seq) for w in layers], sh.keep)
        for t in trees:
            t.sync_status()
        for l, (w, t) in enumerate(zip(layers, trees)):
            one = gpu_run(w, sh.keep, tree=t)
            for k in ("kept_root", "kept_mid", "kept_leaf", "out", "lse"):
                assert torch.equal(got[l][k].cpu(), one[k]), (l, k)
        compare(layers[1], sh.keep, {k: v.cpu() for k, v in got[1].items() if k != "workspace"})
    finally:
        for t in trees:
            t.close()


def test_layers_fp32_and_mismatch_rejected():
    from hierarchical_kv_pruning_b200.binding import ATLASKV_EINVAL, attend_layers
    sh = synth.custom(dtype=torch.float32, n_heads=2, n_kv_heads=1, head_dim=64, fanout=(6, 5, 4),
                      keep=(2, 3, 6), batch=2, n_tokens=3, seq_len=7)
    layers = [synth.make_workload(sh, "cuda", 40 + l) for l in range(2)]
    trees = [HikvpTree.from_workload(w) for w in layers]
    try:
        got = attend_layers(trees, [(w.q_kg, w.q_seq, w.k_seq, w.v_seq) for w in layers], sh.keep)
        for t in trees:
            t.sync_status()
        for l, w in enumerate(layers):
            compare(w, sh.keep, {k: v.cpu() for k, v in got[l].items() if k != "workspace"})
        w0, w1 = layers
        with pytest.raises(AtlaskvError) as ei:     # T differs between the layers
            attend_layers(trees, [(w0.q_kg, w0.q_seq, w0.k_seq, w0.v_seq),
                                  (w1.q_kg, w1.q_seq, w1.k_seq[:, :5].contiguous(), w1.v_seq[:, :5].contiguous())],
                          sh.keep)
        assert ei.value.status == ATLASKV_EINVAL
    finally:
        for t in trees:
            t.close()


@DESCENTS
def test_deterministic_and_b0(descent):
    # the parent-major path groups traversals with atomics: its results must
    # not depend on the order they land in
    sh = synth.custom(dtype=torch.bfloat16, n_heads=8, n_kv_heads=2, head_dim=128, fanout=(10, 10, 10),
                      keep=(3, 4, 16), batch=4, n_tokens=32, seq_len=64)
    w = synth.make_workload(sh, "cuda", 13)
    with HikvpTree.from_workload(w) as tree:
        tree.set_descent(descent)
        a = gpu_run(w, sh.keep, tree=tree)
        b = gpu_run(w, sh.keep, tree=tree)
        for k in ("kept_root", "kept_mid", "kept_leaf", "out", "lse"):
            assert torch.equal(a[k], b[k]), k
        e = tree.attend(w.q_kg[:0], w.q_seq[:0], w.k_seq[:0], w.v_seq[:0], sh.keep)
        tree.sync_status()
        assert e["out"].numel() == 0


def test_device_errors_are_reported():
    sh = synth.custom(dtype=torch.bfloat16, n_heads=2, n_kv_heads=1, head_dim=128, fanout=(4, 4, 4),
                      keep=(2, 2, 2), batch=1, n_tokens=2, seq_len=2, permuted=True)
    w = synth.make_workload(sh, "cuda", 14)
    bad = w.mid_child.clone()
    bad[0, 0, 0] = bad[0, 0, 1]          # not a permutation
    with pytest.raises(AtlaskvError) as ei:
        HikvpTree(w.root_keys, w.mid_keys, w.leaf_keys, w.leaf_values, sh.fanout, w.root_child, bad)
    assert ei.value.status == 1
    bad2 = w.root_child.clone()
    bad2[0, 1, 1] = 99                    # out of range
    with pytest.raises(AtlaskvError):
        HikvpTree(w.root_keys, w.mid_keys, w.leaf_keys, w.leaf_values, sh.fanout, bad2, w.mid_child)
    with HikvpTree.from_workload(w) as tree:
        small = torch.empty(256, dtype=torch.uint8, device="cuda")
        with pytest.raises(AtlaskvError) as ei:
            tree.attend(w.q_kg, w.q_seq, w.k_seq, w.v_seq, sh.keep, workspace=small)
        assert ei.value.status == 2
        with pytest.raises(AtlaskvError) as ei:
            tree.attend(w.q_kg, w.q_seq, w.k_seq, w.v_seq, (2, 9, 2))
        assert ei.value.status == 1



def test_attend_rejects_invalid_calls_without_side_effects():
    # Every host-side reject of the attend boundary returns EINVAL before
    # anything is enqueued; the caller's output buffers keep their contents and
    # the tree stays usable.
    from hierarchical_kv_pruning_b200.binding import ATLASKV_EINVAL
    sh = synth.custom(dtype=torch.bfloat16, n_heads=4, n_kv_heads=2, head_dim=128, fanout=(4, 4, 4),
                      keep=(2, 2, 2), batch=1, n_tokens=2, seq_len=3)
    w = synth.make_workload(sh, "cuda", 17)
    q, qs, k, v = w.q_kg, w.q_seq, w.k_seq, w.v_seq

    def misaligned(t):
        flat = torch.full((t.numel() + 8,), 7.0, dtype=t.dtype, device=t.device)
        m = flat[1:1 + t.numel()].view(t.shape)   # 2 bytes past a 16-byte boundary
        m.copy_(t)
        return m

    out = torch.full_like(q, 7.0)
    cases = [
        dict(K=(5, 2, 2)),                      # K_root > b_R
        dict(K=(0, 2, 2)),                      # K_root < 1
        dict(K=(2, 9, 2)),                      # K_mid > K_root b_I
        dict(K=(2, 2, 9)),                      # K_leaf > K_mid b_L
        dict(scale=-1.0),
        dict(scale=float("inf")),
        dict(q=q[:, :, :3].contiguous(), qs=qs[:, :, :3].contiguous()),   # H = 3 not a multiple of H_kv = 2
        dict(q=torch.cat([q, q], 1), qs=torch.cat([qs, qs], 1)),          # N = 4 > T = 3
        dict(q=misaligned(q)),
        dict(out=misaligned(torch.full_like(q, 7.0))),
    ]
    with HikvpTree.from_workload(w) as tree:
        for c in cases:
            qq, qqs = c.get("q", q), c.get("qs", qs)
            o = c.get("out", out if qq.shape == q.shape else torch.full_like(qq, 7.0))
            with pytest.raises(AtlaskvError) as ei:
                tree.attend(qq, qqs, k, v, c.get("K", sh.keep), scale=c.get("scale", 0.0), out=o)
            assert ei.value.status == ATLASKV_EINVAL, c
            torch.cuda.synchronize()
            assert bool((o.float() == 7.0).all()), c
        g = gpu_run(w, sh.keep, tree=tree)
    compare(w, sh.keep, g)


# ---- benchmark shapes at full size ----------------------------------------

@pytest.fixture(scope="module")
def full_cache():
    return {}


def compare_all_indices(w, K, g, cache=None):
    """Kept root, mid and leaf sets of EVERY traversal against the oracle's
    descent (bit-exact).  cache: a dict keeping the oracle's kept sets per
    workload name across calls."""
    sh = w.shape
    if cache is not None and sh.name in cache:
        kr, km, kl = cache[sh.name]
    else:
        t = oracle_tree(w)
        q = storage(w.q_kg)
        kr, km, kl = oracle.descend(t, q, K)
        if cache is not None:
            cache[sh.name] = (kr, km, kl)
    for name, ref in (("kept_root", kr), ("kept_mid", km), ("kept_leaf", kl)):
        got = g[name].reshape(sh.batch * sh.n_heads, -1).numpy()
        bad = np.nonzero((got != ref).any(axis=1))[0]
        assert bad.size == 0, (name, "traversals differ", [(int(i) // sh.n_heads, int(i) % sh.n_heads)
                                                          for i in bad[:8]], bad.size)


def gpu_run_profiled(w, K, descent=0):
    """gpu_run with the library's descent counters on: returns the outputs and
    per level the number of selections the fp32 band left open."""
    with HikvpTree.from_workload(w) as tree:
        tree.set_descent(descent)
        tree.set_profiling(True)
        g = gpu_run(w, K, tree=tree)
        stats = tree.refine_stats()
    return g, stats


@pytest.mark.parametrize("descent", ["fused", "parent_major"])
@pytest.mark.parametrize("i", [1, 2, 3])
def test_full_size_shapes(i, descent, full_cache):
    # both descents at the benchmark sizes: every traversal's kept sets
    sh = synth.shape(i)
    w = synth.make_workload(sh, "cuda", 1000 + i)
    g, stats = gpu_run_profiled(w, sh.keep, {"fused": 1, "parent_major": 2}[descent])
    print("refined selections per level (%s, %s):" % (sh.name, descent),
          {lvl: (v["refined"], v["exact_scores"]) for lvl, v in stats.items()})
    check_structure(w, sh.keep, g)
    compare_all_indices(w, sh.keep, g, full_cache)
    trav = sample_traversals(sh.batch, sh.n_heads, 256, seed=i)
    compare(w, sh.keep, g, trav)
    del w
    torch.cuda.empty_cache()


def test_full_size_host_leaves():
    sh = synth.shape(4)
    free_host = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_AVPHYS_PAGES")
    need = 2 * sh.n_leaves * sh.head_dim * 2 + (8 << 30)
    if free_host < need:
        pytest.skip("host memory %.0f GB below the %.0f GB the host-leaf shape needs" % (free_host / 1e9, need / 1e9))
    w = synth.make_workload(sh, "cuda", 1004)
    g, stats = gpu_run_profiled(w, sh.keep)
    print("refined selections per level (%s):" % sh.name,
          {lvl: (v["refined"], v["exact_scores"]) for lvl, v in stats.items()})
    check_structure(w, sh.keep, g)
    compare_all_indices(w, sh.keep, g)
    trav = sample_traversals(sh.batch, sh.n_heads, 256, seed=4)
    compare(w, sh.keep, g, trav)


def test_full_size_host_mids():
    # The host-leaf benchmark shape with the mid level in host memory too:
    # every output equals the host-leaf path's on the same buffers, and the
    # kept sets of a sample match the oracle.
    sh = synth.shape("host_mids")
    free_host = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_AVPHYS_PAGES")
    need = 2 * sh.n_leaves * sh.head_dim * 2 + (8 << 30)
    if free_host < need:
        pytest.skip("host memory %.0f GB below the %.0f GB the host-leaf shape needs" % (free_host / 1e9, need / 1e9))
    w = synth.make_workload(sh, "cuda", 1004)
    assert not w.mid_keys.is_cuda and w.mid_keys.is_pinned()
    g_mids = gpu_run(w, sh.keep)
    w_dev_mids = synth.Workload(sh, w.root_keys, w.mid_keys.cuda(), w.leaf_keys, w.leaf_values, None, None,
                                w.q_kg, w.q_seq, w.k_seq, w.v_seq, w.targets)
    g_leaves = gpu_run(w_dev_mids, sh.keep)
    for k in ("kept_root", "kept_mid", "kept_leaf", "out", "lse"):
        assert torch.equal(g_mids[k], g_leaves[k]), k
    check_structure(w, sh.keep, g_mids)
    trav = sample_traversals(sh.batch, sh.n_heads, 256, seed=5)
    compare(w, sh.keep, g_mids, trav)


def test_bounded_device_wait_reports_timeout():
    # A device wait that can never complete gives up after its iteration limit
    # and the host reads ETIMEOUT from the tree's status word; the context
    # stays usable (a fresh tree still attends correctly afterwards).
    import time
    sh = synth.custom(dtype=torch.bfloat16, n_heads=2, n_kv_heads=1, head_dim=128, fanout=(4, 4, 4),
                      keep=(2, 2, 2), batch=1, n_tokens=2, seq_len=2)
    w = synth.make_workload(sh, "cuda", 16)
    with HikvpTree.from_workload(w) as tree:
        t0 = time.time()
        tree.probe_wait_timeout()
        with pytest.raises(AtlaskvError) as ei:
            tree.sync_status()
        assert ei.value.status == 5           # ATLASKV_ETIMEOUT
        assert time.time() - t0 < 60
    g = gpu_run(w, sh.keep)
    compare(w, sh.keep, g)


# ---- trees of any depth with variable numbers of children (CSR) ------------

def _csr_oracle(w):
    return oracle.CsrTree([storage(k) for k in w.keys], storage(w.leaf_values),
                          [o.cpu().numpy() for o in w.child_off],
                          [None if c is None else c.cpu().numpy() for c in w.child_id])


def _compare_csr(w, K, g, traversals=None):
    from hierarchical_kv_pruning_b200.binding import CsrHikvpTree  # noqa: F401
    sh = w.shape
    inp = dict(q_kg=storage(w.q_kg), q_seq=storage(w.q_seq), k_seq=storage(w.k_seq), v_seq=storage(w.v_seq))
    r = oracle.hikvp_csr(_csr_oracle(w), inp["q_kg"], inp["q_seq"], inp["k_seq"], inp["v_seq"], K, traversals)
    for i, (b, h) in enumerate(r["traversals"]):
        for l in range(len(K)):
            assert g["kept"][l][b, h].tolist() == r["kept"][l][i].tolist(), ("level", l, b, h)
        y = g["out"][b, :, h, :].double().numpy()
        err = np.max(np.abs(y - r["y"][i]))
        if sh.dtype == torch.float32:
            assert err <= 1e-5 * np.max(np.abs(r["y"][i])), (b, h, err)
        else:
            assert err <= BF16_TOL, (b, h, err)
        assert np.max(np.abs(g["lse"][b, :, h].double().numpy() - r["lse"][i])) <= LSE_TOL[sh.dtype]


CSR_CASES = [
    # (dtype, H, H_kv, D, n_roots, fan-out ranges, K per level, B, N, T, permuted)
    (torch.bfloat16, 8, 2, 128, 12, ((3, 9),), (4, 12), 3, 16, 40, False),                  # depth 2
    (torch.bfloat16, 8, 2, 128, 20, ((2, 12), (3, 15)), (6, 10, 24), 3, 24, 50, True),      # depth 3, permuted
    (torch.bfloat16, 32, 1, 128, 16, ((4, 9), (2, 7), (3, 6)), (5, 9, 12, 30), 2, 8, 20, True),   # depth 4, G = 32
    (torch.float32, 4, 2, 64, 10, ((1, 6), (2, 5)), (3, 3, 6), 2, 5, 9, False),             # fp32, single children
]


@pytest.mark.parametrize("case", CSR_CASES, ids=[str(i) for i in range(len(CSR_CASES))])
def test_csr_trees(case):
    from hierarchical_kv_pruning_b200.binding import CsrHikvpTree
    dtype, H, H_kv, D, n_roots, ranges, K, B, N, T, perm = case
    sh = synth.CsrShape("csr", dtype, H, H_kv, D, n_roots, ranges, K, B, N, T, permuted=perm)
    w = synth.make_csr_workload(sh, "cuda", 91)
    with CsrHikvpTree.from_workload(w) as tree:
        tree.set_profiling(times=False, counters=True)
        g = tree.attend(w.q_kg, w.q_seq, w.k_seq, w.v_seq, K)
        tree.sync_status()
        assert tree.refine_stats()["root"]["selections"] == B * H
    g = {"out": g["out"].cpu(), "lse": g["lse"].cpu(), "kept": [k.cpu() for k in g["kept"]]}
    _compare_csr(w, K, g)


def test_uniform_tree_as_csr_matches_the_uniform_path():
    from hierarchical_kv_pruning_b200.binding import CsrHikvpTree
    sh = synth.custom(dtype=torch.bfloat16, n_heads=8, n_kv_heads=2, head_dim=128, fanout=(12, 10, 9),
                      keep=(3, 5, 16), batch=3, n_tokens=16, seq_len=48, permuted=True)
    w = synth.make_workload(sh, "cuda", 92)
    g_u = gpu_run(w, sh.keep)
    bR, bI, bL = sh.fanout
    off0 = (torch.arange(bR + 1, dtype=torch.int32, device="cuda") * bI).expand(2, -1).contiguous()
    off1 = (torch.arange(bR * bI + 1, dtype=torch.int32, device="cuda") * bL).expand(2, -1).contiguous()
    ids0 = w.root_child.reshape(2, -1).contiguous()
    ids1 = w.mid_child.reshape(2, -1).contiguous()
    with CsrHikvpTree([w.root_keys, w.mid_keys, w.leaf_keys], w.leaf_values, [off0, off1], [ids0, ids1]) as t:
        g_c = t.attend(w.q_kg, w.q_seq, w.k_seq, w.v_seq, sh.keep)
        t.sync_status()
    for l, name in enumerate(("kept_root", "kept_mid", "kept_leaf")):
        assert torch.equal(g_c["kept"][l].cpu(), g_u[name]), name
    assert torch.equal(g_c["out"].cpu(), g_u["out"]) and torch.equal(g_c["lse"].cpu(), g_u["lse"])


def test_csr_rejects_bad_offsets_and_too_large_K():
    from hierarchical_kv_pruning_b200.binding import ATLASKV_EINVAL, CsrHikvpTree
    sh = synth.CsrShape("bad", torch.bfloat16, 2, 1, 128, 6, ((2, 4), (1, 3)), (2, 2, 2), 1, 2, 3)
    w = synth.make_csr_workload(sh, "cuda", 93)
    bad = w.child_off[0].clone()
    bad[0, 2] = bad[0, 3] + 1                    # decreasing offsets
    with pytest.raises(AtlaskvError) as ei:
        CsrHikvpTree(w.keys, w.leaf_values, [bad, w.child_off[1]])
    assert ei.value.status == ATLASKV_EINVAL
    fewest = int((w.child_off[1][:, 1:] - w.child_off[1][:, :-1]).min())
    with CsrHikvpTree.from_workload(w) as t:
        # level 2 asks for more leaves than 2 kept mids with the fewest children have
        with pytest.raises(AtlaskvError) as ei:
            t.attend(w.q_kg, w.q_seq, w.k_seq, w.v_seq, (2, 2, 2 * fewest + 1))
        assert ei.value.status == ATLASKV_EINVAL
        g = t.attend(w.q_kg, w.q_seq, w.k_seq, w.v_seq, (2, 2, 2 * fewest))
        t.sync_status()
