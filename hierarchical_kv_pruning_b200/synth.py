"""Seeded synthetic HiKVP workloads.

This module only draws inputs: it holds none of the hot path's arithmetic and
imports neither the CUDA library nor the oracle, so both can be fed from it.

The recipe follows the workload descriptions of the five benchmark shapes and
the tree construction of "AtlasKV: Augmenting LLMs with Billion-Scale Knowledge
Graphs in 20GB VRAM", section "Method details / Hierarchical clustering of
KGKVs" (three levels, every higher-level key is a pooling of the keys below it;
here the pooling is the mean of the subtree's stored leaf keys):

* root centroids ~ N(0, 1)^D; mid centroid = parent + 0.5 N(0, 1);
  leaf key = mid centroid + 0.25 N(0, 1), rounded to the storage type;
* stored interior key = mean of its subtree's stored leaf keys, taken in
  float64 and rounded once to the storage type;
* leaf values ~ N(0, 1);
* one target leaf per (query b, KV head), uniform over the M leaves; every KG
  query token of every head of that KV group = target key + 0.1 N(0, 1);
* sequence Q/K/V ~ N(0, 1);
* optional random row permutations of the mid and leaf levels with explicit
  child tables (non-coalesced gathers).

The pages evaluate on a knowledge-graph test set that is not available here;
these seeded inputs stand in for it with the benchmark shapes.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Shape:
    name: str
    dtype: torch.dtype
    n_heads: int          # H query heads
    n_kv_heads: int       # H_kv
    head_dim: int         # D
    fanout: tuple         # (b_R, b_I, b_L)
    keep: tuple           # (K_R, K_I, K_L)
    batch: int            # B independent queries
    n_tokens: int         # N query tokens per query
    seq_len: int          # T causal sequence length (query tokens are the last N)
    permuted: bool = False
    leaf_on_host: bool = False
    mid_on_host: bool = False     # mid keys in pinned host memory too (only the roots stay on the device)

    @property
    def n_leaves(self) -> int:
        b0, b1, b2 = self.fanout
        return b0 * b1 * b2

    @property
    def group(self) -> int:
        return self.n_heads // self.n_kv_heads


SHAPES = {
    0: Shape("tiny_fp32_10x10x10", torch.float32, 1, 1, 64, (10, 10, 10), (2, 2, 4), 1, 16, 16),
    1: Shape("gqa_bf16_47x47x47", torch.bfloat16, 32, 8, 128, (47, 47, 47), (8, 8, 32), 16, 128, 512),
    2: Shape("gqa_bf16_100x100x100", torch.bfloat16, 32, 8, 128, (100, 100, 100), (16, 16, 64), 64, 64, 1024),
    3: Shape("mqa_bf16_215x215x216_permuted", torch.bfloat16, 32, 1, 128, (215, 215, 216), (16, 16, 64),
             256, 32, 256, permuted=True),
    4: Shape("mqa_bf16_500x500x500_host_leaves", torch.bfloat16, 32, 1, 128, (500, 500, 500), (8, 8, 64),
             256, 32, 256, leaf_on_host=True),
}


# Variants of the benchmark shapes that exercise a further part of the path.
VARIANTS = {
    # the 500x500x500 host-leaf shape with the mid level in host memory as well:
    # only the roots stay resident ("Quick read / How it works")
    "host_mids": Shape("mqa_bf16_500x500x500_host_mids", torch.bfloat16, 32, 1, 128, (500, 500, 500), (8, 8, 64),
                       256, 32, 256, leaf_on_host=True, mid_on_host=True),
}


def shape(i) -> Shape:
    """Benchmark shape i (0..4), or a named variant."""
    return VARIANTS[i] if isinstance(i, str) else SHAPES[i]


def custom(**kw) -> Shape:
    """A Shape for tests (tiny trees, ties, ragged sizes)."""
    base = dict(name="custom", dtype=torch.float32, n_heads=1, n_kv_heads=1, head_dim=64,
                fanout=(3, 3, 3), keep=(1, 1, 1), batch=1, n_tokens=1, seq_len=1)
    base.update(kw)
    return Shape(**base)


@dataclasses.dataclass
class Workload:
    shape: Shape
    root_keys: torch.Tensor      # [H_kv][b_R][D]
    mid_keys: torch.Tensor       # [H_kv][b_R*b_I][D]
    leaf_keys: torch.Tensor      # [H_kv][M][D]   (pinned host tensor when leaf_on_host)
    leaf_values: torch.Tensor    # [H_kv][M][D]
    root_child: Optional[torch.Tensor]   # [H_kv][b_R][b_I] int32 or None
    mid_child: Optional[torch.Tensor]    # [H_kv][b_R*b_I][b_L] int32 or None
    q_kg: torch.Tensor           # [B][N][H][D]
    q_seq: torch.Tensor          # [B][N][H][D]
    k_seq: torch.Tensor          # [B][T][H_kv][D]
    v_seq: torch.Tensor          # [B][T][H_kv][D]
    targets: torch.Tensor        # [B][H_kv] leaf row id each query was drawn near


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(g, shape_, device):
    return torch.randn(shape_, generator=g, device=device, dtype=torch.float32)


def _tree_head(sh: Shape, g, device):
    """One KV head's tree in logical order: leaves [b_R][b_I][b_L][D] (stored
    type), mids [b_R][b_I][D], roots [b_R][D]."""
    bR, bI, bL = sh.fanout
    D = sh.head_dim
    root_c = _randn(g, (bR, 1, 1, D), device)
    mid_c = root_c + 0.5 * _randn(g, (bR, bI, 1, D), device)
    leaves = (mid_c + 0.25 * _randn(g, (bR, bI, bL, D), device)).to(sh.dtype)
    wide = leaves.double()
    mids = wide.mean(dim=2).to(sh.dtype)
    roots = wide.sum(dim=(1, 2)).div(bI * bL).to(sh.dtype)
    return leaves, mids, roots


def make_workload(sh: Shape, device="cpu", seed: int = 1000, leaf_values_scale: float = 1.0) -> Workload:
    """Materialise one workload.  Everything lives on ``device`` except the
    leaf keys/values of a leaf_on_host shape, which go to pinned host memory."""
    device = torch.device(device)
    bR, bI, bL = sh.fanout
    M = sh.n_leaves
    D = sh.head_dim
    Hkv = sh.n_kv_heads
    g = _gen(device, seed)

    if sh.leaf_on_host:
        return _make_host_workload(sh, device, g, seed)

    leaf_keys = torch.empty((Hkv, M, D), dtype=sh.dtype, device=device)
    mid_keys = torch.empty((Hkv, bR * bI, D), dtype=sh.dtype, device=device)
    root_keys = torch.empty((Hkv, bR, D), dtype=sh.dtype, device=device)
    root_child = mid_child = None
    if sh.permuted:
        root_child = torch.empty((Hkv, bR, bI), dtype=torch.int32, device=device)
        mid_child = torch.empty((Hkv, bR * bI, bL), dtype=torch.int32, device=device)
    for hk in range(Hkv):
        leaves, mids, roots = _tree_head(sh, g, device)
        root_keys[hk] = roots
        if not sh.permuted:
            leaf_keys[hk] = leaves.reshape(M, D)
            mid_keys[hk] = mids.reshape(bR * bI, D)
        else:
            # logical mid l = r*b_I + j is stored at row pm[l]; logical leaf
            # (l, j) is stored at row pl[l*b_L + j].
            pm = torch.randperm(bR * bI, generator=g, device=device)
            pl = torch.randperm(M, generator=g, device=device)
            mid_keys[hk, pm] = mids.reshape(bR * bI, D)
            leaf_keys[hk, pl] = leaves.reshape(M, D)
            root_child[hk] = pm.view(bR, bI).to(torch.int32)
            mid_child[hk, pm] = pl.view(bR * bI, bL).to(torch.int32)
        del leaves, mids, roots
    leaf_values = (_randn(g, (Hkv, M, D), device) * leaf_values_scale).to(sh.dtype)
    q = _make_queries(sh, g, device, leaf_keys)
    return Workload(sh, root_keys, mid_keys, leaf_keys, leaf_values, root_child, mid_child, **q)


def _make_queries(sh: Shape, g, device, leaf_keys_dev):
    B, N, H, D, T = sh.batch, sh.n_tokens, sh.n_heads, sh.head_dim, sh.seq_len
    Hkv, G = sh.n_kv_heads, sh.group
    M = sh.n_leaves
    targets = torch.randint(0, M, (B, Hkv), generator=g, device=device)
    tk = torch.stack([leaf_keys_dev[hk].index_select(0, targets[:, hk].to(leaf_keys_dev.device)).to(device)
                      for hk in range(Hkv)], dim=1).float()           # [B][H_kv][D]
    tk = tk.repeat_interleave(G, dim=1)                               # [B][H][D]
    q_kg = (tk[:, None, :, :] + 0.1 * _randn(g, (B, N, H, D), device)).to(sh.dtype)
    q_seq = _randn(g, (B, N, H, D), device).to(sh.dtype)
    k_seq = _randn(g, (B, T, Hkv, D), device).to(sh.dtype)
    v_seq = _randn(g, (B, T, Hkv, D), device).to(sh.dtype)
    return dict(q_kg=q_kg, q_seq=q_seq, k_seq=k_seq, v_seq=v_seq, targets=targets.to(torch.int32))


def _make_host_workload(sh: Shape, device, g, seed) -> Workload:
    """Leaf keys and values generated one root subtree at a time on ``device``
    and copied into pinned host memory; interior keys stay on ``device``."""
    bR, bI, bL = sh.fanout
    M = sh.n_leaves
    D = sh.head_dim
    Hkv = sh.n_kv_heads
    leaf_keys = torch.empty((Hkv, M, D), dtype=sh.dtype, pin_memory=(device.type == "cuda"))
    leaf_values = torch.empty((Hkv, M, D), dtype=sh.dtype, pin_memory=(device.type == "cuda"))
    if sh.mid_on_host:
        mid_keys = torch.empty((Hkv, bR * bI, D), dtype=sh.dtype, pin_memory=(device.type == "cuda"))
    else:
        mid_keys = torch.empty((Hkv, bR * bI, D), dtype=sh.dtype, device=device)
    root_keys = torch.empty((Hkv, bR, D), dtype=sh.dtype, device=device)
    per_root = bI * bL
    for hk in range(Hkv):
        root_c = _randn(g, (bR, D), device)
        for r in range(bR):
            mid_c = root_c[r][None, None, :] + 0.5 * _randn(g, (bI, 1, D), device)
            leaves = (mid_c + 0.25 * _randn(g, (bI, bL, D), device)).to(sh.dtype)
            wide = leaves.double()
            mid_keys[hk, r * bI:(r + 1) * bI].copy_(wide.mean(dim=1).to(sh.dtype))
            root_keys[hk, r] = wide.sum(dim=(0, 1)).div(per_root).to(sh.dtype)
            leaf_keys[hk, r * per_root:(r + 1) * per_root].copy_(leaves.reshape(per_root, D), non_blocking=False)
            vals = _randn(g, (per_root, D), device).to(sh.dtype)
            leaf_values[hk, r * per_root:(r + 1) * per_root].copy_(vals, non_blocking=False)
    q = _make_queries(sh, g, device, leaf_keys)
    return Workload(sh, root_keys, mid_keys, leaf_keys, leaf_values, None, None, **q)


def flush_buffer(device="cuda", bytes_=256 << 20) -> torch.Tensor:
    """A buffer larger than the 126 MB L2; writing it evicts the cache."""
    return torch.empty(bytes_ // 4, dtype=torch.float32, device=device)


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


# ---------------------------------------------------------------------------
# Trees of any depth with a variable number of children per node (the unequal
# cluster sizes a clustering gives; "Method details / Hierarchical clustering of
# KGKVs" also lets the depth grow).  Children are stored contiguously in level
# order (child_off alone describes them), or, with permuted=True, at random
# rows of their level with an explicit child_id list.

@dataclasses.dataclass(frozen=True)
class CsrShape:
    name: str
    dtype: torch.dtype
    n_heads: int
    n_kv_heads: int
    head_dim: int
    n_roots: int
    fanout_ranges: tuple      # per level below the roots: (min, max) children per node, inclusive
    keep: tuple               # K per level, roots first
    batch: int
    n_tokens: int
    seq_len: int
    permuted: bool = False

    @property
    def n_levels(self) -> int:
        return 1 + len(self.fanout_ranges)

    @property
    def group(self) -> int:
        return self.n_heads // self.n_kv_heads


@dataclasses.dataclass
class CsrWorkload:
    shape: CsrShape
    keys: list                # per level [H_kv][rows_l][D]
    leaf_values: torch.Tensor
    child_off: list           # per level above the leaves: [H_kv][rows_l + 1] int32
    child_id: list            # per level above the leaves: [H_kv][rows_{l+1}] int32, or None
    q_kg: torch.Tensor
    q_seq: torch.Tensor
    k_seq: torch.Tensor
    v_seq: torch.Tensor
    targets: torch.Tensor     # [B][H_kv] leaf row each query was drawn near

    @property
    def rows(self):
        return [k.shape[1] for k in self.keys]


def make_csr_workload(sh: CsrShape, device="cpu", seed: int = 2000) -> CsrWorkload:
    """Every KV head has its own structure (the same number of nodes per level,
    its clusters' sizes shuffled) and its own keys: root centroids N(0,1)^D,
    each next level's centroid = parent + sigma N(0,1) (sigma 0.5, then halving
    per level), leaves stored as keys, interior keys = mean of their subtree's
    stored leaves (float64, rounded once); values N(0,1); queries as for the
    three-level shapes."""
    device = torch.device(device)
    g = _gen(device, seed)
    gc = torch.Generator()
    gc.manual_seed(int(seed) + 7)
    D, Hkv = sh.head_dim, sh.n_kv_heads
    L = sh.n_levels
    # base child counts per level; each KV head shuffles them among the level's nodes
    base = []
    n = sh.n_roots
    for lo, hi in sh.fanout_ranges:
        c = torch.randint(lo, hi + 1, (n,), generator=gc)
        base.append(c)
        n = int(c.sum())
    rows = [sh.n_roots] + [int(c.sum()) for c in base]
    keys = [torch.empty((Hkv, rows[l], D), dtype=sh.dtype, device=device) for l in range(L)]
    child_off = [torch.empty((Hkv, rows[l] + 1), dtype=torch.int32) for l in range(L - 1)]
    child_id = [torch.empty((Hkv, rows[l + 1]), dtype=torch.int32) if sh.permuted else None for l in range(L - 1)]
    for hk in range(Hkv):
        counts = [c[torch.randperm(len(c), generator=gc)] for c in base]
        # parent (contiguous index) of every node of levels 1..L-1, contiguous child offsets
        parent = [torch.repeat_interleave(torch.arange(rows[l]), counts[l]) for l in range(L - 1)]
        offs = [torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(c, 0)]) for c in counts]
        perms = [torch.randperm(rows[l + 1], generator=gc) if sh.permuted else None for l in range(L - 1)]
        cent = _randn(g, (rows[0], D), device)
        sigma = 0.5
        for l in range(1, L):
            cent = cent[parent[l - 1].to(device)] + sigma * _randn(g, (rows[l], D), device)
            sigma *= 0.5
        leaves = cent.to(sh.dtype)               # contiguous order
        level_keys = [None] * L
        level_keys[L - 1] = leaves
        sums, sizes = leaves.double(), torch.ones(rows[L - 1], dtype=torch.float64, device=device)
        for l in range(L - 2, -1, -1):           # subtree sums and sizes, bottom up
            p = parent[l].to(device)
            sums = torch.zeros((rows[l], D), dtype=torch.float64, device=device).index_add_(0, p, sums)
            sizes = torch.zeros(rows[l], dtype=torch.float64, device=device).index_add_(0, p, sizes)
            level_keys[l] = (sums / sizes[:, None]).to(sh.dtype)
        for l in range(L):
            if l >= 1 and perms[l - 1] is not None:
                keys[l][hk, perms[l - 1].to(device)] = level_keys[l]   # contiguous node i at row perm[i]
            else:
                keys[l][hk] = level_keys[l]
        # CSR per level, indexed by the parent's storage row: with permuted
        # storage the child list is ordered by parent row and names the
        # children's rows
        for l in range(L - 1):
            if perms[l] is None:
                child_off[l][hk] = offs[l].to(torch.int32)
                continue
            if l == 0:
                par_of_row = torch.arange(rows[0])
            else:
                par_of_row = torch.empty(rows[l], dtype=torch.int64)
                par_of_row[perms[l - 1]] = torch.arange(rows[l])
            cnt_row = counts[l][par_of_row]
            child_off[l][hk] = torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(cnt_row, 0)]).to(torch.int32)
            o = offs[l]
            lists = [torch.arange(int(o[i]), int(o[i + 1])) for i in par_of_row.tolist()]
            child_id[l][hk] = perms[l][torch.cat(lists)].to(torch.int32)
    child_off = [o.to(device) for o in child_off]
    child_id = [None if c is None else c.to(device) for c in child_id]
    leaf_values = _randn(g, (Hkv, rows[L - 1], D), device).to(sh.dtype)
    B, N, H, T, G = sh.batch, sh.n_tokens, sh.n_heads, sh.seq_len, sh.group
    targets = torch.randint(0, rows[L - 1], (B, Hkv), generator=g, device=device)
    tk = torch.stack([keys[L - 1][hk].index_select(0, targets[:, hk]) for hk in range(Hkv)], dim=1).float()
    tk = tk.repeat_interleave(G, dim=1)
    q_kg = (tk[:, None, :, :] + 0.1 * _randn(g, (B, N, H, D), device)).to(sh.dtype)
    q_seq = _randn(g, (B, N, H, D), device).to(sh.dtype)
    k_seq = _randn(g, (B, T, Hkv, D), device).to(sh.dtype)
    v_seq = _randn(g, (B, T, Hkv, D), device).to(sh.dtype)
    return CsrWorkload(sh, keys, leaf_values, child_off, child_id, q_kg, q_seq, k_seq, v_seq,
                       targets.to(torch.int32))
