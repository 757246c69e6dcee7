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


def shape(i: int) -> Shape:
    return SHAPES[i]


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
    mid_keys = torch.empty((Hkv, bR * bI, D), dtype=sh.dtype, device=device)
    root_keys = torch.empty((Hkv, bR, D), dtype=sh.dtype, device=device)
    per_root = bI * bL
    for hk in range(Hkv):
        root_c = _randn(g, (bR, D), device)
        for r in range(bR):
            mid_c = root_c[r][None, None, :] + 0.5 * _randn(g, (bI, 1, D), device)
            leaves = (mid_c + 0.25 * _randn(g, (bI, bL, D), device)).to(sh.dtype)
            wide = leaves.double()
            mid_keys[hk, r * bI:(r + 1) * bI] = wide.mean(dim=1).to(sh.dtype)
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
