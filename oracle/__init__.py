"""HiKVP oracle: a plain, slow CPU restatement of what the hot path computes.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``hierarchical_kv_pruning_b200``) never imports it,
and shares no code, header, table or helper with it.

Source: "AtlasKV: Augmenting LLMs with Billion-Scale Knowledge Graphs in 20GB
VRAM" (ICLR 2026 notes).

* Descent (``descend``): section "Quick read / How it works" and "Method
  details / Hierarchical clustering of KGKVs".  Exact ranking in plain C
  (``hikvp_oracle.c``), see that file's header for the node-score reading.
* KG part and sequence part (``kg_attention``, ``sequence_attention``): the
  self-attention equation of "Background / Self-attention" (causal softmax over
  positions i <= n, logits <q, k>/sqrt(D)) applied once to the kept leaves (no
  mask: knowledge keys are not causal, as in the rectangular-attention equation
  of "Background / Rectangular attention in KBLaM") and once to the sequence.
* Merge (``merge``): the equation under "Quick read / How it works" and
  "Method details / Equivalent attention", y = lam_kg * Softmax(logits_kg) V_kg
  + lam_seq * Softmax(logits_seq) V_seq.  The pages lose the lambda formula;
  the reading used is lam_kg = e^{LSE_kg} / (e^{LSE_kg} + e^{LSE_seq}),
  lam_seq = 1 - lam_kg (the normalised exp of the two log-sum-exps).

All floating point here is float64.  Parity status: every function is pinned
(tests/test_oracle_*.py); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hikvp_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libhikvp_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C part of the oracle with gcc (OpenMP over traversals)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-Wextra", "-o", tmp, _SRC])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Tree(ctypes.Structure):
    _fields_ = [
        ("is_bf16", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("b_root", ctypes.c_int),
        ("b_mid", ctypes.c_int),
        ("b_leaf", ctypes.c_int),
        ("root_keys", ctypes.c_void_p),
        ("mid_keys", ctypes.c_void_p),
        ("leaf_keys", ctypes.c_void_p),
        ("root_child", ctypes.c_void_p),
        ("mid_child", ctypes.c_void_p),
    ]


class _CsrTree(ctypes.Structure):
    _fields_ = [
        ("is_bf16", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("n_levels", ctypes.c_int),
        ("rows", ctypes.c_void_p),
        ("keys", ctypes.c_void_p),
        ("child_off", ctypes.c_void_p),
        ("child_id", ctypes.c_void_p),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.oracle_descend.argtypes = [ctypes.POINTER(_Tree), P, I, I, I, I, I, I, I, P, P, P, P, P]
            lib.oracle_descend.restype = I
            lib.oracle_exact_dot_digits.argtypes = [P, I, P, I, I, P]
            lib.oracle_exact_dot_digits.restype = None
            lib.oracle_level_scores.argtypes = [ctypes.POINTER(_Tree), I, P, I, I, I, I, P, I, P]
            lib.oracle_level_scores.restype = None
            lib.oracle_exact_digits.restype = I
            lib.oracle_exact_origin.restype = I
            lib.oracle_descend_csr.argtypes = [ctypes.POINTER(_CsrTree), P, I, I, P, I, P, P, P]
            lib.oracle_descend_csr.restype = I
            _lib = lib
    return _lib


# ---------------------------------------------------------------------------
# Inputs.  Key/query storage is handed to C as raw bit patterns: bfloat16 as
# uint16, binary32 as float32.  Values used by the float64 attention are the
# exact widenings of the same stored numbers.
# ---------------------------------------------------------------------------

def _as_storage(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype not in (np.uint16, np.float32):
        raise TypeError("oracle storage must be uint16 (bfloat16 bits) or float32, got %s" % a.dtype)
    return a


def widen(a: np.ndarray) -> np.ndarray:
    """Exact float64 value of stored bfloat16 bits (uint16) or float32."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


class Tree:
    """Three-level key tree, layout [H_kv][rows][D] per level; child tables
    [H_kv][parents][fanout] of row ids, or None for child(p, j) = p*fanout + j.
    Leaf values are only needed by the attention part."""

    def __init__(self, root_keys, mid_keys, leaf_keys, leaf_values, fanout,
                 root_child=None, mid_child=None):
        self.root_keys = _as_storage(root_keys)
        self.mid_keys = _as_storage(mid_keys)
        self.leaf_keys = _as_storage(leaf_keys)
        self.leaf_values = leaf_values
        self.fanout = tuple(int(f) for f in fanout)
        self.root_child = None if root_child is None else np.ascontiguousarray(root_child, dtype=np.int32)
        self.mid_child = None if mid_child is None else np.ascontiguousarray(mid_child, dtype=np.int32)
        self.is_bf16 = self.root_keys.dtype == np.uint16
        self.n_kv_heads, _, self.head_dim = self.root_keys.shape
        bR, bI, bL = self.fanout
        assert self.root_keys.shape == (self.n_kv_heads, bR, self.head_dim)
        assert self.mid_keys.shape == (self.n_kv_heads, bR * bI, self.head_dim)
        assert self.leaf_keys.shape[:2] == (self.n_kv_heads, bR * bI * bL)
        for a in (self.mid_keys, self.leaf_keys):
            assert a.dtype == self.root_keys.dtype

    def _c(self) -> _Tree:
        bR, bI, bL = self.fanout
        return _Tree(int(self.is_bf16), self.n_kv_heads, self.head_dim, bR, bI, bL,
                     self.root_keys.ctypes.data, self.mid_keys.ctypes.data,
                     self.leaf_keys.ctypes.data,
                     None if self.root_child is None else self.root_child.ctypes.data,
                     None if self.mid_child is None else self.mid_child.ctypes.data)

    def children(self, level: int, hkv: int, parent: int) -> np.ndarray:
        """Row ids of the children of node ``parent`` at ``level`` (0 root, 1 mid)."""
        bR, bI, bL = self.fanout
        if level == 0:
            if self.root_child is not None:
                return self.root_child[hkv, parent].copy()
            return np.arange(parent * bI, (parent + 1) * bI, dtype=np.int32)
        if self.mid_child is not None:
            return self.mid_child[hkv, parent].copy()
        return np.arange(parent * bL, (parent + 1) * bL, dtype=np.int32)


# ---------------------------------------------------------------------------
# Descent
# ---------------------------------------------------------------------------

def descend(tree: Tree, q_kg: np.ndarray, K, traversals=None):
    """Kept node sets of the greedy descent ("Quick read / How it works").

    q_kg: stored query tokens for the KG part, [B][N][H][D] (same storage type
    as the tree).  K = (K_R, K_I, K_L).  traversals: optional list of (b, h);
    default all B*H in (b, h) row-major order.
    Returns kept_root [T][K_R], kept_mid [T][K_I], kept_leaf [T][K_L] (int32,
    ascending row ids) for the T traversals.
    """
    lib = _load()
    q = _as_storage(q_kg)
    assert q.dtype == tree.root_keys.dtype
    B, N, H, D = q.shape
    assert D == tree.head_dim and H % tree.n_kv_heads == 0
    K_R, K_I, K_L = (int(k) for k in K)
    if traversals is None:
        bb, hh = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
        trav = np.stack([bb.ravel(), hh.ravel()], 1)
    else:
        trav = np.asarray(traversals, dtype=np.int64).reshape(-1, 2)
    tb = np.ascontiguousarray(trav[:, 0], dtype=np.int32)
    th = np.ascontiguousarray(trav[:, 1], dtype=np.int32)
    n = len(tb)
    kr = np.zeros((n, K_R), np.int32)
    km = np.zeros((n, K_I), np.int32)
    kl = np.zeros((n, K_L), np.int32)
    ct = tree._c()
    rc = lib.oracle_descend(ctypes.byref(ct), q.ctypes.data, B, N, H, K_R, K_I, K_L, n,
                            tb.ctypes.data, th.ctypes.data,
                            kr.ctypes.data, km.ctypes.data, kl.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_descend rejected the arguments (K above candidate count or bad child table)")
    return kr, km, kl


def exact_digits(q_block: np.ndarray, k_row: np.ndarray):
    """Exact x = sum_n sum_d q[n,d] k[d] as normalized digits (pin support)."""
    lib = _load()
    q = _as_storage(q_block)
    k = _as_storage(k_row)
    assert q.dtype == k.dtype
    N, D = q.shape
    nd = lib.oracle_exact_digits()
    out = np.zeros(nd, np.int64)
    lib.oracle_exact_dot_digits(q.ctypes.data, N, k.ctypes.data, D, int(q.dtype == np.uint16), out.ctypes.data)
    return out


def digits_to_int(digits) -> int:
    """Integer value of normalized digits, i.e. x * 2^origin."""
    v = 0
    for i, d in enumerate(digits):
        v += int(d) << (32 * i)
    return v


def exact_origin() -> int:
    return _load().oracle_exact_origin()


def level_scores(tree: Tree, level: int, q_kg: np.ndarray, b: int, h: int, rows) -> list:
    """Exact node scores (as integers x * 2^origin) of ``rows`` at ``level``
    for traversal (b, h)."""
    lib = _load()
    q = _as_storage(q_kg)
    _, N, H, _ = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    nd = lib.oracle_exact_digits()
    out = np.zeros((len(rows), nd), np.int64)
    ct = tree._c()
    lib.oracle_level_scores(ctypes.byref(ct), int(level), q.ctypes.data, N, H, int(b), int(h),
                            rows.ctypes.data, len(rows), out.ctypes.data)
    return [digits_to_int(r) for r in out]


# ---------------------------------------------------------------------------
# Attention parts, float64.  Shapes per traversal batch:
#   q [T][N][D] (one row of tokens per traversal), keys/values [T][J][D].
# ---------------------------------------------------------------------------

def _softmax_block(logits: np.ndarray, values: np.ndarray):
    """Softmax over the last axis of logits (entries may be -inf) times values.
    Returns (output, log-sum-exp)."""
    m = np.max(logits, axis=-1, keepdims=True)
    w = np.exp(logits - m)
    z = np.sum(w, axis=-1, keepdims=True)
    out = np.einsum("tnj,tjd->tnd", w, values) / z
    lse = (m + np.log(z))[..., 0]
    return out, lse


def kg_attention(q_kg: np.ndarray, leaf_k: np.ndarray, leaf_v: np.ndarray, scale: float):
    """Softmax(logits_kg) . V over the kept leaves, every token sees every kept
    leaf.  q_kg [T][N][D], leaf_k/leaf_v [T][K_L][D].  Returns (O_kg, LSE_kg)."""
    logits = np.einsum("tnd,tjd->tnj", q_kg, leaf_k) * scale
    return _softmax_block(logits, leaf_v)


def sequence_attention(q_seq: np.ndarray, k_seq: np.ndarray, v_seq: np.ndarray, scale: float):
    """Causal softmax attention ("Background / Self-attention" equation).  The N
    query tokens are the last N of the T-token sequence: token n (0-based) sees
    positions i <= T - N + n.  q_seq [T'][N][D], k_seq/v_seq [T'][T][D]."""
    n_tok = q_seq.shape[1]
    t_len = k_seq.shape[1]
    logits = np.einsum("tnd,tid->tni", q_seq, k_seq) * scale
    pos = np.arange(n_tok)[:, None] + (t_len - n_tok)
    visible = np.arange(t_len)[None, :] <= pos
    logits = np.where(visible[None], logits, -np.inf)
    return _softmax_block(logits, v_seq)


def merge(o_kg, lse_kg, o_seq, lse_seq):
    """lam_kg * O_kg + lam_seq * O_seq with lam_kg = e^{LSE_kg}/(e^{LSE_kg}+e^{LSE_seq}).
    Returns (y, LSE of the union)."""
    m = np.maximum(lse_kg, lse_seq)
    a = np.exp(lse_kg - m)
    c = np.exp(lse_seq - m)
    lam_kg = a / (a + c)
    lam_seq = c / (a + c)
    y = lam_kg[..., None] * o_kg + lam_seq[..., None] * o_seq
    return y, m + np.log(a + c)


def attend_traversals(tree: Tree, q_kg, q_seq, k_seq, v_seq, kept_leaf, traversals, scale=None):
    """Outputs y [T][N][D] and LSE [T][N] for the listed traversals (b, h).

    q_kg, q_seq: [B][N][H][D]; k_seq, v_seq: [B][T][H_kv][D]; tree leaf values
    [H_kv][M][D]; kept_leaf [T][K_L] (row ids per KV head).  All arrays are
    stored numbers (uint16 bfloat16 bits or float32); arithmetic is float64.
    """
    trav = np.asarray(traversals, dtype=np.int64).reshape(-1, 2)
    B, N, H, D = q_kg.shape
    G = H // tree.n_kv_heads
    if scale is None or scale == 0:
        scale = 1.0 / np.sqrt(D)
    b = trav[:, 0]
    h = trav[:, 1]
    hkv = h // G
    qk = widen(q_kg[b, :, h, :])                  # [T][N][D]
    qs = widen(q_seq[b, :, h, :])
    ks = widen(k_seq[b, :, hkv, :])               # [T][Tseq][D]
    vs = widen(v_seq[b, :, hkv, :])
    kept = np.asarray(kept_leaf)
    lk = widen(tree.leaf_keys[hkv[:, None], kept])    # [T][K_L][D]
    lv = widen(np.asarray(tree.leaf_values)[hkv[:, None], kept])
    o_kg, lse_kg = kg_attention(qk, lk, lv, scale)
    o_seq, lse_seq = sequence_attention(qs, ks, vs, scale)
    return merge(o_kg, lse_kg, o_seq, lse_seq)


def hikvp(tree: Tree, q_kg, q_seq, k_seq, v_seq, K, traversals=None, scale=None):
    """Whole hot path for the listed traversals: descent then merged attention.
    Returns dict with kept_root, kept_mid, kept_leaf, y [T][N][D], lse [T][N]."""
    B, N, H, D = q_kg.shape
    if traversals is None:
        bb, hh = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
        traversals = np.stack([bb.ravel(), hh.ravel()], 1)
    kr, km, kl = descend(tree, q_kg, K, traversals)
    y, lse = attend_traversals(tree, q_kg, q_seq, k_seq, v_seq, kl, traversals, scale)
    return {"kept_root": kr, "kept_mid": km, "kept_leaf": kl, "y": y, "lse": lse,
            "traversals": np.asarray(traversals).reshape(-1, 2)}


# ---------------------------------------------------------------------------
# Trees of any depth with variable numbers of children ("Method details /
# Hierarchical clustering of KGKVs": clusters of unequal size; the depth can be
# set larger).
# ---------------------------------------------------------------------------

class CsrTree:
    """Levels 0 (roots) .. L-1 (leaves), keys [H_kv][rows_l][D] per level (stored
    numbers), leaf values [H_kv][rows_{L-1}][D].  child_off[l]: [H_kv][rows_l + 1]
    int32 offsets into level l's child list; child_id[l]: [H_kv][rows_{l+1}]
    int32 row ids of level l + 1, or None (the child list positions are the row
    ids: children stored contiguously)."""

    def __init__(self, keys, leaf_values, child_off, child_id=None):
        self.keys = [_as_storage(k) for k in keys]
        self.leaf_values = leaf_values
        self.n_levels = len(self.keys)
        self.child_off = [np.ascontiguousarray(o, dtype=np.int32) for o in child_off]
        ids = child_id if child_id is not None else [None] * (self.n_levels - 1)
        self.child_id = [None if c is None else np.ascontiguousarray(c, dtype=np.int32) for c in ids]
        assert len(self.child_off) == self.n_levels - 1 == len(self.child_id)
        self.n_kv_heads, _, self.head_dim = self.keys[0].shape
        self.rows = [k.shape[1] for k in self.keys]
        self.is_bf16 = self.keys[0].dtype == np.uint16
        for l in range(self.n_levels - 1):
            assert self.child_off[l].shape == (self.n_kv_heads, self.rows[l] + 1)

    @property
    def leaf_keys(self):
        return self.keys[-1]

    def children(self, level: int, hkv: int, parent: int) -> np.ndarray:
        o = self.child_off[level][hkv]
        pos = np.arange(o[parent], o[parent + 1])
        ids = self.child_id[level]
        return (pos if ids is None else ids[hkv][pos]).astype(np.int32)


def descend_csr(tree: CsrTree, q_kg: np.ndarray, K, traversals=None):
    """Kept node sets per level of the greedy descent on a CSR tree: a list of
    [T][K_l] int32 arrays (ascending row ids), one per level."""
    lib = _load()
    q = _as_storage(q_kg)
    assert q.dtype == tree.keys[0].dtype
    B, N, H, D = q.shape
    assert len(K) == tree.n_levels
    if traversals is None:
        bb, hh = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
        trav = np.stack([bb.ravel(), hh.ravel()], 1)
    else:
        trav = np.asarray(traversals, dtype=np.int64).reshape(-1, 2)
    tb = np.ascontiguousarray(trav[:, 0], dtype=np.int32)
    th = np.ascontiguousarray(trav[:, 1], dtype=np.int32)
    n = len(tb)
    kk = np.ascontiguousarray(K, dtype=np.int32)
    kept = [np.zeros((n, int(k)), np.int32) for k in K]
    L = tree.n_levels
    rows = np.ascontiguousarray(tree.rows, dtype=np.int64)
    keys = (ctypes.c_void_p * L)(*[k.ctypes.data for k in tree.keys])
    offs = (ctypes.c_void_p * (L - 1))(*[o.ctypes.data for o in tree.child_off])
    ids = (ctypes.c_void_p * (L - 1))(*[None if c is None else c.ctypes.data for c in tree.child_id])
    outs = (ctypes.c_void_p * L)(*[k.ctypes.data for k in kept])
    ct = _CsrTree(int(tree.is_bf16), tree.n_kv_heads, tree.head_dim, L, rows.ctypes.data,
                  ctypes.cast(keys, ctypes.c_void_p), ctypes.cast(offs, ctypes.c_void_p),
                  ctypes.cast(ids, ctypes.c_void_p))
    rc = lib.oracle_descend_csr(ctypes.byref(ct), q.ctypes.data, N, H, kk.ctypes.data, n, tb.ctypes.data,
                                th.ctypes.data, ctypes.cast(outs, ctypes.c_void_p))
    if rc != 0:
        raise ValueError("oracle_descend_csr rejected the arguments (a level with fewer candidates than K, or a "
                         "child id out of range)")
    return kept


def hikvp_csr(tree: CsrTree, q_kg, q_seq, k_seq, v_seq, K, traversals=None, scale=None):
    """Whole hot path on a CSR tree: descent, then the merged attention over the
    kept leaves (the last level) and the causal sequence."""
    B, N, H, D = q_kg.shape
    if traversals is None:
        bb, hh = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
        traversals = np.stack([bb.ravel(), hh.ravel()], 1)
    kept = descend_csr(tree, q_kg, K, traversals)
    y, lse = attend_traversals(tree, q_kg, q_seq, k_seq, v_seq, kept[-1], traversals, scale)
    return {"kept": kept, "y": y, "lse": lse, "traversals": np.asarray(traversals).reshape(-1, 2)}
