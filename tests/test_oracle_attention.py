"""Pins for the oracle's attention parts and the lambda merge.

* Sequence part: the causal self-attention equation ("Background /
  Self-attention") against PyTorch's scaled_dot_product_attention in float64
  with an explicit boolean mask (a library routine).
* Merge: lam_kg*Softmax(logits_kg)V_kg + lam_seq*Softmax(logits_seq)V_seq with
  lam = normalised exp of the two log-sum-exps must equal ONE softmax over the
  concatenated logits (closed-form identity; the joint softmax is torch's).
* Whole path with K equal to the fan-out at every level keeps every leaf, so it
  must equal the rectangular attention over all M knowledge keys plus the causal
  sequence ("Background / Rectangular attention in KBLaM" equation).
* Closed forms: all-zero queries give uniform weights.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from hierarchical_kv_pruning_b200 import synth
from tests._util import oracle_inputs, oracle_tree, storage


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("N,T", [(1, 1), (4, 4), (5, 17), (16, 16), (3, 64)])
def test_sequence_part_matches_sdpa(N, T):
    D = 32
    q = _rand((6, N, D), 1)
    k = _rand((6, T, D), 2)
    v = _rand((6, T, D), 3)
    scale = 1.0 / math.sqrt(D)
    o, lse = oracle.sequence_attention(q, k, v, scale)
    mask = torch.arange(T)[None, :] <= (torch.arange(N)[:, None] + (T - N))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=mask, scale=scale)
    assert np.max(np.abs(o - ref.numpy())) < 1e-12
    logits = torch.from_numpy(q) @ torch.from_numpy(k).transpose(1, 2) * scale
    ref_lse = torch.logsumexp(logits.masked_fill(~mask, float("-inf")), dim=-1)
    assert np.max(np.abs(lse - ref_lse.numpy())) < 1e-12


@pytest.mark.parametrize("kg_scale", [1.0, 0.15, 4.0])
def test_merge_equals_joint_softmax(kg_scale):
    T_, N, J, S, D = 5, 4, 7, 9, 16
    scale = 1.0 / math.sqrt(D)
    qk = _rand((T_, N, D), 10, kg_scale)
    lk = _rand((T_, J, D), 11)
    lv = _rand((T_, J, D), 12)
    qs = _rand((T_, N, D), 13)
    ks = _rand((T_, S, D), 14)
    vs = _rand((T_, S, D), 15)
    o_kg, lse_kg = oracle.kg_attention(qk, lk, lv, scale)
    o_seq, lse_seq = oracle.sequence_attention(qs, ks, vs, scale)
    y, lse = oracle.merge(o_kg, lse_kg, o_seq, lse_seq)
    # joint softmax over [kept leaves | causal sequence] logits
    lg_kg = torch.from_numpy(qk) @ torch.from_numpy(lk).transpose(1, 2) * scale
    lg_seq = torch.from_numpy(qs) @ torch.from_numpy(ks).transpose(1, 2) * scale
    vis = torch.arange(S)[None, :] <= (torch.arange(N)[:, None] + (S - N))
    lg_seq = lg_seq.masked_fill(~vis, float("-inf"))
    logits = torch.cat([lg_kg, lg_seq], dim=-1)
    p = torch.softmax(logits, dim=-1)
    ref = p @ torch.cat([torch.from_numpy(lv), torch.from_numpy(vs)], dim=1)
    assert np.max(np.abs(y - ref.numpy())) < 1e-12
    assert np.max(np.abs(lse - torch.logsumexp(logits, -1).numpy())) < 1e-12


def test_lambda_is_one_half_when_blocks_balance():
    # identical KG and sequence blocks (one token, one key each) -> lam = 1/2
    D = 8
    q = _rand((1, 1, D), 20)
    k = _rand((1, 1, D), 21)
    v1 = _rand((1, 1, D), 22)
    v2 = _rand((1, 1, D), 23)
    o1, l1 = oracle.kg_attention(q, k, v1, 0.3)
    o2, l2 = oracle.sequence_attention(q, k, v2, 0.3)
    y, lse = oracle.merge(o1, l1, o2, l2)
    assert np.allclose(y, 0.5 * (v1 + v2), atol=1e-15, rtol=0)
    assert abs(lse[0, 0] - (l1[0, 0] + math.log(2.0))) < 1e-15


def test_zero_queries_give_uniform_weights():
    sh = synth.custom(dtype=torch.float32, n_heads=2, n_kv_heads=1, head_dim=16, fanout=(3, 3, 4),
                      keep=(2, 3, 5), batch=2, n_tokens=3, seq_len=7)
    w = synth.make_workload(sh, "cpu", 9)
    w.q_kg.zero_()
    w.q_seq.zero_()
    t = oracle_tree(w)
    inp = oracle_inputs(w)
    r = oracle.hikvp(t, inp["q_kg"], inp["q_seq"], inp["k_seq"], inp["v_seq"], (2, 3, 5))
    # zero query: all roots/mids/leaves tie -> lowest rows; logits all 0
    assert (r["kept_leaf"] == np.arange(5)).all()
    lv = w.leaf_values.double().numpy()[0]
    vs = w.v_seq.double().numpy()
    for i, (b, h) in enumerate(r["traversals"]):
        for n in range(3):
            visible = 7 - 3 + n + 1
            expected = (lv[:5].sum(0) + vs[b, :visible, 0].sum(0)) / (5 + visible)
            assert np.max(np.abs(r["y"][i, n] - expected)) < 1e-12
            assert abs(r["lse"][i, n] - math.log(5 + visible)) < 1e-12


def _rectangular(w, b, h, scale):
    """Joint softmax over ALL M knowledge keys plus the causal sequence."""
    sh = w.shape
    hkv = h // sh.group
    qk = w.q_kg[b, :, h].double()
    qs = w.q_seq[b, :, h].double()
    lg_kg = qk @ w.leaf_keys[hkv].double().T * scale
    lg_seq = qs @ w.k_seq[b, :, hkv].double().T * scale
    N, T = sh.n_tokens, sh.seq_len
    vis = torch.arange(T)[None, :] <= (torch.arange(N)[:, None] + (T - N))
    lg_seq = lg_seq.masked_fill(~vis, float("-inf"))
    logits = torch.cat([lg_kg, lg_seq], -1)
    vals = torch.cat([w.leaf_values[hkv].double(), w.v_seq[b, :, hkv].double()], 0)
    return (torch.softmax(logits, -1) @ vals).numpy(), torch.logsumexp(logits, -1).numpy()


def test_full_k_equals_rectangular_attention_tiny_config():
    sh = synth.shape(0)
    w = synth.make_workload(sh, "cpu", 1000)
    t = oracle_tree(w)
    inp = oracle_inputs(w)
    bR, bI, bL = sh.fanout
    K = (bR, bR * bI, bR * bI * bL)           # 10 / 100 / 1000: nothing pruned
    r = oracle.hikvp(t, inp["q_kg"], inp["q_seq"], inp["k_seq"], inp["v_seq"], K)
    assert (np.sort(r["kept_leaf"][0]) == np.arange(sh.n_leaves)).all()
    ref_y, ref_lse = _rectangular(w, 0, 0, 1.0 / math.sqrt(sh.head_dim))
    assert np.max(np.abs(r["y"][0] - ref_y)) < 1e-12
    assert np.max(np.abs(r["lse"][0] - ref_lse)) < 1e-12


def test_full_k_equals_rectangular_attention_grouped_permuted():
    sh = synth.custom(dtype=torch.bfloat16, n_heads=4, n_kv_heads=2, head_dim=16, fanout=(3, 4, 5),
                      batch=2, n_tokens=4, seq_len=9, permuted=True)
    w = synth.make_workload(sh, "cpu", 77)
    t = oracle_tree(w)
    inp = oracle_inputs(w)
    K = (3, 12, 60)
    r = oracle.hikvp(t, inp["q_kg"], inp["q_seq"], inp["k_seq"], inp["v_seq"], K)
    for i, (b, h) in enumerate(r["traversals"]):
        ref_y, ref_lse = _rectangular(w, b, h, 0.25)
        assert np.max(np.abs(r["y"][i] - ref_y)) < 1e-12
        assert np.max(np.abs(r["lse"][i] - ref_lse)) < 1e-12


def test_pruned_output_is_joint_softmax_over_kept_union():
    # partial K: the merged output is one softmax over (kept leaves + visible sequence)
    sh = synth.shape(0)
    w = synth.make_workload(sh, "cpu", 1000)
    t = oracle_tree(w)
    inp = oracle_inputs(w)
    r = oracle.hikvp(t, inp["q_kg"], inp["q_seq"], inp["k_seq"], inp["v_seq"], sh.keep)
    kept = torch.from_numpy(r["kept_leaf"][0].astype(np.int64))
    scale = 1.0 / math.sqrt(sh.head_dim)
    lg_kg = w.q_kg[0, :, 0].double() @ w.leaf_keys[0, kept].double().T * scale
    lg_seq = w.q_seq[0, :, 0].double() @ w.k_seq[0, :, 0].double().T * scale
    vis = torch.arange(16)[None, :] <= torch.arange(16)[:, None]
    logits = torch.cat([lg_kg, lg_seq.masked_fill(~vis, float("-inf"))], -1)
    vals = torch.cat([w.leaf_values[0, kept].double(), w.v_seq[0, :, 0].double()], 0)
    assert np.max(np.abs(r["y"][0] - (torch.softmax(logits, -1) @ vals).numpy())) < 1e-12
