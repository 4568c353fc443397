"""Pins of the fp64 oracle against what the RecSA abstract and mathematics fix.

Each test checks the oracle against something other than itself: a library
routine, a closed form written out by hand, an invariant the abstract states,
a special case that reduces to plain attention, or a structural count worked by
hand (Recursive Sparse Attention, abstract).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import recsa_inputs as I
from oracle import recsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SCALE = 1.0 / math.sqrt(128)


def _bits(t):
    return I.bf16_bits(t)


# --------------------------------------------------------------------------- bf16

def test_bf16_known_patterns():
    pats = {0x3F80: 1.0, 0xC000: -2.0, 0x0000: 0.0, 0x3EAB: 0.333984375, 0x7F7F: 3.3895313892515355e38,
            0x0001: 2.0 ** -133, 0x4049: 3.140625}
    got = O.bf16_bits_to_f64(np.array(list(pats), dtype=np.uint16))
    assert got.tolist() == list(pats.values())


def test_round_to_bf16_matches_torch_cast_including_ties():
    rng = np.random.default_rng(5)
    base = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0)
    # exact halfway points between neighbouring bf16 values, both parities
    b16 = torch.from_numpy(base).to(torch.bfloat16).to(torch.float32).numpy()
    bits = b16.view(np.uint32)
    half = (bits + np.uint32(0x8000)).view(np.float32)  # b16 + half an ulp (same sign)
    tiny = np.float32(2.0 ** -130) * rng.standard_normal(200).astype(np.float32)  # subnormal range
    x = np.concatenate([base, half, tiny]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_to_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)
    assert np.array_equal(O.f64_to_bf16_bits(x.astype(np.float64)),
                          torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def test_round_to_bf16_is_idempotent_and_nearest():
    rng = np.random.default_rng(6)
    x = rng.standard_normal(5000) * 10
    r = O.round_to_bf16(x)
    assert np.array_equal(O.round_to_bf16(r), r)
    # nearest: |x - r| <= half an ulp of r's binade
    ulp = np.ldexp(1.0, np.frexp(np.abs(r))[1] - 8)
    assert np.all(np.abs(x - r) <= ulp / 2 * (1 + 1e-12))


# --------------------------------------------------------------------------- structure

def test_level_counts_golden():
    cases = json.load(open(os.path.join(GOLDEN, "level_counts.json")))["cases"]
    for c in cases:
        assert O.level_counts(c["length"], c["b"]) == c["levels"], c


@pytest.mark.parametrize("length,b,k", [(4096, 8, 4), (4096, 16, 8), (65536, 16, 8), (131072, 16, 8)])
def test_entry_counts_golden(length, b, k):
    want = [c for c in json.load(open(os.path.join(GOLDEN, "entry_counts.json")))["cases"]
            if (c["length"], c["b"], c["k"]) == (length, b, k)][0]
    rng = np.random.default_rng(length + b)
    kt = np.zeros((length, 128))
    vt = np.zeros((length, 128))
    kt[:, :4] = rng.standard_normal((length, 4))  # cheap but non-degenerate scores
    tree = O.build_tree(kt, vt, np.eye(128), b, storage="exact")
    tr = O.Trace()
    O.attend(rng.standard_normal((4, 128)), tree, length, k, trace=tr)
    assert (tr.keys_read, tr.values_read) == (want["keys"], want["values"])


def test_max_rope_offset_bounded():
    # A5: every relative distance stays within the range seen at short length:
    # decode offsets are <= max(n_T, k*b); causal ones <= (k+1)*b.
    rng = np.random.default_rng(11)
    L, b, k = 5000, 8, 3
    kt = rng.standard_normal((L, 128))
    tree = O.build_tree(kt, rng.standard_normal((L, 128)), np.eye(128), b)
    tr = O.Trace()
    O.attend(rng.standard_normal((2, 128)), tree, L, k, trace=tr)
    assert max(tr.entry_positions) <= max(b, k * b) and min(tr.entry_positions) >= 1
    for p in (4097, 4999, 1234):
        tr = O.Trace()
        O.attend(rng.standard_normal((2, 128)), tree, p, k, causal=True, trace=tr)
        assert max(tr.entry_positions) <= (k + 1) * b


# --------------------------------------------------------------------------- RoPE

def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 128))
    pos = np.array([0, 1, 2, 17, 128, 4095, 1 << 20])
    got = O.rope(x, pos, 1.0e6)
    z = x[:, :64] + 1j * x[:, 64:]
    theta = 1.0e6 ** (-np.arange(64) / 64.0)
    w = z * np.exp(1j * pos[:, None] * theta[None, :])
    assert np.allclose(got[:, :64], w.real, atol=1e-12) and np.allclose(got[:, 64:], w.imag, atol=1e-12)
    assert np.array_equal(O.rope(x, np.zeros(7), 1.0e6), x)
    # dimension 0 turns by exactly 1 rad per position
    e0 = np.zeros(128)
    e0[0] = 1.0
    r = O.rope(e0, 3, 1.0e6)
    assert abs(r[0] - math.cos(3)) < 1e-15 and abs(r[64] - math.sin(3)) < 1e-15


def test_rope_relative_property():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for a, b in [(5, 2), (128, 0), (7, 7), (3, 90)]:
        lhs = O.rope(q, a, 1e6) @ O.rope(k, b, 1e6)
        rhs = q @ O.rope(k, b - a, 1e6)
        assert abs(lhs - rhs) < 1e-10


# --------------------------------------------------------------------------- build

def test_build_values_are_subtree_means_exact_mode():
    rng = np.random.default_rng(3)
    for L, b in [(4096, 8), (1000, 4), (37, 3), (17, 16)]:
        kt, vt = rng.standard_normal((L, 128)), rng.standard_normal((L, 128))
        tree = O.build_tree(kt, vt, np.eye(128), b, storage="exact")
        for lvl in range(1, tree.top + 1):
            span = b ** lvl
            for j in range(tree.values[lvl].shape[0]):
                want = vt[j * span:min((j + 1) * span, L)].mean(axis=0)
                assert np.abs(tree.values[lvl][j] - want).max() < 1e-12
                assert tree.counts[lvl][j] == O.subtree_tokens(lvl, j, b, L)


def test_appending_tokens_leaves_complete_nodes_unchanged():
    # A node depends only on its subtree's tokens (its value is their mean; its key is W applied
    # to its children's stored keys), so growing the cache from L to L + C changes no node whose
    # span ends at or before L, and every node that does change meets [L, L + C) or lies on a
    # level that did not exist.  The incremental update rebuilds exactly those nodes.
    rng = np.random.default_rng(12)
    w = np.linalg.qr(rng.standard_normal((128, 128)))[0]
    for L, C, b in [(1000, 1, 4), (1023, 1, 4), (700, 40, 16), (255, 3, 2)]:
        kt, vt = rng.standard_normal((L + C, 128)), rng.standard_normal((L + C, 128))
        before = O.build_tree(kt[:L], vt[:L], w, b)
        after = O.build_tree(kt, vt, w, b)
        for lvl in range(1, after.top + 1):
            span = b ** lvl
            n_after = after.keys[lvl].shape[0]
            n_before = before.keys[lvl].shape[0] if lvl <= before.top else 0
            for j in range(n_after):
                complete = (j + 1) * span <= L and j < n_before
                same = (j < n_before and np.array_equal(before.keys[lvl][j], after.keys[lvl][j])
                        and np.array_equal(before.values[lvl][j], after.values[lvl][j]))
                if complete:
                    assert same, (L, C, b, lvl, j)
                else:  # the node holds a new token (or its level is new): it is rebuilt
                    assert j * span < L + C and ((j + 1) * span > L or j >= n_before)


def test_build_keys_closed_form_full_nodes():
    # Full nodes: K_l[j] = W^l (subtree token mean); with W = I it is the subtree mean.
    rng = np.random.default_rng(4)
    L, b = 512, 8
    kt = rng.standard_normal((L, 128))
    W = I.pooler_matrix(99).double().numpy()
    tree = O.build_tree(kt, np.zeros((L, 128)), W, b, storage="exact")
    for lvl in range(1, tree.top + 1):
        Wl = np.linalg.matrix_power(W, lvl)
        span = b ** lvl
        for j in range(L // span):
            want = Wl @ kt[j * span:(j + 1) * span].mean(axis=0)
            assert np.abs(tree.keys[lvl][j] - want).max() < 1e-12


def test_build_partial_node_key_is_unweighted_child_mean():
    # b = 2, L = 7: level 1 = [t0+t1, t2+t3, t4+t5]/2 and t6; level 2 node 1 has children
    # (t4+t5)/2 and t6, so its key is (t4+t5)/4 + t6/2 while its value is (t4+t5+t6)/3.
    t = np.zeros((7, 128))
    t[:, 0] = [1, 2, 4, 8, 16, 32, 64]
    tree = O.build_tree(t, t, np.eye(128), 2, storage="exact")
    assert [x.shape[0] for x in tree.keys] == [7, 4, 2]
    assert tree.keys[2][1][0] == (16 + 32) / 4 + 64 / 2
    assert tree.values[2][1][0] == (16 + 32 + 64) / 3
    assert tree.keys[2][0][0] == (1 + 2 + 4 + 8) / 4
    assert tree.values[1][3][0] == 64 and tree.counts[2].tolist() == [4, 3]


def test_build_bf16_mode_rounds_each_stored_row():
    rng = np.random.default_rng(7)
    L, b = 300, 4
    kt = O.round_to_bf16(rng.standard_normal((L, 128)))
    vt = O.round_to_bf16(rng.standard_normal((L, 128)))
    W = I.pooler_matrix(3).double().numpy()
    tb = O.build_tree(kt, vt, W, b, storage="bf16")
    for lvl in range(1, tb.top + 1):
        assert np.array_equal(O.round_to_bf16(tb.keys[lvl]), tb.keys[lvl])
        # each level is the exact build of the stored level below, then rounded
        sub = O.build_tree(tb.keys[lvl - 1], tb.values[lvl - 1], W, b, storage="exact")
        # sub's level 1 is computed from stored children with unit counts; fix the value weights
        cnt = tb.counts[lvl - 1]
        n = tb.keys[lvl].shape[0]
        for j in range(n):
            c0, c1 = j * b, min((j + 1) * b, tb.keys[lvl - 1].shape[0])
            wv = (cnt[c0:c1, None] * tb.values[lvl - 1][c0:c1]).sum(0) / cnt[c0:c1].sum()
            assert np.array_equal(tb.values[lvl][j], O.round_to_bf16(wv))
            assert np.array_equal(tb.keys[lvl][j], O.round_to_bf16(sub.keys[1][j]))


# --------------------------------------------------------------------------- attend invariants

def _tiny():
    w = I.WORKLOADS["tiny_decode"]
    inp = I.decode_inputs(w)
    return w, _bits(inp["k_tok"]), _bits(inp["v_tok"]), _bits(inp["q"]), inp["pooler"].double().numpy()


def test_softmax_weights_sum_to_one():
    w, kb, vb, qb, W = _tiny()
    trees = O.build_all(kb, vb, W, w.branching, w.length)
    for qi in range(w.queries):
        tr = O.Trace()
        O.attend(O.bf16_bits_to_f64(qb[0, qi]), trees[0][0], w.length, w.top_k, trace=tr)
        assert np.abs(tr.weights.sum(axis=1) - 1).max() < 1e-12
        assert tr.weights.shape[1] == 92


def test_topk_all_equals_dense_rope_attention():
    # k >= node count everywhere: every token is read at its original position.
    w, kb, vb, qb, W = _tiny()
    trees = O.build_all(kb, vb, W, w.branching, w.length)
    kt, vt = O.bf16_bits_to_f64(kb[0, 0]), O.bf16_bits_to_f64(vb[0, 0])
    for qi in range(w.queries):
        q = O.bf16_bits_to_f64(qb[0, qi])
        got = O.attend(q, trees[0][0], w.length, O.TOPK_ALL)
        want = O.dense_attention(q, kt, vt, w.length)
        assert np.abs(got - want).max() < 1e-10


def test_topk_all_causal_equals_causal_dense():
    rng = np.random.default_rng(8)
    L, b = 700, 4
    kt, vt = rng.standard_normal((L, 128)), rng.standard_normal((L, 128))
    tree = O.build_tree(kt, vt, I.pooler_matrix(5).double().numpy(), b)
    for p in (1, 3, 4, 5, 64, 65, 699, 256, 257):
        q = rng.standard_normal((3, 128))
        got = O.attend(q, tree, p, O.TOPK_ALL, causal=True)
        want = O.dense_attention(q, kt[:p], vt[:p], p)
        assert np.abs(got - want).max() < 1e-10, p


def test_k0_equals_attention_over_top_summaries():
    w, kb, vb, qb, W = _tiny()
    trees = O.build_all(kb, vb, W, w.branching, w.length)
    t = trees[0][0]
    for qi in range(4):
        q = O.bf16_bits_to_f64(qb[0, qi])
        got = O.attend(q, t, w.length, 0)
        want = O.dense_attention(q, t.keys[t.top], t.values[t.top], t.keys[t.top].shape[0])
        assert np.abs(got - want).max() < 1e-12


def test_ties_keep_lower_index():
    # zero keys score exactly 0 everywhere, so every level ties and keeps its first k candidates
    L, b, k = 256, 4, 3  # levels 256 -> 64 -> 16 -> 4
    rng = np.random.default_rng(9)
    tree = O.build_tree(np.zeros((L, 128)), rng.standard_normal((L, 128)), np.eye(128), b)
    tr = O.Trace()
    O.attend(rng.standard_normal((2, 128)), tree, L, k, trace=tr)
    sel = tr.selections()
    assert sel[0] == [0, 1, 2]
    for s in sel[1:]:
        assert s == [0, 1, 2]


def test_selection_is_a_topk_by_brute_force():
    rng = np.random.default_rng(10)
    for trial in range(20):
        L, b, k = int(rng.integers(20, 600)), int(rng.integers(2, 9)), int(rng.integers(1, 6))
        G = int(rng.choice([1, 2, 4]))
        kt = O.round_to_bf16(rng.standard_normal((L, 128)))
        tree = O.build_tree(kt, rng.standard_normal((L, 128)), I.pooler_matrix(trial).double().numpy(), b)
        tr = O.Trace()
        O.attend(rng.standard_normal((G, 128)), tree, L, k, trace=tr)
        for d in tr.levels:
            if d["level"] == 0:
                continue
            kept = set(d["kept"])
            S = d["S"]
            assert len(kept) == min(k, len(S))
            for a in kept:
                for c in S:
                    if c not in kept:
                        assert S[a] > S[c] or (S[a] == S[c] and a < c)


def test_causal_output_ignores_future_tokens():
    rng = np.random.default_rng(12)
    L, b, k = 900, 4, 2
    kt, vt = rng.standard_normal((L, 128)), rng.standard_normal((L, 128))
    W = I.pooler_matrix(6).double().numpy()
    t1 = O.build_tree(kt, vt, W, b)
    for p in (300, 513, 777):
        k2, v2 = kt.copy(), vt.copy()
        k2[p:] = rng.standard_normal((L - p, 128)) * 5
        v2[p:] = rng.standard_normal((L - p, 128)) * 5
        t2 = O.build_tree(k2, v2, W, b)
        q = rng.standard_normal((4, 128))
        assert np.array_equal(O.attend(q, t1, p, k, causal=True), O.attend(q, t2, p, k, causal=True))


def test_prefill_query_at_aligned_length_equals_decode():
    rng = np.random.default_rng(13)
    b, k = 4, 2
    L = 4 ** 4  # aligned: no partial node at any level
    kt, vt = rng.standard_normal((L + 40, 128)), rng.standard_normal((L + 40, 128))
    W = I.pooler_matrix(7).double().numpy()
    dec = O.build_tree(kt[:L], vt[:L], W, b)
    pre = O.build_tree(kt, vt, W, b)  # tree after a 40-token chunk was appended
    q = rng.standard_normal((4, 128))
    assert np.abs(O.attend(q, dec, L, k) - O.attend(q, pre, L, k, causal=True)).max() < 1e-13


def test_empty_prefix_outputs_zero():
    tree = O.build_tree(np.ones((5, 128)), np.ones((5, 128)), np.eye(128), 2)
    assert np.array_equal(O.attend(np.ones((2, 128)), tree, 0, 3, causal=True), np.zeros((2, 128)))


def test_replay_rejects_a_selection_that_drops_a_clear_winner():
    rng = np.random.default_rng(14)
    L, b, k = 256, 4, 1
    tree = O.build_tree(rng.standard_normal((L, 128)) * 3, rng.standard_normal((L, 128)), np.eye(128), b)
    q = rng.standard_normal((2, 128)) * 3
    tr = O.Trace()
    O.attend(q, tree, L, k, trace=tr)
    sel = tr.selections()
    # keep the worst top-level candidate instead of the best
    S = tr.levels[0]["S"]
    worst = min(S, key=S.get)
    assert S[sel[0][0]] - S[worst] > 1e-3
    with pytest.raises(ValueError):
        O.attend(q, tree, L, k, selection=[[worst]] + sel[1:])
    assert np.array_equal(O.attend(q, tree, L, k, selection=sel), O.attend(q, tree, L, k))


# --------------------------------------------------------------------------- closed-form worked examples

def _e(i, a=1.0):
    v = np.zeros(128)
    v[i] = a
    return v


def test_worked_example_decode_closed_form():
    # b = 4, L = 16: one level of 4 nodes above the tokens (T = 1), k = 1, W = I.
    # Keys are zero except token 9, whose key is A e_0 (dim 0 turns 1 rad per position).
    # Values: v_t = t e_1 + e_2.
    A = -8.0
    L, b = 16, 4
    kt = np.zeros((L, 128))
    kt[9] = _e(0, A)
    vt = np.array([_e(1, t) + _e(2) for t in range(L)])
    tree = O.build_tree(kt, vt, np.eye(128), b, storage="exact")
    q = _e(0)[None, :]
    # top level: 4 candidates at positions 0..3, query at 4.  Node 2's key is (A/4) e_0
    # at position 2, so its logit is s2 = scale (A/4) cos(4 - 2); the rest score 0.
    s2 = SCALE * (A / 4) * math.cos(2)
    assert s2 > 0  # node 2 is kept; nodes 0, 1, 3 join the softmax as summaries (logit 0)
    # token level: children 8..11 at positions 0..3, query at 4; token 9 sits at position 1
    s9 = SCALE * A * math.cos(3)
    means = [vt[4 * j:4 * j + 4].mean(0) for j in (0, 1, 3)]
    num = sum(means) + vt[8] + vt[10] + vt[11] + math.exp(s9) * vt[9]
    want = num / (6 + math.exp(s9))
    tr = O.Trace()
    got = O.attend(q, tree, L, 1, trace=tr)
    assert tr.selections() == [[2]]
    assert np.abs(got[0] - want).max() < 1e-13


def test_worked_example_group_sum_and_tie_break():
    # Same tree; two query heads e_0 and -2 e_0.  The group score of node 2 is
    # s(h0) + s(h1) = -(A/4) scale cos 2 < 0, so nodes 0, 1, 3 tie at 0 and node 0 (lowest) is kept.
    A = -8.0
    L, b = 16, 4
    kt = np.zeros((L, 128))
    kt[9] = _e(0, A)
    vt = np.array([_e(1, t) + _e(2) for t in range(L)])
    tree = O.build_tree(kt, vt, np.eye(128), b, storage="exact")
    q = np.stack([_e(0), _e(0, -2.0)])
    tr = O.Trace()
    got = O.attend(q, tree, L, 1, trace=tr)
    assert tr.selections() == [[0]]
    s2 = SCALE * (A / 4) * math.cos(2) * np.array([1.0, -2.0])  # per-head logit of summary 2
    means = {j: vt[4 * j:4 * j + 4].mean(0) for j in (1, 2, 3)}
    for h in range(2):
        num = means[1] + means[3] + math.exp(s2[h]) * means[2] + vt[0:4].sum(0)
        want = num / (6 + math.exp(s2[h]))
        assert np.abs(got[h] - want).max() < 1e-13


def test_worked_example_causal_forced_partial_node():
    # b = 4, cache of 16 tokens, causal query at p = 10: one level above the tokens
    # (ceil(10/4) = 3 <= 4).  Candidates: complete nodes 0, 1 and the partial node 2
    # (tokens 8, 9 visible), which is forced: not scored, expanded, and it holds a position.
    # Key of token 5 is A e_0; node 1's key is (A/4) e_0 at position 1, query at 3.
    A = 8.0
    L, b, p = 16, 4, 10
    kt = np.zeros((L, 128))
    kt[5] = _e(0, A)
    vt = np.array([_e(1, t) + _e(2) for t in range(L)])
    tree = O.build_tree(kt, vt, np.eye(128), b, storage="exact")
    q = _e(0)[None, :]
    s1 = SCALE * (A / 4) * math.cos(3 - 1)
    assert s1 < 0  # node 0 (logit 0) wins; node 1 joins the softmax as a summary
    tr = O.Trace()
    got = O.attend(q, tree, p, 1, causal=True, trace=tr)
    assert tr.selections() == [[0]]
    assert tr.levels[0]["forced"] == [False, False, True]
    # token level: tokens 0..3 (from node 0) and 8, 9 (from forced node 2) at positions 0..5, query at 6
    num = math.exp(s1) * vt[4:8].mean(0) + vt[0:4].sum(0) + vt[8] + vt[9]
    want = num / (math.exp(s1) + 6)
    assert np.abs(got[0] - want).max() < 1e-13


def test_dense_attention_two_token_closed_form():
    # keys A e_0 at position 0 and 0 at position 1, query e_0 at position 2: the pair
    # (0, 64) turns 1 rad per position, so the first logit is scale * A * cos(2 - 0).
    A = 5.0
    keys = np.stack([_e(0, A), np.zeros(128)])
    vals = np.stack([_e(1), _e(2)])
    s0 = SCALE * A * math.cos(2.0)
    want = (math.exp(s0) * _e(1) + _e(2)) / (math.exp(s0) + 1.0)
    got = O.dense_attention(_e(0)[None, :], keys, vals, 2)
    assert np.abs(got[0] - want).max() < 1e-14


# --------------------------------------------------------------------------- whole-call drivers
# The drivers slice the call's tensors into tiles: query heads g*G .. g*G+G-1 belong to
# KV group g (the repeat-kv convention), decode queries sit at p = L, prefill query i
# at p = L + i, and a chunk arrives as [B][C][Hkv][128].  Each is pinned here against
# inputs whose right answer does not depend on the driver's own slicing.

def _bf16_bits_of(x):
    return O.f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def test_decode_all_groups_query_heads_in_contiguous_blocks():
    # every value row of (sequence s, KV head h) is the constant 10 s + h, so any softmax
    # over that tree outputs exactly 10 s + h: output head j of sequence s must read
    # 10 s + j // G.  An interleaved mapping (j % Hkv) or a swapped sequence fails.
    B, Hkv, G, Q, L, b, k = 2, 2, 4, 3, 40, 4, 2
    rng = np.random.default_rng(21)
    kb = _bf16_bits_of(rng.standard_normal((B, Hkv, L, 128)))
    vals = np.zeros((B, Hkv, L, 128))
    for s in range(B):
        for h in range(Hkv):
            vals[s, h] = 10 * s + h
    vb = _bf16_bits_of(vals)
    qb = _bf16_bits_of(rng.standard_normal((B, Q, Hkv * G, 128)))
    trees = O.build_all(kb, vb, np.eye(128), b, L)
    out = O.decode_all(trees, qb, k)
    for s in range(B):
        for qi in range(Q):
            for j in range(Hkv * G):
                assert np.abs(out[s, qi, j] - (10 * s + j // G)).max() < 1e-12, (s, qi, j)


def test_decode_all_topk_all_is_dense_per_query_head():
    # k = all: each output head is dense RoPE attention of its own query row over its
    # group's tokens at their positions, query at L (checked head by head).
    B, Hkv, G, Q, L, b = 2, 3, 2, 2, 50, 4
    rng = np.random.default_rng(22)
    kb = _bf16_bits_of(rng.standard_normal((B, Hkv, L, 128)))
    vb = _bf16_bits_of(rng.standard_normal((B, Hkv, L, 128)))
    qb = _bf16_bits_of(rng.standard_normal((B, Q, Hkv * G, 128)) * 2)
    out = O.decode_all(O.build_all(kb, vb, np.eye(128), b, L), qb, O.TOPK_ALL)
    for s in range(B):
        for qi in range(Q):
            for j in range(Hkv * G):
                h = j // G
                want = O.dense_attention(O.bf16_bits_to_f64(qb[s, qi, j])[None, :], O.bf16_bits_to_f64(kb[s, h]),
                                         O.bf16_bits_to_f64(vb[s, h]), L)
                assert np.abs(out[s, qi, j] - want[0]).max() < 1e-10, (s, qi, j)


def test_append_chunk_places_token_c_of_head_h_at_row_length_plus_c():
    # each row encodes its place: dims 0, 1, 2 hold (sequence, head, token) + 1, exact in bf16
    B, Hkv, L, C, cap = 2, 3, 5, 4, 12
    full = np.zeros((B, Hkv, L + C, 128))
    for s in range(B):
        for h in range(Hkv):
            for t in range(L + C):
                full[s, h, t, :3] = (s + 1, h + 1, t + 1)
    cache = np.full((B, Hkv, cap, 128), -1.0)
    cache[:, :, :L] = full[:, :, :L]
    chunk = np.zeros((B, C, Hkv, 128))  # the chunk's own layout, filled element by element
    for s in range(B):
        for c in range(C):
            for h in range(Hkv):
                chunk[s, c, h] = full[s, h, L + c]
    kc, vc = O.append_chunk(_bf16_bits_of(cache), _bf16_bits_of(cache), _bf16_bits_of(chunk),
                            _bf16_bits_of(chunk), L)
    assert np.array_equal(O.bf16_bits_to_f64(kc), full)
    assert np.array_equal(O.bf16_bits_to_f64(vc), full)


@pytest.mark.parametrize("L", [0, 37])
def test_prefill_all_query_i_sees_tokens_below_length_plus_i(L):
    # k = all: query i of the chunk is dense RoPE attention over tokens [0, L + i) of its
    # group, at position L + i.  The caches hold garbage past L (only the chunk may fill
    # it) and the chunk's rows are distinct per (sequence, head, token).
    B, Hkv, G, C, b = 2, 2, 2, 6, 4
    rng = np.random.default_rng(23 + L)
    kf = rng.standard_normal((B, Hkv, L + C, 128))
    vf = rng.standard_normal((B, Hkv, L + C, 128))
    kcache = rng.standard_normal((B, Hkv, L + C + 3, 128)) * 50
    vcache = rng.standard_normal((B, Hkv, L + C + 3, 128)) * 50
    kcache[:, :, :L], vcache[:, :, :L] = kf[:, :, :L], vf[:, :, :L]
    knew, vnew = np.zeros((B, C, Hkv, 128)), np.zeros((B, C, Hkv, 128))
    for s in range(B):
        for c in range(C):
            for h in range(Hkv):
                knew[s, c, h], vnew[s, c, h] = kf[s, h, L + c], vf[s, h, L + c]
    qb = _bf16_bits_of(rng.standard_normal((B, C, Hkv * G, 128)))
    out, trees = O.prefill_all(_bf16_bits_of(kcache), _bf16_bits_of(vcache), _bf16_bits_of(knew),
                               _bf16_bits_of(vnew), qb, np.eye(128), b, L, O.TOPK_ALL)
    kf, vf = O.round_to_bf16(kf), O.round_to_bf16(vf)
    for s in range(B):
        for i in range(C):
            for j in range(Hkv * G):
                h = j // G
                want = O.dense_attention(O.bf16_bits_to_f64(qb[s, i, j])[None, :], kf[s, h, :L + i],
                                         vf[s, h, :L + i], L + i)
                assert np.abs(out[s, i, j] - want[0]).max() < 1e-10, (s, i, j)
    assert trees[0][0].length == L + C
