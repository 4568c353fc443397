"""GPU parity of recsa_append (token append + update of the nodes over the new tokens).

The appended tree is held to the oracle level by level (each level's rows against the
oracle's level step over the library's own rows below, within two bf16 ulps of each row's
largest element), to the oracle's fresh build over all tokens up to 8 levels deep, the
token slots bit for bit,
and to the library's own full build bit for bit: both paths of the update (one launch
walking each head's ancestor path, and the per-level launches used for long chunks)
share the level build's per-node arithmetic.  A decode loop of append + decode is held
to the oracle at every step.
"""

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_build_b200 as R
import recsa_inputs as I
from oracle import recsa_oracle as O
from parity_helpers import GpuCase, Stats, bits, check_node_rows, check_tile, gpu_selection

pytestmark = pytest.mark.gpu


def _params(hkv, g, b, k):
    return R.params(num_kv_heads=hkv, num_q_heads=hkv * g, branching=b, top_k=k)


def _compare_nodes(case, trees):
    mism = total = 0
    for lvl in range(1, trees[0][0].top + 1):
        gk, gv = case.node_bits(lvl)
        for s in range(len(trees)):
            for h in range(len(trees[0])):
                t = trees[s][h]
                n = t.keys[lvl].shape[0]
                for got, want in ((gk[s, h, :n], t.keys[lvl]), (gv[s, h, :n], t.values[lvl])):
                    m, c = check_node_rows(got, want)
                    mism += m
                    total += c
    return mism, total


def _compare_levels_stepwise(case, kc, vc, pooler, B, hkv, length, b):
    """Each level's rows against the oracle's level step applied to the library's own
    stored rows of the level below: the node-row bar for one level's arithmetic, whatever
    the depth.  Returns (elements not bit-identical, total)."""
    mism = total = 0
    top = len(O.level_counts(length, b)) - 1
    gpu = [case.node_bits(lvl) for lvl in range(1, top + 1)]
    for s in range(B):
        for h in range(hkv):
            kp = O.bf16_bits_to_f64(kc[s, h, :length])
            vp = O.bf16_bits_to_f64(vc[s, h, :length])
            cp = np.ones(length)
            for lvl in range(1, top + 1):
                kn, vn, cn = O.build_level(kp, vp, cp, pooler, b)
                gk, gv = gpu[lvl - 1][0][s, h, :kn.shape[0]], gpu[lvl - 1][1][s, h, :kn.shape[0]]
                for got, want in ((gk, kn), (gv, vn)):
                    m, c = check_node_rows(got, want)
                    mism += m
                    total += c
                kp, vp, cp = O.bf16_bits_to_f64(gk), O.bf16_bits_to_f64(gv), cn
    return mism, total


def _appended_case(B, hkv, L, C, b, seed, k=2, G=4, extra=0):
    inp = I.random_case(B, L, hkv, hkv * G, 0, seed=seed, capacity=L + C + extra, chunk=C)
    case = GpuCase(inp, _params(hkv, G, b, k), L)
    if L:
        case.build()
    R.append(case.p, case.tree, inp["k_new"].cuda().contiguous(), inp["v_new"].cuda().contiguous())
    R.check_device_errors(case.ws)
    torch.cuda.synchronize()
    assert case.tree.length == L + C
    return inp, case


# (B, hkv, L, C, b): the one-launch path for a token or a short chunk (at most 4 nodes a
# level), the per-level path for longer chunks, new top levels, an empty and a tiny cache
CASES = [
    (2, 2, 1000, 1, 4),      # one token, ragged nodes at every level
    (1, 2, 1023, 1, 4),      # 1024 = 4^5 tokens: a new top level appears
    (1, 1, 4095, 5, 16),     # 4100 tokens: a new level of 2 nodes over 17
    (2, 3, 777, 7, 3),       # b = 3
    (1, 1, 500, 40, 16),     # 3 level-1 nodes rebuilt in one launch
    (1, 2, 0, 3, 4),         # empty cache, no level yet
    (1, 2, 2, 30, 4),        # 8 level-1 nodes from scratch: per-level launches
    (1, 1, 100, 200, 4),     # a long chunk: per-level launches
    (3, 8, 4096, 1, 16),     # 24 (sequence, head) warps over 3 blocks
    (1, 2, 70000, 1, 2),     # b = 2: 16 levels, one node each, carried up the single-token path
]


@pytest.mark.parametrize("B,hkv,L,C,b", CASES)
def test_append_matches_oracle(B, hkv, L, C, b):
    inp, case = _appended_case(B, hkv, L, C, b, seed=L + 7 * C + b)
    kc, vc = O.append_chunk(bits(inp["k_tok"]), bits(inp["v_tok"]), bits(inp["k_new"]), bits(inp["v_new"]), L)
    # token slots: the new rows in place, every other slot untouched
    assert np.array_equal(bits(case.k_tok)[:, :, :L + C], kc[:, :, :L + C])
    assert np.array_equal(bits(case.v_tok)[:, :, :L + C], vc[:, :, :L + C])
    W = inp["pooler"].double().numpy()
    mism, total = _compare_levels_stepwise(case, kc, vc, W, B, hkv, L + C, b)
    assert mism <= max(total, 1) * 1e-2
    trees = O.build_all(kc, vc, W, b, L + C)
    assert case.tree.levels >= trees[0][0].top
    # the whole tree against the oracle's own: rows rounded independently on both sides drift
    # apart by about sqrt(depth) half-ulps as they pass up the levels, past the two-ulp bar in
    # deep trees (b = 2, 16 levels: 2.5 ulps seen), so this holds up to 8 levels
    if trees[0][0].top <= 8:
        mism, total = _compare_nodes(case, trees)
        assert mism <= max(total, 1) * 1e-2


@pytest.mark.parametrize("B,hkv,L,C,b", CASES)
def test_append_equals_full_build_bit_for_bit(B, hkv, L, C, b):
    inp, case = _appended_case(B, hkv, L, C, b, seed=3 * L + C)
    fresh = GpuCase(inp, case.p, L + C)
    fresh.k_tok.copy_(case.k_tok)
    fresh.v_tok.copy_(case.v_tok)
    fresh.build()
    torch.cuda.synchronize()
    top = len(O.level_counts(L + C, b)) - 1
    for lvl in range(1, top + 1):
        n = O.level_counts(L + C, b)[lvl]
        for a, f in zip(case.node_bits(lvl), fresh.node_bits(lvl)):
            assert np.array_equal(a[:, :, :n], f[:, :, :n]), lvl


def test_append_keeps_rows_beyond_the_update():
    """Nodes whose spans end before the first new token are not rewritten."""
    B, hkv, L, b = 1, 2, 1000, 4
    inp = I.random_case(B, L, hkv, hkv * 4, 0, seed=5, capacity=L + 1, chunk=1)
    case = GpuCase(inp, _params(hkv, 4, b, 2), L)
    case.build()
    torch.cuda.synchronize()
    before = [case.node_bits(l) for l in range(1, case.tree.levels + 1)]
    R.append(case.p, case.tree, inp["k_new"].cuda().contiguous(), inp["v_new"].cuda().contiguous())
    torch.cuda.synchronize()
    for lvl in range(1, len(before) + 1):
        j0 = L // b ** lvl  # first node that holds token L
        for a, bb in zip(before[lvl - 1], case.node_bits(lvl)):
            assert np.array_equal(a[:, :, :j0], bb[:, :, :j0]), lvl


def test_append_then_decode_loop():
    """A decode loop: each step appends the step's token (its K and V) and decodes its
    query over all tokens so far; the steps cross 1024 = 4^5 tokens, where a new top level
    appears.  Every step against the oracle."""
    L, S, b, k, hkv, G = 1021, 6, 4, 2, 2, 4
    inp = I.random_case(1, L, hkv, hkv * G, 0, seed=41, capacity=L + S, chunk=S)
    case = GpuCase(inp, _params(hkv, G, b, k), L)
    case.build()
    kc, vc = bits(inp["k_tok"]), bits(inp["v_tok"])
    pooler = inp["pooler"].double().numpy()
    stats = Stats()
    for s in range(S):
        kn, vn, qs = (inp[x][:, s:s + 1].contiguous() for x in ("k_new", "v_new", "q"))
        R.append(case.p, case.tree, kn.cuda(), vn.cuda())
        out, sel, ent = case.decode(qs)
        assert case.tree.length == L + s + 1
        kc, vc = O.append_chunk(kc, vc, bits(kn), bits(vn), L + s)
        trees = O.build_all(kc, vc, pooler, b, L + s + 1)
        qb = bits(qs)
        for h in range(hkv):
            t = trees[0][h]
            check_tile(stats, O.bf16_bits_to_f64(qb[0, 0, h * G:(h + 1) * G]), t, t.length, k, False,
                       out[0, 0, h * G:(h + 1) * G].numpy(), gpu_selection(sel, h, t.top), ent[h])
    stats.assert_ok()
    print("append + decode loop", stats)


def test_append_rejects_overflow_without_queuing():
    inp = I.random_case(1, 10, 1, 4, 0, seed=2, capacity=12, chunk=3)
    case = GpuCase(inp, _params(1, 4, 4, 2), 10)
    case.build()
    with pytest.raises(R.RecsaError):
        R.append(case.p, case.tree, inp["k_new"].cuda().contiguous(), inp["v_new"].cuda().contiguous())
    assert case.tree.length == 10
