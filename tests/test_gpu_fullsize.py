"""GPU parity at the full sizes of the benchmarked workloads, on sampled outputs.

Every call runs in the launch shape the benchmark times (automatic kernel choice) over
the whole batch; the oracle then rebuilds only the sampled (sequence, KV head) trees and
checks their node rows, the sampled tiles' selections (exact up to validated near-ties)
and outputs, and the tiles' row counts.  The decode cases check every tile of one whole
sequence (all of its KV heads) and a few heads of other sequences.
"""

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_build_b200 as R
import recsa_inputs as I
from oracle import recsa_oracle as O
from parity_helpers import Stats, bits, check_node_rows, check_tile, gpu_selection

pytestmark = pytest.mark.gpu


def _params(w):
    return R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)


def _oracle_tree(inp, s, h, length, b, k_extra=None, v_extra=None):
    kt = O.bf16_bits_to_f64(bits(inp["k_tok"][s, h, :length]))
    vt = O.bf16_bits_to_f64(bits(inp["v_tok"][s, h, :length]))
    if k_extra is not None:
        kt = np.concatenate([kt, O.bf16_bits_to_f64(k_extra)])
        vt = np.concatenate([vt, O.bf16_bits_to_f64(v_extra)])
    return O.build_tree(kt, vt, inp["pooler"].double().cpu().numpy(), b)


def _check_rows(tree_gpu, t_oracle, s, h):
    mism = total = 0
    for lvl in range(1, t_oracle.top + 1):
        kv, vv = tree_gpu.level_rows(lvl)
        n = t_oracle.keys[lvl].shape[0]
        for got, want in ((bits(kv[s, h, :n]), t_oracle.keys[lvl]), (bits(vv[s, h, :n]), t_oracle.values[lvl])):
            m, c = check_node_rows(got, want)
            mism += m
            total += c
    assert mism <= total * 1e-2
    return mism, total


def _decode_case(name, samples):
    w = I.WORKLOADS[name]
    inp = I.decode_inputs(w, device="cuda")
    p = _params(w)
    tree = R.RecsaTree(p, inp["k_tok"], inp["v_tok"], inp["pooler"], w.length)
    ws = R.Workspace(p, tree.capacity, "cuda")
    R.build_tree(p, tree)
    q = inp["q"]
    B, Q, Hq, _ = q.shape
    tiles = B * w.kv_heads * Q
    out = torch.empty(B, Q, Hq, 128, dtype=torch.float32, device="cuda")
    sel = torch.full((tiles, tree.levels, w.top_k), -7, dtype=torch.int32, device="cuda")
    ent = torch.zeros(tiles, 2, dtype=torch.int32, device="cuda")
    R.decode(p, tree, q, out, ws, sel_idx=sel, sel_levels=tree.levels, entries=ent)
    R.check_device_errors(ws)
    out, sel, ent = out.cpu().numpy(), sel.cpu().numpy(), ent.cpu().numpy()
    qb = bits(q)
    G = w.q_heads // w.kv_heads
    stats = Stats()
    for s, h in samples:
        t = _oracle_tree(inp, s, h, w.length, w.branching)
        _check_rows(tree, t, s, h)
        for qi in range(Q):
            tile = (s * w.kv_heads + h) * Q + qi
            check_tile(stats, O.bf16_bits_to_f64(qb[s, qi, h * G:(h + 1) * G]), t, w.length, w.top_k, False,
                       out[s, qi, h * G:(h + 1) * G], gpu_selection(sel, tile, t.top), ent[tile])
    stats.assert_ok()
    print(name, stats)
    return stats


# every KV head (every tile) of one sequence, plus heads of other sequences
def test_decode_131k_batch8():
    _decode_case("decode_131k", [(3, h) for h in range(8)] + [(0, 0), (7, 7)])


def test_decode_1m_batch4_needles():
    _decode_case("decode_1m", [(1, h) for h in range(8)] + [(0, 0), (3, 7)])


def test_build_and_decode_2m():
    _decode_case("build_decode_2m", [(0, h) for h in range(8)])


def test_prefill_524k_chunk_8192():
    w = I.WORKLOADS["prefill_524k"]
    inp = I.prefill_inputs(w, device="cuda")
    p = _params(w)
    tree = R.RecsaTree(p, inp["k_tok"], inp["v_tok"], inp["pooler"], w.length)
    ws = R.Workspace(p, tree.capacity, "cuda")
    R.build_tree(p, tree)
    k_new, v_new, q = inp["k_new"], inp["v_new"], inp["q"]
    C, G = w.chunk, w.q_heads // w.kv_heads
    tiles = w.batch * w.kv_heads * C
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    sel = torch.full((tiles, tree.levels, w.top_k), -7, dtype=torch.int32, device="cuda")
    ent = torch.zeros(tiles, 2, dtype=torch.int32, device="cuda")
    R.prefill_chunk(p, tree, k_new, v_new, q, out, ws, sel_idx=sel, sel_levels=tree.levels, entries=ent)
    R.check_device_errors(ws)
    assert tree.length == w.length + C
    out, sel, ent = out.cpu().numpy(), sel.cpu().numpy(), ent.cpu().numpy()
    qb = bits(q)
    rng = np.random.default_rng(4)
    queries = sorted({0, 1, 15, 16, 255, 256, 4095, C - 1, *rng.choice(C, 12, replace=False).tolist()})
    stats = Stats()
    for h in (1, 6):
        t = _oracle_tree(inp, 0, h, w.length, w.branching, bits(k_new[0, :, h]), bits(v_new[0, :, h]))
        _check_rows(tree, t, 0, h)
        for i in queries:
            tile = h * C + i
            pos = w.length + i
            top = len(O.level_counts(pos, w.branching)) - 1
            check_tile(stats, O.bf16_bits_to_f64(qb[0, i, h * G:(h + 1) * G]), t, pos, w.top_k, True,
                       out[0, i, h * G:(h + 1) * G], gpu_selection(sel, tile, top), ent[tile])
    stats.assert_ok()
    print("prefill_524k", stats)


def test_decode_loop_1m_append_then_decode():
    """The decode loop the benchmark times (1M tokens, B = 4): two steps of recsa_append (one
    token per sequence) + recsa_decode of its query; the sampled trees after both appends and
    the last step's tiles against the oracle over L + 2 tokens."""
    w = I.WORKLOADS["decode_1m"]
    S = 2
    inp = I.decode_inputs(w, device="cuda", capacity=w.length + S + 2)
    p = _params(w)
    tree = R.RecsaTree(p, inp["k_tok"], inp["v_tok"], inp["pooler"], w.length)
    ws = R.Workspace(p, tree.capacity, "cuda")
    R.build_tree(p, tree)
    B, Hkv, Hq, G = w.batch, w.kv_heads, w.q_heads, w.q_heads // w.kv_heads
    g = torch.Generator(device="cuda").manual_seed(61)
    steps = [tuple(torch.randn(B, 1, h, 128, generator=g, device="cuda").to(torch.bfloat16) for h in (Hkv, Hkv, Hq))
             for _ in range(S)]
    tiles = B * Hkv
    for kn, vn, qn in steps:
        R.append(p, tree, kn, vn)
        out = torch.empty(B, 1, Hq, 128, dtype=torch.float32, device="cuda")
        sel = torch.full((tiles, tree.levels, w.top_k), -7, dtype=torch.int32, device="cuda")
        ent = torch.zeros(tiles, 2, dtype=torch.int32, device="cuda")
        R.decode(p, tree, qn, out, ws, sel_idx=sel, sel_levels=tree.levels, entries=ent)
        R.check_device_errors(ws)
    assert tree.length == w.length + S
    out, sel, ent = out.cpu().numpy(), sel.cpu().numpy(), ent.cpu().numpy()
    qb = bits(steps[-1][2])
    stats = Stats()
    for s, h in ((0, 0), (3, 7)):
        kx = np.stack([bits(kn[s, 0, h]) for kn, _, _ in steps])
        vx = np.stack([bits(vn[s, 0, h]) for _, vn, _ in steps])
        t = _oracle_tree(inp, s, h, w.length, w.branching, kx, vx)
        _check_rows(tree, t, s, h)
        tile = s * Hkv + h
        check_tile(stats, O.bf16_bits_to_f64(qb[s, 0, h * G:(h + 1) * G]), t, w.length + S, w.top_k, False,
                   out[s, 0, h * G:(h + 1) * G], gpu_selection(sel, tile, t.top), ent[tile])
    stats.assert_ok()
    print("decode_loop_1m", stats)
