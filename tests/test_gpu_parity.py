"""GPU parity of the CUDA library against the fp64 oracle on small seeded cases.

Sizes span several gather chunks and tree levels, with ragged tails (partial nodes),
degenerate trees (L <= b, L = 1), every supported query-group size and every
cluster shape.  Calls go through the C ABI via the ctypes binding.
"""

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_build_b200 as R
import recsa_inputs as I
from oracle import recsa_oracle as O
from parity_helpers import GpuCase, Stats, bits, check_node_rows, check_tile, gpu_selection, oracle_trees

pytestmark = pytest.mark.gpu


def _params(hkv, g, b, k):
    return R.params(num_kv_heads=hkv, num_q_heads=hkv * g, branching=b, top_k=k)


def _compare_build(case: GpuCase, trees, b):
    total = mism = 0
    for lvl in range(1, case.tree.levels + 1):
        if lvl > trees[0][0].top:
            break
        kb, vb = case.node_bits(lvl)
        for s in range(len(trees)):
            for h in range(len(trees[0])):
                t = trees[s][h]
                n = t.keys[lvl].shape[0]
                for got, want in ((kb[s, h, :n], t.keys[lvl]), (vb[s, h, :n], t.values[lvl])):
                    m, c = check_node_rows(got, want)
                    mism += m
                    total += c
    return mism, total


# launch shapes: (kernel, cluster_size); kernel 1 = CTA/cluster per tile, 2 = warp per tile,
# 3 = lean cluster per tile (score exchange by DSMEM stores)
SHAPES = [(1, 1), (1, 2), (1, 4), (2, 0), (3, 2), (3, 4)]


def _decode_and_check(case, trees, q, k, cluster_size=0, kernel=0):
    out, sel, ent = case.decode(q, cluster_size=cluster_size, kernel=kernel)
    p = case.p
    G = p.num_q_heads // p.num_kv_heads
    B, Q = q.shape[:2]
    qb = bits(q)
    stats = Stats()
    for s in range(B):
        for h in range(p.num_kv_heads):
            t = trees[s][h]
            for qi in range(Q):
                tile = (s * p.num_kv_heads + h) * Q + qi
                gsel = gpu_selection(sel, tile, t.top) if sel is not None else None
                check_tile(stats, O.bf16_bits_to_f64(qb[s, qi, h * G:(h + 1) * G]), t, t.length, k, False,
                           out[s, qi, h * G:(h + 1) * G].numpy(), gsel, ent[tile])
    stats.assert_ok()
    return stats


def test_build_tiny_matches_oracle_rows():
    w = I.WORKLOADS["tiny_decode"]
    inp = I.decode_inputs(w)
    case = GpuCase(inp, _params(1, 4, w.branching, w.top_k), w.length)
    case.build()
    torch.cuda.synchronize()
    mism, total = _compare_build(case, oracle_trees(inp, w.branching, w.length), w.branching)
    print(f"tiny build: {mism} of {total} elements not bit-identical")
    assert mism <= total * 1e-2


@pytest.mark.parametrize("B,hkv,L,cap,b", [(2, 2, 1000, 1000, 3), (1, 1, 17, 40, 16), (1, 3, 5, 5, 2),
                                           (3, 2, 4097, 5000, 8), (1, 1, 1, 8, 4), (1, 2, 300, 300, 300)])
def test_build_odd_shapes_match_oracle_rows(B, hkv, L, cap, b):
    inp = I.random_case(B, L, hkv, hkv * 4, 1, seed=100 + L, capacity=cap)
    case = GpuCase(inp, _params(hkv, 4, b, 2), L)
    case.build()
    torch.cuda.synchronize()
    mism, total = _compare_build(case, oracle_trees(inp, b, L), b)
    assert mism <= max(2, total * 1e-2)
    print(f"build: {mism} of {total} elements not bit-identical")


@pytest.mark.parametrize("kernel,cluster_size", [(0, 0)] + SHAPES)
def test_decode_tiny_end_to_end(kernel, cluster_size):
    w = I.WORKLOADS["tiny_decode"]
    inp = I.decode_inputs(w)
    case = GpuCase(inp, _params(1, 4, w.branching, w.top_k), w.length)
    case.build()
    stats = _decode_and_check(case, oracle_trees(inp, w.branching, w.length), inp["q"], w.top_k, cluster_size,
                              kernel)
    print("tiny decode", kernel, cluster_size, stats)


def test_decode_tiny_attend_on_oracle_tree():
    # the node arena is filled from the oracle's bf16 tree, so only the attend kernel is compared
    w = I.WORKLOADS["tiny_decode"]
    inp = I.decode_inputs(w)
    case = GpuCase(inp, _params(1, 4, w.branching, w.top_k), w.length)
    trees = oracle_trees(inp, w.branching, w.length)
    for lvl in range(1, trees[0][0].top + 1):
        kv, vv = case.tree.level_rows(lvl)
        n = trees[0][0].keys[lvl].shape[0]
        for dst, src in ((kv, trees[0][0].keys[lvl]), (vv, trees[0][0].values[lvl])):
            b16 = torch.from_numpy(O.f64_to_bf16_bits(src).view(np.int16)).view(torch.bfloat16)
            dst[0, 0, :n].copy_(b16.to(dst.device))
    stats = _decode_and_check(case, trees, inp["q"], w.top_k)
    print("tiny attend on oracle tree", stats)


@pytest.mark.parametrize("kernel,cluster_size", SHAPES)
def test_decode_topk_all_equals_dense_attention(kernel, cluster_size):
    w = I.WORKLOADS["tiny_decode"]
    inp = I.decode_inputs(w)
    case = GpuCase(inp, _params(1, 4, w.branching, R.TOPK_ALL), w.length)
    case.build()
    out, _, ent = case.decode(inp["q"], cluster_size=cluster_size, kernel=kernel)
    kt, vt = O.bf16_bits_to_f64(bits(inp["k_tok"])[0, 0]), O.bf16_bits_to_f64(bits(inp["v_tok"])[0, 0])
    qb = bits(inp["q"])
    stats = Stats()
    for qi in range(w.queries):
        want = O.dense_attention(O.bf16_bits_to_f64(qb[0, qi]), kt, vt, w.length)
        stats.add(out[0, qi].numpy() - want)
        assert ent[qi, 0] == w.length + 8 + 64 + 512 and ent[qi, 1] == w.length
    stats.assert_ok()
    print("k=all vs dense", stats)


@pytest.mark.parametrize("kernel,cluster_size", SHAPES)
def test_decode_k0_is_attention_over_top_summaries(kernel, cluster_size):
    w = I.WORKLOADS["tiny_decode"]
    inp = I.decode_inputs(w)
    case = GpuCase(inp, _params(1, 4, w.branching, 0), w.length)
    case.build()
    out, _, _ = case.decode(inp["q"], cluster_size=cluster_size, kernel=kernel)
    t = oracle_trees(inp, w.branching, w.length)[0][0]
    qb = bits(inp["q"])
    stats = Stats()
    for qi in range(w.queries):
        want = O.dense_attention(O.bf16_bits_to_f64(qb[0, qi]), t.keys[t.top], t.values[t.top], t.keys[t.top].shape[0])
        stats.add(out[0, qi].numpy() - want)
    stats.assert_ok()


@pytest.mark.parametrize("B,hkv,G,L,b,k,Q", [
    (2, 2, 1, 1000, 3, 2, 3),      # ragged tails at every level, b = 3
    (1, 1, 2, 17, 16, 8, 2),       # one partial node
    (1, 1, 8, 5, 2, 1, 1),         # b = 2, G = 8
    (3, 2, 4, 4097, 8, 3, 2),      # one token past a power of b
    (1, 1, 4, 16, 16, 8, 1),       # L <= b: plain attention (no level above the tokens)
    (1, 1, 4, 1, 16, 8, 1),        # a single token
    (1, 2, 4, 3000, 5, 40, 1),     # many candidates per level (several gather chunks)
    (2, 1, 4, 2048, 4, 1, 4),      # k = 1
    (1, 2, 4, 20000, 2, 2, 2),     # b = 2: 14 levels above the tokens
])
@pytest.mark.parametrize("kernel,cluster_size", [(1, 1), (1, 4), (2, 0), (3, 2), (3, 4)])
def test_decode_odd_shapes(B, hkv, G, L, b, k, Q, kernel, cluster_size):
    inp = I.random_case(B, L, hkv, hkv * G, Q, seed=7 * L + b)
    case = GpuCase(inp, _params(hkv, G, b, k), L)
    case.build()
    _decode_and_check(case, oracle_trees(inp, b, L), inp["q"], k, cluster_size, kernel)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("kernel", [0, 1, 4])
def test_decode_more_tiles_than_sms(G, kernel):
    # 40 queries per sequence: 160 to 640 tiles, more than the B200's 148 SMs, where a CTA per
    # tile runs two CTAs per SM (G <= 4) and the automatic choice picks that shape up to 592
    B, hkv, L, b, k, Q = 2, max(2, 8 // G), 3000, 8, 4, 40
    inp = I.random_case(B, L, hkv, hkv * G, Q, seed=11 * G + kernel)
    case = GpuCase(inp, _params(hkv, G, b, k), L)
    case.build()
    assert B * hkv * Q > 148
    _decode_and_check(case, oracle_trees(inp, b, L), inp["q"], k, 0, kernel)


@pytest.mark.parametrize("kernel,cluster_size", SHAPES)
def test_decode_ties_keep_lower_index(kernel, cluster_size):
    L, b, k = 4096, 8, 3
    inp = I.random_case(1, L, 1, 4, 2, seed=3)
    inp["k_tok"].zero_()  # every score is exactly 0
    case = GpuCase(inp, _params(1, 4, b, k), L)
    case.build()
    _, sel, _ = case.decode(inp["q"], cluster_size=cluster_size, kernel=kernel)
    for tile in range(2):
        for lvl_sel in gpu_selection(sel, tile, 3):
            assert lvl_sel == [0, 1, 2]


@pytest.mark.parametrize("kernel", [1, 2, 3])
def test_decode_bf16_output_is_rounded_fp32_output(kernel):
    w = I.WORKLOADS["tiny_decode"]
    inp = I.decode_inputs(w)
    case = GpuCase(inp, _params(1, 4, w.branching, w.top_k), w.length)
    case.build()
    o32, _, _ = case.decode(inp["q"], kernel=kernel)
    o16, _, _ = case.decode(inp["q"], fp32=False, kernel=kernel)
    assert torch.equal(o32.to(torch.bfloat16), o16)


def _prefill_check(B, hkv, G, L, C, b, k, cluster_size=0, seed=1, kernel=0):
    cap = L + C
    inp = I.random_case(B, L, hkv, hkv * G, 0, seed=seed, capacity=cap, chunk=C)
    case = GpuCase(inp, _params(hkv, G, b, k), L)
    if L:
        case.build()
    out, sel, ent = case.prefill(inp["k_new"], inp["v_new"], inp["q"], cluster_size=cluster_size, kernel=kernel)
    assert case.tree.length == L + C
    kb, vb = bits(inp["k_tok"]), bits(inp["v_tok"])
    kc, vc = O.append_chunk(kb, vb, bits(inp["k_new"]), bits(inp["v_new"]), L)
    trees = O.build_all(kc, vc, inp["pooler"].double().numpy(), b, L + C)
    # the extended tree equals a fresh build over L + C tokens
    mism = 0
    for lvl in range(1, trees[0][0].top + 1):
        gk, gv = case.node_bits(lvl)
        for s in range(B):
            for h in range(hkv):
                t = trees[s][h]
                n = t.keys[lvl].shape[0]
                for got, want in ((gk[s, h, :n], t.keys[lvl]), (gv[s, h, :n], t.values[lvl])):
                    mism += check_node_rows(got, want)[0]
    qb = bits(inp["q"])
    stats = Stats()
    for s in range(B):
        for h in range(hkv):
            t = trees[s][h]
            for i in range(C):
                tile = (s * hkv + h) * C + i
                p = L + i
                top = len(O.level_counts(p, b)) - 1
                gsel = gpu_selection(sel, tile, top) if sel is not None else None
                check_tile(stats, O.bf16_bits_to_f64(qb[s, i, h * G:(h + 1) * G]), t, p, k, True,
                           out[s, i, h * G:(h + 1) * G].numpy(), gsel, ent[tile])
    stats.assert_ok()
    return stats, out


@pytest.mark.parametrize("B,hkv,G,L,C,b,k", [
    (2, 2, 4, 1000, 300, 4, 2),
    (1, 1, 4, 4096, 64, 8, 4),     # aligned cache
    (1, 2, 2, 777, 260, 3, 3),     # partial nodes at every level, b = 3
    (1, 1, 8, 250, 20, 16, 8),     # the chunk crosses into a new top level
])
@pytest.mark.parametrize("kernel", [0, 1, 2, 4])
def test_prefill_chunk_matches_oracle(B, hkv, G, L, C, b, k, kernel):
    stats, _ = _prefill_check(B, hkv, G, L, C, b, k, kernel=kernel)
    print("prefill", kernel, stats)


@pytest.mark.parametrize("kernel,cluster_size", SHAPES)
def test_prefill_launch_shapes(kernel, cluster_size):
    _prefill_check(1, 1, 4, 500, 40, 4, 2, cluster_size=cluster_size, seed=9, kernel=kernel)


def test_prefill_from_empty_cache():
    stats, out = _prefill_check(1, 2, 4, 0, 150, 4, 2)
    assert torch.count_nonzero(out[:, 0]) == 0  # query 0 sees nothing


def test_prefill_then_decode():
    L, C, b, k = 600, 200, 4, 2
    inp = I.random_case(1, L, 1, 4, 3, seed=21, capacity=L + C, chunk=C)
    case = GpuCase(inp, _params(1, 4, b, k), L)
    case.build()
    case.prefill(inp["k_new"], inp["v_new"], torch.randn(1, C, 4, 128).to(torch.bfloat16))
    q = torch.randn(1, 3, 4, 128, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    kc, vc = O.append_chunk(bits(inp["k_tok"]), bits(inp["v_tok"]), bits(inp["k_new"]), bits(inp["v_new"]), L)
    trees = O.build_all(kc, vc, inp["pooler"].double().numpy(), b, L + C)
    _decode_and_check(case, trees, q, k)


def test_token_by_token_decode_loop():
    """A decode loop: each step appends one token (chunk of 1) and attends its query, so the
    tree is extended by one node per level per step; the steps cross 1024 = 4^5 tokens, where
    a new top level appears.  Every step against the oracle, then the node rows against a
    fresh build over all tokens."""
    L, S, b, k, hkv, G = 1021, 6, 4, 2, 2, 4
    inp = I.random_case(1, L, hkv, hkv * G, 1, seed=33, capacity=L + S, chunk=S)
    case = GpuCase(inp, _params(hkv, G, b, k), L)
    case.build()
    kc, vc = bits(inp["k_tok"]), bits(inp["v_tok"])
    pooler = inp["pooler"].double().numpy()
    stats = Stats()
    for s in range(S):
        kn, vn, qs = (inp[x][:, s:s + 1].contiguous() for x in ("k_new", "v_new", "q"))
        out, sel, ent = case.prefill(kn, vn, qs)
        assert case.tree.length == L + s + 1
        kc, vc = O.append_chunk(kc, vc, bits(kn), bits(vn), L + s)
        trees = O.build_all(kc, vc, pooler, b, L + s + 1)
        p = L + s
        top = len(O.level_counts(p, b)) - 1
        qb = bits(qs)
        for h in range(hkv):
            check_tile(stats, O.bf16_bits_to_f64(qb[0, 0, h * G:(h + 1) * G]), trees[0][h], p, k, True,
                       out[0, 0, h * G:(h + 1) * G].numpy(), gpu_selection(sel, h, top), ent[h])
    stats.assert_ok()
    mism = total = 0
    for lvl in range(1, trees[0][0].top + 1):
        gk, gv = case.node_bits(lvl)
        for h in range(hkv):
            t = trees[0][h]
            n = t.keys[lvl].shape[0]
            for got, want in ((gk[0, h, :n], t.keys[lvl]), (gv[0, h, :n], t.values[lvl])):
                m, c = check_node_rows(got, want)
                mism += m
                total += c
    assert mism <= total * 1e-2
    print("decode loop", stats)


def test_prefill_levels_past_128_candidates():
    # causal, b = 16, k = 8: a level holds up to (k + 1) b = 144 candidates, so the cluster
    # kernel takes 3 rows per half-warp and ranks by the generic count (24 tiles: automatic
    # launch picks 4-CTA clusters)
    stats, _ = _prefill_check(1, 1, 4, 3000, 24, 16, 8, seed=5)
    print("prefill 144 candidates", stats)


@pytest.mark.parametrize("pinned", [True, False])
def test_decode_from_host_buffers_equals_decode(pinned):
    """recsa_decode_host: host queries in, host outputs back, one call; the same results as
    recsa_decode on device buffers (fp32 and bf16 outputs).  Pinned buffers are read and
    written by the kernel through their device mapping, pageable ones through the staging
    buffers."""
    w = I.WORKLOADS["tiny_decode"]
    inp = I.decode_inputs(w, device="cpu")
    case = GpuCase(inp, _params(w.kv_heads, w.q_heads // w.kv_heads, w.branching, w.top_k), w.length)
    case.build()
    q = inp["q"].contiguous()
    for dtype in (torch.float32, torch.bfloat16):
        out_ref = torch.empty(q.shape, dtype=dtype, device="cuda")
        R.decode(case.p, case.tree, q.cuda(), out_ref, case.ws)
        q_host = q.clone()
        out_host = torch.full(q.shape, -3.0, dtype=dtype)
        if pinned:
            q_host, out_host = q_host.pin_memory(), out_host.pin_memory()
        q_dev = torch.zeros(q.shape, dtype=torch.bfloat16, device="cuda")
        out_dev = torch.zeros(q.shape, dtype=dtype, device="cuda")
        R.decode_host(case.p, case.tree, q_host, out_host, q_dev, out_dev, case.ws)
        torch.cuda.synchronize()
        R.check_device_errors(case.ws)
        assert torch.equal(out_host, out_ref.cpu())
        # the staging buffers are used exactly when the host buffers are pageable
        assert (torch.count_nonzero(out_dev).item() == 0) == pinned
