"""GPU parity of batches whose sequences have their own lengths (recsa_tree.seq_len).

Every sequence is held to the oracle's tree over its own tokens: node rows after a build,
decode tiles at p = its own length (a sequence of length 0 outputs zeros), an append loop
and a causal prefill chunk at its own offset.  With every length equal, the per-sequence
path gives the same bits as the uniform one.  An out-of-range entry is flagged, not faulted.
"""

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_build_b200 as R
import recsa_inputs as I
from oracle import recsa_oracle as O
from parity_helpers import Stats, bits, check_node_rows, check_tile, gpu_selection

pytestmark = pytest.mark.gpu

SHAPES = [(0, 0), (1, 1), (1, 4), (2, 0), (3, 2), (3, 4)]


class VarCase:
    """Device caches of the longest length, a per-sequence length tensor and a workspace."""

    def __init__(self, lens, hkv, G, b, k, seed, extra=0, chunk=0, queries=1):
        self.lens = list(lens)
        self.B, self.hkv, self.G, self.b, self.k = len(lens), hkv, G, b, k
        L = max(lens)
        self.inp = I.random_case(self.B, L, hkv, hkv * G, queries, seed=seed, capacity=L + extra + chunk,
                                 chunk=chunk)
        self.p = R.params(num_kv_heads=hkv, num_q_heads=hkv * G, branching=b, top_k=k)
        self.k_tok = self.inp["k_tok"].cuda().contiguous()
        self.v_tok = self.inp["v_tok"].cuda().contiguous()
        self.seq_len = torch.tensor(self.lens, dtype=torch.int64, device="cuda")
        self.tree = R.RecsaTree(self.p, self.k_tok, self.v_tok, self.inp["pooler"].cuda().contiguous(), L,
                                seq_len=self.seq_len)
        self.ws = R.Workspace(self.p, self.tree.capacity, "cuda")
        self.pooler = self.inp["pooler"].double().numpy()

    def oracle_tree(self, s, h, n, kb=None, vb=None):
        kb = bits(self.k_tok) if kb is None else kb
        vb = bits(self.v_tok) if vb is None else vb
        return O.build_tree(O.bf16_bits_to_f64(kb[s, h, :n]), O.bf16_bits_to_f64(vb[s, h, :n]), self.pooler, self.b)

    def decode(self, q, kernel=0, cluster_size=0):
        B, Q, Hq, _ = q.shape
        tiles = B * self.hkv * Q
        lv = max(self.tree.levels, 1)
        sel = torch.full((tiles, lv, self.k), -7, dtype=torch.int32, device="cuda")
        ent = torch.zeros(tiles, 2, dtype=torch.int32, device="cuda")
        out = torch.empty(B, Q, Hq, 128, dtype=torch.float32, device="cuda")
        R.decode(self.p, self.tree, q.cuda().contiguous(), out, self.ws, sel_idx=sel, sel_levels=lv, entries=ent,
                 kernel=kernel, cluster_size=cluster_size)
        R.check_device_errors(self.ws)
        return out.cpu(), sel.cpu().numpy(), ent.cpu().numpy()

    def check_decode(self, q, out, sel, ent, lens):
        Q = q.shape[1]
        qb = bits(q)
        stats = Stats()
        G = self.G
        for s in range(self.B):
            for h in range(self.hkv):
                if lens[s] == 0:
                    assert torch.count_nonzero(out[s, :, h * G:(h + 1) * G]) == 0
                    continue
                t = self.oracle_tree(s, h, lens[s])
                for qi in range(Q):
                    tile = (s * self.hkv + h) * Q + qi
                    check_tile(stats, O.bf16_bits_to_f64(qb[s, qi, h * G:(h + 1) * G]), t, lens[s], self.k, False,
                               out[s, qi, h * G:(h + 1) * G].numpy(), gpu_selection(sel, tile, t.top), ent[tile])
        stats.assert_ok()
        return stats


@pytest.mark.parametrize("lens,hkv,b", [
    ([1000, 1, 257, 64, 1021], 2, 4),   # ragged lengths, one of a single token
    ([4096, 300, 4095, 17], 1, 16),     # a full tree next to shallow ones
    ([0, 700, 3], 2, 3),                # an empty sequence, b = 3
])
def test_varlen_build_matches_oracle(lens, hkv, b):
    c = VarCase(lens, hkv, 4, b, 2, seed=sum(lens) % 97)
    R.build_tree(c.p, c.tree)
    torch.cuda.synchronize()
    mism = total = 0
    for lvl in range(1, c.tree.levels + 1):
        gk, gv = (bits(x) for x in c.tree.level_rows(lvl))
        for s, n in enumerate(lens):
            counts = O.level_counts(n, b) if n else [0]
            if lvl >= len(counts):
                continue
            for h in range(hkv):
                t = c.oracle_tree(s, h, n)
                m = counts[lvl]
                for got, want in ((gk[s, h, :m], t.keys[lvl]), (gv[s, h, :m], t.values[lvl])):
                    a, tt = check_node_rows(got, want)
                    mism += a
                    total += tt
    assert total > 0 and mism <= total * 1e-2


@pytest.mark.parametrize("kernel,cluster_size", SHAPES)
def test_varlen_decode_matches_oracle(kernel, cluster_size):
    lens = [1000, 1, 257, 0, 64, 1021]
    c = VarCase(lens, 2, 4, 4, 2, seed=3, queries=2)
    R.build_tree(c.p, c.tree)
    q = c.inp["q"]
    out, sel, ent = c.decode(q, kernel, cluster_size)
    c.check_decode(q, out, sel, ent, lens)


@pytest.mark.parametrize("kernel,cluster_size", SHAPES)
def test_equal_lengths_give_the_uniform_bits(kernel, cluster_size):
    lens = [777, 777, 777]
    c = VarCase(lens, 2, 4, 4, 2, seed=8, queries=3)
    R.build_tree(c.p, c.tree)
    out_v, sel_v, _ = c.decode(c.inp["q"], kernel, cluster_size)
    u = R.RecsaTree(c.p, c.k_tok, c.v_tok, c.inp["pooler"].cuda().contiguous(), 777)
    R.build_tree(c.p, u)
    out_u = torch.empty_like(out_v, device="cuda")
    R.decode(c.p, u, c.inp["q"].cuda().contiguous(), out_u, c.ws, kernel=kernel, cluster_size=cluster_size)
    R.check_device_errors(c.ws)
    assert torch.equal(out_v, out_u.cpu())
    for lvl in range(1, len(O.level_counts(777, 4))):
        n = O.level_counts(777, 4)[lvl]
        for a, b in zip(c.tree.level_rows(lvl), u.level_rows(lvl)):
            assert np.array_equal(bits(a)[:, :, :n], bits(b)[:, :, :n])


def test_varlen_append_decode_loop():
    """Each step appends one token to every sequence at its own end, then decodes the new
    query; the lengths cross 1024 = 4^5 (a new top level) in one sequence and start at 0 in
    another.  Every step against the oracle; the device lengths advance with the calls."""
    lens = [700, 1022, 0, 64]
    S = 4
    c = VarCase(lens, 2, 4, 4, 2, seed=12, chunk=S)
    R.build_tree(c.p, c.tree)
    kn_all, vn_all, q_all = c.inp["k_new"], c.inp["v_new"], c.inp["q"]
    kb, vb = bits(c.k_tok).copy(), bits(c.v_tok).copy()
    cur = list(lens)
    for st in range(S):
        kn, vn, q = (x[:, st:st + 1].contiguous() for x in (kn_all, vn_all, q_all))
        R.append(c.p, c.tree, kn.cuda(), vn.cuda())
        for s in range(c.B):  # the oracle's caches: the token at the sequence's own end
            kb[s, :, cur[s]] = bits(kn)[s, 0]
            vb[s, :, cur[s]] = bits(vn)[s, 0]
            cur[s] += 1
        assert c.tree.length == max(lens) + st + 1
        assert c.seq_len.cpu().tolist() == cur
        out, sel, ent = c.decode(q)
        qb = bits(q)
        stats = Stats()
        for s in range(c.B):
            for h in range(c.hkv):
                t = c.oracle_tree(s, h, cur[s], kb, vb)
                check_tile(stats, O.bf16_bits_to_f64(qb[s, 0, h * 4:(h + 1) * 4]), t, cur[s], c.k, False,
                           out[s, 0, h * 4:(h + 1) * 4].numpy(), gpu_selection(sel, s * c.hkv + h, t.top),
                           ent[s * c.hkv + h])
        stats.assert_ok()
    # the appended trees equal a fresh build over the same per-sequence lengths, bit for bit
    fresh_len = c.seq_len.clone()
    f = R.RecsaTree(c.p, c.k_tok.clone(), c.v_tok.clone(), c.inp["pooler"].cuda().contiguous(), c.tree.length,
                    seq_len=fresh_len)
    R.build_tree(c.p, f)
    torch.cuda.synchronize()
    for s in range(c.B):
        counts = O.level_counts(cur[s], 4)
        for lvl in range(1, len(counts)):
            for a, b in zip(c.tree.level_rows(lvl), f.level_rows(lvl)):
                assert np.array_equal(bits(a)[s, :, :counts[lvl]], bits(b)[s, :, :counts[lvl]]), (s, lvl)


@pytest.mark.parametrize("C", [20, 200])  # 200: several nodes a level in the one-launch update
def test_varlen_prefill_chunk_matches_oracle(C):
    lens = [300, 0, 77, 1000]
    c = VarCase(lens, 2, 4, 4, 2, seed=21 + C, chunk=C)
    R.build_tree(c.p, c.tree)
    kn, vn, q = (c.inp[x].cuda().contiguous() for x in ("k_new", "v_new", "q"))
    out = torch.empty(c.B, C, 8, 128, dtype=torch.float32, device="cuda")
    tiles = c.B * c.hkv * C
    lv = c.tree.levels
    sel = torch.full((tiles, lv, c.k), -7, dtype=torch.int32, device="cuda")
    ent = torch.zeros(tiles, 2, dtype=torch.int32, device="cuda")
    R.prefill_chunk(c.p, c.tree, kn, vn, q, out, c.ws, sel_idx=sel, sel_levels=lv, entries=ent)
    R.check_device_errors(c.ws)
    assert c.seq_len.cpu().tolist() == [n + C for n in lens]
    assert c.tree.length == max(lens) + C
    out, sel, ent = out.cpu(), sel.cpu().numpy(), ent.cpu().numpy()
    kb, vb = bits(c.inp["k_tok"]).copy(), bits(c.inp["v_tok"]).copy()
    qb = bits(q)
    stats = Stats()
    for s, n in enumerate(lens):
        kb[s, :, n:n + C] = bits(kn)[s].transpose(1, 0, 2)
        vb[s, :, n:n + C] = bits(vn)[s].transpose(1, 0, 2)
        for h in range(c.hkv):
            t = c.oracle_tree(s, h, n + C, kb, vb)
            for i in range(C):
                tile = (s * c.hkv + h) * C + i
                top = len(O.level_counts(n + i, c.b)) - 1 if n + i else 0
                check_tile(stats, O.bf16_bits_to_f64(qb[s, i, h * 4:(h + 1) * 4]), t, n + i, c.k, True,
                           out[s, i, h * 4:(h + 1) * 4].numpy(), gpu_selection(sel, tile, top), ent[tile])
    stats.assert_ok()


def test_out_of_range_length_is_flagged():
    c = VarCase([500, 300], 1, 4, 4, 2, seed=4)
    R.build_tree(c.p, c.tree)
    c.seq_len[1] = 900  # above the tree's longest length
    out = torch.empty(2, 1, 4, 128, dtype=torch.float32, device="cuda")
    R.decode(c.p, c.tree, c.inp["q"].cuda().contiguous(), out, c.ws)
    with pytest.raises(R.RecsaError):
        R.check_device_errors(c.ws)
    # the context stays usable and the error word was cleared
    c.seq_len[1] = 300
    R.decode(c.p, c.tree, c.inp["q"].cuda().contiguous(), out, c.ws)
    R.check_device_errors(c.ws)


@pytest.mark.parametrize("G,b,k,kernel,cluster_size", [
    (1, 3, 2, 0, 0), (2, 16, 8, 3, 2), (8, 16, 8, 3, 4), (8, 4, 2, 1, 2), (2, 3, 3, 2, 0),
])
def test_varlen_decode_other_group_sizes(G, b, k, kernel, cluster_size):
    lens = [900, 0, 1, 333]
    c = VarCase(lens, 2, G, b, k, seed=G * 10 + b)
    R.build_tree(c.p, c.tree)
    out, sel, ent = c.decode(c.inp["q"], kernel, cluster_size)
    c.check_decode(c.inp["q"], out, sel, ent, lens)
