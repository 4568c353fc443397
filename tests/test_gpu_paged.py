"""GPU checks of the paged token cache (recsa_tree.page_table).

A paged cache holds the same tokens as a contiguous one, in pages of a pool placed by a
shuffled page table (with unused pages in between).  Every call reads the same rows either
way, so build, decode in every launch shape, prefill (both update paths), the append loop
and per-sequence lengths must give the contiguous path's bits exactly; the contiguous path
is itself held to the oracle, and one decode here is checked against the oracle directly.
A table entry outside the pool is flagged and never dereferenced.
"""

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_build_b200 as R
import recsa_inputs as I
from oracle import recsa_oracle as O
from parity_helpers import Stats, bits, check_tile, gpu_selection

pytestmark = pytest.mark.gpu

SHAPES = [(0, 0), (1, 1), (1, 4), (2, 0), (3, 2), (3, 4)]


def _params(hkv, G, b, k):
    return R.params(num_kv_heads=hkv, num_q_heads=hkv * G, branching=b, top_k=k)


def paginate(k_tok, v_tok, P, seed, spare=3):
    """Contiguous caches [B][Hkv][cap][128] -> pools [num_pages][Hkv][P][128] and a shuffled
    int32 page table [B][cap / P]; `spare` unused pages hold noise."""
    B, H, cap, D = k_tok.shape
    pps = cap // P
    n = B * pps + spare
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n, generator=g)[:B * pps].to(torch.int32)
    table = perm.view(B, pps).contiguous()
    pools = []
    for x in (k_tok, v_tok):
        pool = torch.randn(n, H, P, D, generator=g).to(torch.bfloat16)
        src = x.cpu().view(B, H, pps, P, D).permute(0, 2, 1, 3, 4).reshape(B * pps, H, P, D)
        pool[perm.long()] = src
        pools.append(pool.cuda().contiguous())
    return pools[0], pools[1], table.cuda()


def unpaginate(pool, table, cap):
    B, pps = table.shape
    _, H, P, D = pool.shape
    rows = pool.cpu()[table.cpu().long().view(-1)]  # [B * pps][H][P][D]
    return rows.view(B, pps, H, P, D).permute(0, 2, 1, 3, 4).reshape(B, H, cap, D)


class Pair:
    """The same caches as a contiguous tree and as a paged one."""

    def __init__(self, B, hkv, G, L, b, k, P, seed, chunk=0, queries=1, lens=None):
        cap = L + chunk
        cap = -(-cap // P) * P
        self.inp = I.random_case(B, L, hkv, hkv * G, queries, seed=seed, capacity=cap, chunk=chunk)
        self.p = _params(hkv, G, b, k)
        pooler = self.inp["pooler"].cuda().contiguous()
        kc, vc = self.inp["k_tok"].cuda().contiguous(), self.inp["v_tok"].cuda().contiguous()
        kp, vp, table = paginate(kc, vc, P, seed + 1)
        self.sl = [torch.tensor(lens, dtype=torch.int64, device="cuda") if lens else None for _ in range(2)]
        self.c = R.RecsaTree(self.p, kc, vc, pooler, L, seq_len=self.sl[0])
        self.g = R.RecsaTree(self.p, kp, vp, pooler, L, seq_len=self.sl[1], page_table=table)
        assert self.g.capacity == self.c.capacity == cap
        self.ws = R.Workspace(self.p, cap, "cuda")
        self.cap, self.P, self.table = cap, P, table

    def build(self):
        R.build_tree(self.p, self.c)
        R.build_tree(self.p, self.g)

    def assert_same_trees(self):
        torch.cuda.synchronize()
        assert self.c.length == self.g.length
        for lvl in range(1, self.c.levels + 1):
            for a, b in zip(self.c.level_rows(lvl), self.g.level_rows(lvl)):
                n = -(-self.c.length // self.p.branching ** lvl)
                assert np.array_equal(bits(a)[:, :, :n], bits(b)[:, :, :n]), lvl
        L = self.c.length
        for cont, pool in ((self.c.k_tok, self.g.k_tok), (self.c.v_tok, self.g.v_tok)):
            assert np.array_equal(bits(cont)[:, :, :L], bits(unpaginate(pool, self.table, self.cap))[:, :, :L])

    def decode_both(self, q, kernel=0, cluster_size=0):
        outs = []
        for t in (self.c, self.g):
            out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
            R.decode(self.p, t, q.cuda().contiguous(), out, self.ws, kernel=kernel, cluster_size=cluster_size)
            R.check_device_errors(self.ws)
            outs.append(out.cpu())
        return outs


@pytest.mark.parametrize("P", [1, 4, 16, 64])
@pytest.mark.parametrize("kernel,cluster_size", SHAPES)
def test_paged_build_and_decode_equal_contiguous(P, kernel, cluster_size):
    x = Pair(2, 2, 4, 1000, 4, 2, P, seed=P + kernel, queries=3)
    x.build()
    x.assert_same_trees()
    a, b = x.decode_both(x.inp["q"], kernel, cluster_size)
    assert torch.equal(a, b)


@pytest.mark.parametrize("P,C", [(16, 40), (8, 300), (1, 5)])
def test_paged_prefill_equals_contiguous(P, C):
    # C = 40: the one-launch path update; C = 300: the copy + per-level launches
    x = Pair(2, 2, 4, 700, 4, 2, P, seed=C, chunk=C)
    x.build()
    outs = []
    for t in (x.c, x.g):
        out = torch.empty(x.inp["q"].shape, dtype=torch.float32, device="cuda")
        R.prefill_chunk(x.p, t, x.inp["k_new"].cuda().contiguous(), x.inp["v_new"].cuda().contiguous(),
                        x.inp["q"].cuda().contiguous(), out, x.ws)
        R.check_device_errors(x.ws)
        outs.append(out.cpu())
    assert torch.equal(outs[0], outs[1])
    x.assert_same_trees()


def test_paged_append_loop_with_per_sequence_lengths_equals_contiguous():
    lens = [700, 1021, 3]
    S = 5
    x = Pair(3, 2, 4, 1021, 4, 2, 16, seed=5, chunk=S, lens=lens)
    x.build()
    for st in range(S):
        kn, vn, q = (x.inp[n][:, st:st + 1].cuda().contiguous() for n in ("k_new", "v_new", "q"))
        for t in (x.c, x.g):
            R.append(x.p, t, kn, vn)
        a, b = x.decode_both(q)
        assert torch.equal(a, b)
    assert x.sl[0].tolist() == x.sl[1].tolist() == [n + S for n in lens]
    torch.cuda.synchronize()
    for lvl in range(1, x.c.levels + 1):
        for a, b in zip(x.c.level_rows(lvl), x.g.level_rows(lvl)):
            for s, n in enumerate(x.sl[0].tolist()):
                if lvl >= len(O.level_counts(n, 4)):
                    continue  # not a level of this sequence's tree
                m = O.level_counts(n, 4)[lvl]
                assert np.array_equal(bits(a)[s, :, :m], bits(b)[s, :, :m]), (lvl, s)


def test_paged_decode_matches_oracle():
    x = Pair(1, 2, 4, 1500, 4, 2, 32, seed=77, queries=2)
    x.build()
    _, out = x.decode_both(x.inp["q"], kernel=3, cluster_size=4)
    q = bits(x.inp["q"])
    kb, vb = bits(x.inp["k_tok"]), bits(x.inp["v_tok"])
    pooler = x.inp["pooler"].double().numpy()
    stats = Stats()
    for h in range(2):
        t = O.build_tree(O.bf16_bits_to_f64(kb[0, h, :1500]), O.bf16_bits_to_f64(vb[0, h, :1500]), pooler, 4)
        for qi in range(2):
            check_tile(stats, O.bf16_bits_to_f64(q[0, qi, h * 4:(h + 1) * 4]), t, 1500, 2, False,
                       out[0, qi, h * 4:(h + 1) * 4].numpy(), None)
    stats.assert_ok()


def test_page_outside_the_pool_is_flagged():
    x = Pair(1, 1, 4, 64, 4, R.TOPK_ALL, 8, seed=9)  # every token is read at the last level
    x.build()
    x.table[0, 3] = 10_000  # no such page
    out = torch.empty(x.inp["q"].shape, dtype=torch.float32, device="cuda")
    for kernel, cs in ((3, 4), (1, 1), (2, 0)):
        R.decode(x.p, x.g, x.inp["q"].cuda().contiguous(), out, x.ws, kernel=kernel, cluster_size=cs)
        with pytest.raises(R.RecsaError):
            R.check_device_errors(x.ws)
    R.build_tree(x.p, x.g)  # skips the page's rows; nothing to flag without a workspace
    torch.cuda.synchronize()


@pytest.mark.parametrize("G,b,P,kernel,cluster_size", [
    (8, 16, 16, 3, 4), (1, 3, 4, 1, 1), (2, 16, 32, 2, 0), (8, 4, 8, 1, 4),
])
def test_paged_other_group_sizes_equal_contiguous(G, b, P, kernel, cluster_size):
    x = Pair(2, 2, G, 900, b, 4, P, seed=G + b + P, queries=2)
    x.build()
    x.assert_same_trees()
    a, c = x.decode_both(x.inp["q"], kernel, cluster_size)
    assert torch.equal(a, c)


@pytest.mark.parametrize("pinned", [True, False])
def test_host_buffer_and_no_alloc_decode_over_paged_varlen_cache(pinned):
    """recsa_decode_host and recsa_decode_no_alloc over a paged cache with per-sequence lengths
    give recsa_decode's bits."""
    x = Pair(3, 2, 4, 800, 4, 2, 16, seed=31, queries=2, lens=[800, 5, 333])
    x.build()
    q = x.inp["q"].cuda().contiguous()
    want = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    R.decode(x.p, x.g, q, want, x.ws)
    R.check_device_errors(x.ws)
    q_host = x.inp["q"].contiguous()
    out_host = torch.empty(q.shape, dtype=torch.float32)
    if pinned:
        q_host, out_host = q_host.pin_memory(), out_host.pin_memory()
    q_dev, out_dev = torch.empty_like(q), torch.empty_like(want)
    R.decode_host(x.p, x.g, q_host, out_host, q_dev, out_dev, x.ws)
    torch.cuda.synchronize()
    R.check_device_errors(x.ws)
    assert torch.equal(out_host, want.cpu())
    got = torch.empty_like(want)
    R.decode_no_alloc(x.p, x.g, q, got)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
