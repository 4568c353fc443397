"""KV-head sharding of the library, run shard by shard on one GPU.

A (sequence, KV head) tree and the tiles of that KV group read nothing else, so a batch
can be split into blocks of KV heads, each block run through the library as a smaller
model (Hkv' heads, G * Hkv' query heads), and the blocks' outputs joined along the
head axis (``sharding.py``).  Here the 8 KV heads of a batch are split 3 + 3 + 2, as
three ranks would hold them; each block is built, decoded and prefilled in turn on one
device.  The joined outputs must be bit-identical to the unsharded calls in the same
launch shape, and the sampled tiles must meet the oracle bar.
"""

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_build_b200 as R
from hierarchical_sparse_attention_build_b200 import sharding as S
import recsa_inputs as I
from oracle import recsa_oracle as O
from parity_helpers import Stats, bits, check_tile, gpu_selection

pytestmark = pytest.mark.gpu

B, HKV, G, L, C, Q, BR, K = 2, 8, 4, 5000, 24, 2, 16, 8
WORLD = 3


def _inputs():
    return I.random_case(B, L, HKV, HKV * G, Q, seed=4242, capacity=L + C, chunk=C), \
        I.random_case(B, L, HKV, HKV * G, Q, seed=4243)["q"]


def _run(p, k_tok, v_tok, pooler, q_dec, k_new, v_new, q_pre, dec_shape, pre_shape):
    """Build, decode (queries at L), then append the chunk and attend it causally."""
    dev = "cuda"
    tree = R.RecsaTree(p, k_tok.to(dev).contiguous(), v_tok.to(dev).contiguous(), pooler.to(dev), L)
    ws = R.Workspace(p, tree.capacity, dev)
    R.build_tree(p, tree)
    tiles = B * p.num_kv_heads * Q
    dec = torch.empty(B, Q, p.num_q_heads, 128, dtype=torch.float32, device=dev)
    sel = torch.full((tiles, tree.levels, K), -7, dtype=torch.int32, device=dev)
    R.decode(p, tree, q_dec.to(dev).contiguous(), dec, ws, sel_idx=sel, sel_levels=tree.levels,
             kernel=dec_shape[0], cluster_size=dec_shape[1])
    pre = torch.empty(B, C, p.num_q_heads, 128, dtype=torch.float32, device=dev)
    R.prefill_chunk(p, tree, k_new.to(dev).contiguous(), v_new.to(dev).contiguous(), q_pre.to(dev).contiguous(),
                    pre, ws, kernel=pre_shape[0], cluster_size=pre_shape[1])
    R.check_device_errors(ws)
    torch.cuda.synchronize()
    return dec.cpu(), sel.cpu().numpy(), pre.cpu()


@pytest.mark.parametrize("dec_shape,pre_shape", [((3, 4), (2, 0)), ((2, 0), (1, 1))])
def test_head_shards_join_to_the_unsharded_calls(dec_shape, pre_shape):
    inp, q_dec = _inputs()
    p = R.params(num_kv_heads=HKV, num_q_heads=HKV * G, branching=BR, top_k=K)
    full_dec, full_sel, full_pre = _run(p, inp["k_tok"], inp["v_tok"], inp["pooler"], q_dec, inp["k_new"],
                                        inp["v_new"], inp["q"], dec_shape, pre_shape)
    dec_parts, pre_parts, sel_parts = [], [], []
    ranges = [S.kv_head_range(HKV, r, WORLD) for r in range(WORLD)]
    assert [h1 - h0 for h0, h1 in ranges] == [3, 3, 2]
    for r, (h0, h1) in enumerate(ranges):
        ps = S.shard_params(p, r, WORLD)
        d, sl, pr = _run(ps, S.shard_cache(inp["k_tok"], h0, h1), S.shard_cache(inp["v_tok"], h0, h1),
                         inp["pooler"], S.shard_queries(q_dec, G, h0, h1), S.shard_tokens(inp["k_new"], h0, h1),
                         S.shard_tokens(inp["v_new"], h0, h1), S.shard_queries(inp["q"], G, h0, h1),
                         dec_shape, pre_shape)
        dec_parts.append(d)
        pre_parts.append(pr)
        sel_parts.append(sl.reshape(B, h1 - h0, Q, *sl.shape[1:]))
    assert torch.equal(torch.cat(dec_parts, dim=2), full_dec)
    assert torch.equal(torch.cat(pre_parts, dim=2), full_pre)
    assert np.array_equal(np.concatenate(sel_parts, axis=1).reshape(full_sel.shape), full_sel)

    # the joined decode against the oracle, every tile of sequence 0 and head 0..7 of sequence 1 at query 0
    kb, vb, qb = bits(inp["k_tok"]), bits(inp["v_tok"]), bits(q_dec)
    W = inp["pooler"].double().numpy()
    st = Stats()
    for s in range(B):
        for h in range(HKV):
            t = O.build_tree(O.bf16_bits_to_f64(kb[s, h, :L]), O.bf16_bits_to_f64(vb[s, h, :L]), W, BR)
            for qi in (range(Q) if s == 0 else (0,)):
                tile = (s * HKV + h) * Q + qi
                check_tile(st, O.bf16_bits_to_f64(qb[s, qi, h * G:(h + 1) * G]), t, L, K, False,
                           full_dec[s, qi, h * G:(h + 1) * G].numpy(), gpu_selection(full_sel, tile, t.top))
    st.assert_ok()
    # the joined prefill: first and last query of the chunk, every head of sequence 1
    kc, vc = O.append_chunk(kb, vb, bits(inp["k_new"]), bits(inp["v_new"]), L)
    qp = bits(inp["q"])
    sp = Stats()
    for h in range(HKV):
        t = O.build_tree(O.bf16_bits_to_f64(kc[1, h]), O.bf16_bits_to_f64(vc[1, h]), W, BR)
        for i in (0, C - 1):
            check_tile(sp, O.bf16_bits_to_f64(qp[1, i, h * G:(h + 1) * G]), t, L + i, K, True,
                       full_pre[1, i, h * G:(h + 1) * G].numpy(), None)
    sp.assert_ok()
