"""GPU checks of recsa_decode_step (append + decode of one token per sequence, lengths on the
device, every kernel parameter from the capacity).

A step gives the bits of recsa_append followed by recsa_decode, called on the same tree; the
step captured once into a CUDA graph and replayed gives them too, step after step, with the
device lengths advancing; a sequence without room is skipped and flagged; and the decoded
tokens are held to the oracle.
"""

import numpy as np
import pytest
import torch

import hierarchical_sparse_attention_build_b200 as R
import recsa_inputs as I
from oracle import recsa_oracle as O
from parity_helpers import Stats, bits, check_tile

pytestmark = pytest.mark.gpu


def _trees(lens, hkv, G, b, k, S, seed, extra=0):
    """Two trees over the same caches with per-sequence lengths: one for the steps, one for
    the reference calls."""
    B, L = len(lens), max(lens)
    cap = L + S + extra
    inp = I.random_case(B, L, hkv, hkv * G, 0, seed=seed, capacity=cap, chunk=S)
    p = R.params(num_kv_heads=hkv, num_q_heads=hkv * G, branching=b, top_k=k)
    pooler = inp["pooler"].cuda().contiguous()
    out = []
    for _ in range(2):
        kc, vc = inp["k_tok"].cuda().contiguous(), inp["v_tok"].cuda().contiguous()
        sl = torch.tensor(lens, dtype=torch.int64, device="cuda")
        t = R.RecsaTree(p, kc, vc, pooler, L, seq_len=sl)
        R.build_tree(p, t)
        out.append(t)
    ws = [R.Workspace(p, cap, "cuda") for _ in range(2)]
    return inp, p, out, ws


def _reference_step(p, tree, ws, kn, vn, qn):
    R.append(p, tree, kn, vn)
    o = torch.empty(qn.shape, dtype=torch.float32, device="cuda")
    R.decode(p, tree, qn, o, ws)
    R.check_device_errors(ws)
    return o


def test_decode_step_equals_append_then_decode_and_the_oracle():
    lens, S = [700, 1021, 40, 333], 4
    inp, p, (ts, tr), (ws_s, ws_r) = _trees(lens, 2, 4, 4, 2, S, seed=3)
    kb, vb = bits(inp["k_tok"]).copy(), bits(inp["v_tok"]).copy()
    pooler = inp["pooler"].double().numpy()
    cur = list(lens)
    for st in range(S):
        kn, vn, qn = (inp[x][:, st:st + 1].cuda().contiguous() for x in ("k_new", "v_new", "q"))
        o = torch.empty(qn.shape, dtype=torch.float32, device="cuda")
        R.decode_step(p, ts, kn, vn, qn, o, ws_s)
        R.check_device_errors(ws_s)
        want = _reference_step(p, tr, ws_r, kn, vn, qn)
        assert torch.equal(o, want)
        for s in range(len(lens)):
            kb[s, :, cur[s]] = bits(kn)[s, 0]
            vb[s, :, cur[s]] = bits(vn)[s, 0]
            cur[s] += 1
        assert ts.seq_len.tolist() == cur == tr.seq_len.tolist()
    # the last step's tokens against the oracle
    qb, on = bits(qn), o.cpu().numpy()
    stats = Stats()
    for s in range(len(lens)):
        for h in range(2):
            t = O.build_tree(O.bf16_bits_to_f64(kb[s, h, :cur[s]]), O.bf16_bits_to_f64(vb[s, h, :cur[s]]), pooler, 4)
            check_tile(stats, O.bf16_bits_to_f64(qb[s, 0, h * 4:(h + 1) * 4]), t, cur[s], 2, False,
                       on[s, 0, h * 4:(h + 1) * 4], None)
    stats.assert_ok()


def test_decode_step_replayed_from_a_cuda_graph():
    lens, S = [900, 64, 1020], 6
    inp, p, (ts, tr), (ws_s, ws_r) = _trees(lens, 2, 4, 4, 2, S + 1, seed=7)
    B = len(lens)
    kbuf = torch.empty(B, 1, 2, 128, dtype=torch.bfloat16, device="cuda")
    vbuf, qbuf = torch.empty_like(kbuf), torch.empty(B, 1, 8, 128, dtype=torch.bfloat16, device="cuda")
    obuf = torch.empty(B, 1, 8, 128, dtype=torch.float32, device="cuda")
    steps = [tuple(inp[x][:, st:st + 1].cuda().contiguous() for x in ("k_new", "v_new", "q")) for st in range(S + 1)]
    # one step outside the graph (first launches set kernel attributes), then capture the next
    for buf, src in zip((kbuf, vbuf, qbuf), steps[0]):
        buf.copy_(src)
    R.decode_step(p, ts, kbuf, vbuf, qbuf, obuf, ws_s)
    want = _reference_step(p, tr, ws_r, *steps[0])
    assert torch.equal(obuf, want)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=side):
        R.decode_step(p, ts, kbuf, vbuf, qbuf, obuf, ws_s)  # captured, not run
    torch.cuda.synchronize()
    for st in range(1, S + 1):
        for buf, src in zip((kbuf, vbuf, qbuf), steps[st]):
            buf.copy_(src)
        g.replay()
        want = _reference_step(p, tr, ws_r, *steps[st])
        torch.cuda.synchronize()
        assert torch.equal(obuf, want), st
    R.check_device_errors(ws_s)
    assert ts.seq_len.tolist() == [n + S + 1 for n in lens] == tr.seq_len.tolist()
    for lvl in range(1, ts.levels + 1):
        for a, b in zip(ts.level_rows(lvl), tr.level_rows(lvl)):
            for s, n in enumerate(ts.seq_len.tolist()):
                c = O.level_counts(n, 4)
                if lvl < len(c):
                    assert np.array_equal(bits(a)[s, :, :c[lvl]], bits(b)[s, :, :c[lvl]]), (lvl, s)
    del g


def test_a_full_sequence_is_skipped_and_flagged():
    lens = [50, 60]
    inp, p, (ts, _), (ws, _) = _trees(lens, 1, 4, 4, 2, 1, seed=11)  # capacity 61: sequence 1 is full after one more
    ts.seq_len[1] = ts.capacity
    kn, vn, qn = (inp[x][:, 0:1].cuda().contiguous() for x in ("k_new", "v_new", "q"))
    o = torch.empty(qn.shape, dtype=torch.float32, device="cuda")
    R.decode_step(p, ts, kn, vn, qn, o, ws)
    with pytest.raises(R.RecsaError):
        R.check_device_errors(ws)
    assert ts.seq_len.tolist() == [51, ts.capacity]
    R.decode_step(p, ts, kn, vn, qn, o, ws)  # sequence 0 goes on; the context stays usable
    assert ts.seq_len.tolist()[0] == 52
