"""recsa_decode_no_alloc: decode for callers that cannot allocate device memory.

Such callers (a host that owns every device allocation and gives the library a fixed
budget, a serving loop that forbids allocation after warm-up) cannot provide the
workspace recsa_decode takes; this entry point keeps that scratch in a fixed device
array of the library.  It runs the same kernel as recsa_decode with a RoPE table
computed the same way, so its output must be bit-identical to recsa_decode's on the
same inputs, call after call.  The two cases use different RoPE bases, so a call that
ran with the previous call's table left in the shared array would differ.  The file
name makes pytest collect it last.
"""

import ctypes

import pytest
import torch

import hierarchical_sparse_attention_build_b200 as R
import recsa_inputs as I

pytestmark = pytest.mark.gpu

def _no_alloc(p, tree, q, out):
    lib = R.raw_library()
    return lib.recsa_decode_no_alloc(ctypes.byref(p), ctypes.byref(tree.c), ctypes.c_void_p(q.data_ptr()),
                                     q.shape[1], ctypes.c_void_p(out.data_ptr()),
                                     int(out.dtype == torch.float32),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_no_alloc_decode_matches_decode_on_two_calls():
    cases = []
    for seed, (L, b, k, hkv, G, Q, base) in enumerate([(4096, 8, 4, 1, 4, 16, 1.0e6), (3000, 16, 8, 2, 4, 3, 1.0e4)]):
        inp = I.random_case(1, L, hkv, hkv * G, Q, seed=900 + seed)
        p = R.params(num_kv_heads=hkv, num_q_heads=hkv * G, branching=b, top_k=k, rope_base=base)
        dev = "cuda"
        tree = R.RecsaTree(p, inp["k_tok"].to(dev), inp["v_tok"].to(dev), inp["pooler"].to(dev), L)
        R.build_tree(p, tree)
        q = inp["q"].to(dev)
        ws = R.Workspace(p, tree.capacity, dev)
        ref = torch.empty(q.shape, dtype=torch.float32, device=dev)
        R.decode(p, tree, q, ref, ws)
        cases.append((p, tree, q, ref))
    # two calls in a row per case, alternating cases so each call overwrites the other's table
    for rnd in range(2):
        for p, tree, q, ref in cases:
            out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
            assert _no_alloc(p, tree, q, out) == 0, R.last_error()
            torch.cuda.synchronize()
            assert torch.equal(out, ref), (rnd, (out - ref).abs().max().item())


def test_no_alloc_rejects_scratch_beyond_its_maximum():
    L = 4096
    inp = I.random_case(1, L, 1, 4, 1, seed=5)
    p = R.params(num_kv_heads=1, num_q_heads=4, branching=8, top_k=R.TOPK_ALL)  # positions up to 4096
    tree = R.RecsaTree(p, inp["k_tok"].cuda(), inp["v_tok"].cuda(), inp["pooler"].cuda(), L)
    out = torch.empty(inp["q"].shape, dtype=torch.float32, device="cuda")
    rc = _no_alloc(p, tree, inp["q"].cuda(), out)
    assert rc == 2 and "fixed scratch" in R.last_error()
