"""The lean attend kernel's own source, run on host threads against the oracle (no GPU).

tests/host_emulation cuts the kernel out of the attend source unchanged and compiles it
with g++ against host versions of the CUDA features it uses: one std::thread per CUDA
thread, one cluster of CS x 256 threads per tile, real rendezvous for block and cluster
barriers and for every warp collective, and AddressSanitizer.  A barrier or collective
that some thread never reaches is reported with the place every thread waits (a stall
on the GPU); an out-of-bounds access aborts.  The results are then held to the same bar
as the GPU parity tests: kept node sets, entry counts and outputs against the oracle, on
trees the oracle builds and the library's arena layout holds.
"""

import math
import os
import shutil
import subprocess
import sys

import numpy as np
import pytest

import hierarchical_sparse_attention_build_b200 as R
import recsa_inputs as I
from oracle import recsa_oracle as O
from parity_helpers import Stats, bits, check_tile, gpu_selection

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
EMU = os.path.join(HERE, "host_emulation")
CSRC = os.path.join(ROOT, "hierarchical_sparse_attention_build_b200", "csrc")
sys.path.insert(0, EMU)
from extract import extract_lean  # noqa: E402


@pytest.fixture(scope="module")
def emu_bin(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("lean_emu")
    extract_lean(os.path.join(CSRC, "recsa_attend.cu"), str(d / "lean_extracted.h"))
    exe = str(d / "emu_lean")
    cmd = ["g++", "-std=c++20", "-O1", "-g", "-fsanitize=address,undefined", "-pthread",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-I", EMU, "-I", str(d),
           os.path.join(EMU, "emu_main.cpp"), "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-4000:]
    return exe


def _rph(G, CS, max_cand):
    # the launcher's choice of rows per half-warp
    if CS == 4 and max_cand <= 128:
        return 2
    if G <= 4 and CS == 4 and max_cand <= 192:
        return 3
    if G <= 4 and CS == 2 and max_cand <= 128:
        return 4
    raise ValueError("no lean shape")


def _run(emu_bin, tmp_path, B, hkv, G, L, b, k, Q, CS, causal=False, seed=1, lens=None, zero_keys=False):
    """Lay out the oracle's bf16 tree, run the kernel on host threads, check every tile.
    lens: per-sequence lengths (decode; L is then their maximum).  zero_keys: every key
    is zero, so every score ties at 0 and each level keeps its lowest positions."""
    C = Q if causal else 0
    cap = L + C
    inp = I.random_case(B, L, hkv, hkv * G, Q, seed=seed, capacity=cap, chunk=C)
    if zero_keys:
        inp["k_tok"].zero_()
        if C:
            inp["k_new"].zero_()
    kb, vb = bits(inp["k_tok"]), bits(inp["v_tok"])
    if causal:
        kb, vb = O.append_chunk(kb, vb, bits(inp["k_new"]), bits(inp["v_new"]), L)
        length_tree = L + C
    else:
        kb, vb = kb[:, :, :cap], vb[:, :, :cap]
        length_tree = L
    pooler = inp["pooler"].double().numpy()
    if lens is None:
        trees = O.build_all(kb, vb, pooler, b, length_tree)
    else:
        trees = [[O.build_tree(O.bf16_bits_to_f64(kb[s, h, :n]), O.bf16_bits_to_f64(vb[s, h, :n]), pooler, b)
                  if n else None for h in range(hkv)] for s, n in enumerate(lens)]

    p = R.params(num_kv_heads=hkv, num_q_heads=hkv * G, branching=b, top_k=k)
    node_rows, levels, offs = R.tree_layout(p, B, cap)
    slots = [cap] + [math.ceil(cap / b ** lv) for lv in range(1, levels + 1)]
    knode = np.zeros((max(node_rows, 1), 128), np.uint16)
    vnode = np.zeros_like(knode)
    for s in range(B):
        for h in range(hkv):
            t = trees[s][h]
            for lv in range(1, t.top + 1 if t is not None else 1):
                n = t.keys[lv].shape[0]
                r0 = offs[lv] + (s * hkv + h) * slots[lv]
                knode[r0:r0 + n] = O.f64_to_bf16_bits(t.keys[lv])
                vnode[r0:r0 + n] = O.f64_to_bf16_bits(t.values[lv])
    ktok = np.zeros((B, hkv, cap, 128), np.uint16)
    vtok = np.zeros_like(ktok)
    ktok[:, :, :kb.shape[2]] = kb
    vtok[:, :, :vb.shape[2]] = vb

    mc = max(b, min((k + (1 if causal else 0)) * b, length_tree))
    max_cand = (mc + 31) // 32 * 32
    table_rows = min(max(b, min((k + 1) * b, cap)), 4096) + 1
    tiles = B * hkv * Q
    sel_levels = max(levels, 1)
    prm = dict(G=G, CS=CS, RPH=_rph(G, CS, max_cand), table_rows=table_rows, rope_base=1.0e6, tiles=tiles,
               top_k=k, sel_levels=sel_levels, cap=cap, length=L if causal else length_tree, b=b, levels=levels,
               hkv=hkv, nq=Q, causal=int(causal), table_rows_needed=mc + 1, max_cand=max_cand,
               scale=1.0 / math.sqrt(128.0))
    d = tmp_path / f"case_{B}_{hkv}_{G}_{L}_{b}_{k}_{Q}_{CS}_{int(causal)}_{int(lens is not None)}"
    d.mkdir()
    with open(d / "params.txt", "w") as f:
        for key, val in prm.items():
            f.write(f"{key} {val!r}\n")
        f.write("row_off " + " ".join(str(offs[i] if i <= levels else 0) for i in range(R.MAX_LEVELS + 1)) + "\n")
        f.write("slots " + " ".join(str(slots[i] if i <= levels else 0) for i in range(R.MAX_LEVELS + 1)) + "\n")
        if lens is not None:
            f.write("seq_len " + " ".join(str(n) for n in lens) + "\n")
    for name, arr in (("k_tok", ktok), ("v_tok", vtok), ("k_node", knode), ("v_node", vnode), ("q", bits(inp["q"]))):
        np.ascontiguousarray(arr, dtype=np.uint16).tofile(d / f"{name}.bin")
    r = subprocess.run([emu_bin, str(d)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    assert int(open(d / "err.txt").read()) == 0
    out = np.fromfile(d / "out.bin", np.float32).reshape(B, Q, hkv * G, 128)
    sel = np.fromfile(d / "sel.bin", np.int32).reshape(tiles, sel_levels, min(max(k, 1), 64))
    ent = np.fromfile(d / "entries.bin", np.int32).reshape(tiles, 2)

    qb = bits(inp["q"])
    stats = Stats()
    for s in range(B):
        for h in range(hkv):
            for qi in range(Q):
                tile = (s * hkv + h) * Q + qi
                pos = L + qi if causal else (L if lens is None else lens[s])
                if pos == 0:  # nothing visible: zeros
                    assert not out[s, qi, h * G:(h + 1) * G].any()
                    continue
                top = len(O.level_counts(pos, b)) - 1
                gsel = gpu_selection(sel, tile, top) if 1 <= k <= 64 else None
                check_tile(stats, O.bf16_bits_to_f64(qb[s, qi, h * G:(h + 1) * G]), trees[s][h], pos, k, causal,
                           out[s, qi, h * G:(h + 1) * G], gsel, ent[tile])
    stats.assert_ok()
    return stats


@pytest.mark.parametrize("CS", [2, 4])
def test_two_candidates_over_a_cluster(emu_bin, tmp_path, CS):
    # one top-level row per CTA, in half-warp 0 only: every lane must still join the
    # warp collectives of the score step
    _run(emu_bin, tmp_path, 1, 1, 2, 17, 16, 8, 2, CS)


@pytest.mark.parametrize("B,hkv,G,L,b,k,Q,CS", [
    (1, 1, 4, 1000, 4, 3, 3, 4),    # ragged tails, 6 levels
    (1, 2, 1, 700, 3, 2, 2, 2),     # b = 3, G = 1
    (1, 1, 8, 300, 16, 8, 1, 4),    # G = 8 (the only G = 8 shape)
    (1, 1, 4, 700, 8, 0, 2, 4),     # k = 0: the top-level summaries alone
    (2, 1, 4, 4096, 16, 8, 1, 4),   # the 1M tree's per-level shape: 16 -> 128 -> 128 candidates
    (1, 1, 4, 150, 4, R.TOPK_ALL, 2, 4),  # k = all: every candidate kept, up to 150 a level
])
def test_decode_matches_oracle(emu_bin, tmp_path, B, hkv, G, L, b, k, Q, CS):
    _run(emu_bin, tmp_path, B, hkv, G, L, b, k, Q, CS)


@pytest.mark.parametrize("CS", [2, 4])
def test_causal_prefill_matches_oracle(emu_bin, tmp_path, CS):
    _run(emu_bin, tmp_path, 1, 1, 4, 200, 4, 2, 6, CS, causal=True)


def test_causal_levels_past_128_candidates(emu_bin, tmp_path):
    # b = 16, k = 8, causal: up to 144 candidates a level, 3 rows per half-warp, and the
    # ranking by the generic count
    _run(emu_bin, tmp_path, 1, 1, 4, 3000, 16, 8, 6, 4, causal=True, seed=5)


@pytest.mark.parametrize("CS", [2, 4])
def test_decode_with_per_sequence_lengths(emu_bin, tmp_path, CS):
    # an empty sequence, a single token, a shallow tree and the deepest one in one launch
    _run(emu_bin, tmp_path, 4, 1, 4, 1000, 4, 2, 1, CS, lens=[0, 1, 37, 1000], seed=6)


@pytest.mark.parametrize("k", [3, 8])
def test_all_scores_tied_keep_the_lowest_positions(emu_bin, tmp_path, k):
    # zero keys: every group score is exactly 0, so selection is decided by position alone
    st = _run(emu_bin, tmp_path, 1, 1, 4, 2000, 8, k, 2, 4, zero_keys=True, seed=7)
    assert st.near_ties == 0
