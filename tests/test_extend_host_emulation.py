"""The append and level-build kernels' own source, run on host threads against the oracle (no GPU).

tests/host_emulation cuts the append kernel (one CTA per (sequence, KV head) that copies the
new tokens and rebuilds the nodes over them, level by level) out of the build source and
compiles it with g++ against host versions of the CUDA features it uses: one std::thread
per CUDA thread, real rendezvous for every __syncthreads, and AddressSanitizer.  The tree
before the append is the oracle's, laid out in the library's arena; after it, the token
slots must hold the new rows bit for bit and every node row must meet the node-row parity
bar against the oracle's tree over the longer cache — for equal lengths, per-sequence
lengths and a paged token cache.  The level-build kernel runs the same way over every level
(a grid that strides over the level's nodes, or a node per warp), its node rows held to the
oracle's trees, with per-sequence lengths and a paged cache too.  Both kernels also run with
a tensor-core product that never completes, to check that their bounded waits report the
timeout and return.
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
from parity_helpers import bits, check_node_rows

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
EMU = os.path.join(HERE, "host_emulation")
CSRC = os.path.join(ROOT, "hierarchical_sparse_attention_build_b200", "csrc")
sys.path.insert(0, EMU)
from extract import extract_extend  # noqa: E402


@pytest.fixture(scope="module")
def emu_bin(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("extend_emu")
    extract_extend(os.path.join(CSRC, "recsa_build.cu"), str(d / "extend_extracted.h"))
    exe = str(d / "emu_extend")
    cmd = ["g++", "-std=c++20", "-O1", "-g", "-fsanitize=address,undefined", "-pthread",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-I", EMU, "-I", str(d),
           os.path.join(EMU, "emu_extend.cpp"), "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-4000:]
    return exe


def _tree_rows(t, lv):
    return O.f64_to_bf16_bits(t.keys[lv]), O.f64_to_bf16_bits(t.values[lv])


TIMEOUT_BIT = 4  # kErrTimeout, the device error word's bit for a bounded wait that ran out


def _timeout_words(d):
    """The emulated call's error words: the call's own (append) and the build kernels'."""
    return [int(x) for x in open(d / "err.txt").read().split()]


def _run(emu_bin, tmp_path, lens, hkv, C, b, P=None, per_seq=False, seed=1, stuck=False):
    """Oracle trees over `lens`, the kernel appends C tokens per sequence, check against the
    oracle's trees over lens + C.  per_seq: the kernel reads the lengths from seq_len (else
    every sequence has max(lens) and lens must be equal).  stuck: no tensor-core product ever
    completes; the kernel must report the timeout and return (returns the error words)."""
    B = len(lens)
    L = max(lens)
    cap = L + C
    if P:
        cap = -(-cap // P) * P
    inp = I.random_case(B, L, hkv, hkv * 4, 0, seed=seed, capacity=cap, chunk=C)
    kb, vb = bits(inp["k_tok"]).copy(), bits(inp["v_tok"]).copy()
    knew, vnew = bits(inp["k_new"]), bits(inp["v_new"])
    pooler = inp["pooler"].double().numpy()
    p = R.params(num_kv_heads=hkv, num_q_heads=hkv * 4, branching=b, top_k=2)
    node_rows, levels_cap, offs = R.tree_layout(p, B, cap)
    slots = [cap] + [math.ceil(cap / b ** lv) for lv in range(1, levels_cap + 1)]

    def tree_of(k, v, s, h, n):
        return O.build_tree(O.bf16_bits_to_f64(k[s, h, :n]), O.bf16_bits_to_f64(v[s, h, :n]), pooler, b)

    knode = np.zeros((max(node_rows, 1), 128), np.uint16)
    vnode = np.zeros_like(knode)
    for s, n in enumerate(lens):
        if n == 0:
            continue
        for h in range(hkv):
            t = tree_of(kb, vb, s, h, n)
            for lv in range(1, t.top + 1):
                r0 = offs[lv] + (s * hkv + h) * slots[lv]
                kr, vr = _tree_rows(t, lv)
                knode[r0:r0 + len(kr)] = kr
                vnode[r0:r0 + len(vr)] = vr
    # the expected caches after the append
    ka, va = kb.copy(), vb.copy()
    for s, n in enumerate(lens):
        ka[s, :, n:n + C] = knew[s].transpose(1, 0, 2)
        va[s, :, n:n + C] = vnew[s].transpose(1, 0, 2)

    span = [min(b ** lv, 1 << 62) for lv in range(R.MAX_LEVELS + 1)]
    prm = dict(batch=B, hkv=hkv, b=b, capacity=cap, at=L, chunk=C,
               levels=len(O.level_counts(L + C, b)) - 1, page_shift=0, num_pages=0, stuck=int(stuck))
    pages = None
    k_in, v_in = kb, vb
    if P:
        pps = cap // P
        rng = np.random.default_rng(seed)
        n_pages = B * pps + 2
        perm = rng.permutation(n_pages)[:B * pps].astype(np.int32)
        pages = perm.reshape(B, pps)
        prm.update(page_shift=int(math.log2(P)), num_pages=n_pages)
        k_in = rng.integers(0, 1 << 16, size=(n_pages, hkv, P, 128), dtype=np.uint16)
        v_in = k_in.copy()
        for s in range(B):
            for j in range(pps):
                k_in[pages[s, j]] = kb[s, :, j * P:(j + 1) * P]
                v_in[pages[s, j]] = vb[s, :, j * P:(j + 1) * P]
    d = tmp_path / f"case_{B}_{hkv}_{L}_{C}_{b}_{P}_{int(per_seq)}_{int(stuck)}"
    d.mkdir()
    with open(d / "params.txt", "w") as f:
        for key, val in prm.items():
            f.write(f"{key} {val}\n")
        f.write("row_off " + " ".join(str(offs[i] if i <= levels_cap else 0) for i in range(R.MAX_LEVELS + 1)) + "\n")
        f.write("slots " + " ".join(str(slots[i] if i <= levels_cap else 0) for i in range(R.MAX_LEVELS + 1)) + "\n")
        f.write("span " + " ".join(str(x) for x in span) + "\n")
        if per_seq:
            f.write("seq_len " + " ".join(str(n) for n in lens) + "\n")
        if pages is not None:
            f.write("pages " + " ".join(str(x) for x in pages.reshape(-1)) + "\n")
    for name, arr in (("k_tok", k_in), ("v_tok", v_in), ("k_node", knode), ("v_node", vnode),
                      ("k_new", knew), ("v_new", vnew)):
        np.ascontiguousarray(arr, dtype=np.uint16).tofile(d / f"{name}.bin")
    np.ascontiguousarray(inp["pooler"].numpy(), dtype=np.float32).tofile(d / "pooler.bin")
    r = subprocess.run([emu_bin, str(d)], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    if stuck:
        return _timeout_words(d)

    k_out = np.fromfile(d / "k_tok_out.bin", np.uint16).reshape(k_in.shape)
    v_out = np.fromfile(d / "v_tok_out.bin", np.uint16).reshape(v_in.shape)
    if P:  # back to logical order
        k_out = np.concatenate([k_out[pages[:, j]] for j in range(cap // P)], axis=2)
        v_out = np.concatenate([v_out[pages[:, j]] for j in range(cap // P)], axis=2)
    kn_out = np.fromfile(d / "k_node_out.bin", np.uint16).reshape(knode.shape)
    vn_out = np.fromfile(d / "v_node_out.bin", np.uint16).reshape(vnode.shape)
    mism = total = 0
    for s, n in enumerate(lens):
        m = n + C
        assert np.array_equal(k_out[s, :, :m], ka[s, :, :m]) and np.array_equal(v_out[s, :, :m], va[s, :, :m])
        for h in range(hkv):
            t = tree_of(ka, va, s, h, m)
            for lv in range(1, t.top + 1):
                r0 = offs[lv] + (s * hkv + h) * slots[lv]
                cnt = t.keys[lv].shape[0]
                for got, want in ((kn_out[r0:r0 + cnt], t.keys[lv]), (vn_out[r0:r0 + cnt], t.values[lv])):
                    a, c = check_node_rows(got, want)
                    mism += a
                    total += c
    assert total > 0 and mism <= total * 1e-2


@pytest.mark.parametrize("lens,hkv,C,b", [
    ([1000, 1000], 2, 1, 4),     # one token, ragged nodes at every level
    ([1023], 1, 1, 4),           # 1024 = 4^5: a new top level appears
    ([700, 700], 1, 40, 16),     # several level-1 nodes in one walk
    ([0], 2, 9, 4),              # an empty cache: one level of 3 nodes built from scratch
    ([4096], 1, 1, 16),          # one token: levels 1-2 on the single-node path, level 3 new (2 nodes)
    ([4111], 1, 1, 16),          # one token completing a level-1 node (its 16th child)
    ([3000], 1, 1, 2),           # b = 2: 11 levels of one node each on the single-token path
])
def test_append_matches_oracle(emu_bin, tmp_path, lens, hkv, C, b):
    _run(emu_bin, tmp_path, lens, hkv, C, b)


def test_append_with_per_sequence_lengths(emu_bin, tmp_path):
    _run(emu_bin, tmp_path, [700, 1022, 0, 64], 1, 3, 4, per_seq=True, seed=4)


def test_append_one_token_with_per_sequence_lengths(emu_bin, tmp_path):
    _run(emu_bin, tmp_path, [700, 1023, 0, 4, 65], 1, 1, 4, per_seq=True, seed=6)


@pytest.mark.parametrize("P,C", [(1, 5), (16, 5), (16, 1)])
def test_append_into_a_paged_cache(emu_bin, tmp_path, P, C):
    _run(emu_bin, tmp_path, [600, 301], 1, C, 4, P=P, per_seq=True, seed=P + C)


def _run_build(emu_bin, tmp_path, lens, hkv, b, grid, P=None, per_seq=False, seed=3, stuck=False):
    """The level-build kernel over every level (at most `grid` CTAs striding over the tiles of
    128 nodes) on the CPU; each sequence's node rows against the oracle's tree over its tokens."""
    B, L = len(lens), max(lens)
    cap = -(-L // P) * P if P else L
    inp = I.random_case(B, L, hkv, hkv * 4, 0, seed=seed, capacity=cap)
    kb, vb = bits(inp["k_tok"]), bits(inp["v_tok"])
    pooler = inp["pooler"].double().numpy()
    p = R.params(num_kv_heads=hkv, num_q_heads=hkv * 4, branching=b, top_k=2)
    node_rows, levels_cap, offs = R.tree_layout(p, B, cap)
    slots = [cap] + [math.ceil(cap / b ** lv) for lv in range(1, levels_cap + 1)]
    prm = dict(mode=1, length=L, grid=grid, batch=B, hkv=hkv, b=b, capacity=cap, at=0, chunk=0,
               levels=len(O.level_counts(L, b)) - 1, page_shift=0, num_pages=0, stuck=int(stuck))
    k_in, v_in, pages = kb, vb, None
    if P:
        pps = cap // P
        rng = np.random.default_rng(seed)
        n_pages = B * pps + 3
        pages = rng.permutation(n_pages)[:B * pps].astype(np.int32).reshape(B, pps)
        prm.update(page_shift=int(math.log2(P)), num_pages=n_pages)
        k_in = rng.integers(0, 1 << 16, size=(n_pages, hkv, P, 128), dtype=np.uint16)
        v_in = k_in.copy()
        for s in range(B):
            for j in range(pps):
                k_in[pages[s, j]] = kb[s, :, j * P:(j + 1) * P]
                v_in[pages[s, j]] = vb[s, :, j * P:(j + 1) * P]
    d = tmp_path / f"build_{B}_{hkv}_{L}_{b}_{grid}_{P}_{int(per_seq)}_{int(stuck)}"
    d.mkdir()
    span = [min(b ** lv, 1 << 62) for lv in range(R.MAX_LEVELS + 1)]
    with open(d / "params.txt", "w") as f:
        for key, val in prm.items():
            f.write(f"{key} {val}\n")
        f.write("row_off " + " ".join(str(offs[i] if i <= levels_cap else 0) for i in range(R.MAX_LEVELS + 1)) + "\n")
        f.write("slots " + " ".join(str(slots[i] if i <= levels_cap else 0) for i in range(R.MAX_LEVELS + 1)) + "\n")
        f.write("span " + " ".join(str(x) for x in span) + "\n")
        if per_seq:
            f.write("seq_len " + " ".join(str(n) for n in lens) + "\n")
        if pages is not None:
            f.write("pages " + " ".join(str(x) for x in pages.reshape(-1)) + "\n")
    zeros = np.zeros((max(node_rows, 1), 128), np.uint16)
    for name, arr in (("k_tok", k_in), ("v_tok", v_in), ("k_node", zeros), ("v_node", zeros),
                      ("k_new", np.zeros(0, np.uint16)), ("v_new", np.zeros(0, np.uint16))):
        np.ascontiguousarray(arr, dtype=np.uint16).tofile(d / f"{name}.bin")
    np.ascontiguousarray(inp["pooler"].numpy(), dtype=np.float32).tofile(d / "pooler.bin")
    r = subprocess.run([emu_bin, str(d)], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    if stuck:
        return _timeout_words(d)
    kn_out = np.fromfile(d / "k_node_out.bin", np.uint16).reshape(zeros.shape)
    vn_out = np.fromfile(d / "v_node_out.bin", np.uint16).reshape(zeros.shape)
    mism = total = 0
    for s, n in enumerate(lens):
        if n == 0:
            continue
        for h in range(hkv):
            t = O.build_tree(O.bf16_bits_to_f64(kb[s, h, :n]), O.bf16_bits_to_f64(vb[s, h, :n]), pooler, b)
            for lv in range(1, t.top + 1):
                r0 = offs[lv] + (s * hkv + h) * slots[lv]
                cnt = t.keys[lv].shape[0]
                for got, want in ((kn_out[r0:r0 + cnt], t.keys[lv]), (vn_out[r0:r0 + cnt], t.values[lv])):
                    a, c = check_node_rows(got, want)
                    mism += a
                    total += c
    assert total > 0 and mism <= total * 1e-2


@pytest.mark.parametrize("grid", [1, 1000])  # one CTA striding over every tile, and a CTA a tile
def test_level_build_matches_oracle(emu_bin, tmp_path, grid):
    _run_build(emu_bin, tmp_path, [1000, 1000], 2, 4, grid)


def test_level_build_with_per_sequence_lengths_and_pages(emu_bin, tmp_path):
    _run_build(emu_bin, tmp_path, [700, 0, 301, 64], 1, 4, 3, P=8, per_seq=True)


# The timeout path: a tensor-core product that never completes (on the host, every mbarrier
# wait gives up).  The kernels must set the timeout bit, stop, and return: the emulator's
# rendezvous would report a thread left waiting, and AddressSanitizer a bad access.
@pytest.mark.parametrize("C", [1, 5])  # the single-token path and the general one
def test_append_reports_a_product_that_never_completes(emu_bin, tmp_path, C):
    call_word, build_word = _run(emu_bin, tmp_path, [1000], 2, C, 4, stuck=True)
    assert call_word & TIMEOUT_BIT and build_word & TIMEOUT_BIT


@pytest.mark.parametrize("grid", [1, 1000])  # the wait inside the tile loop, and the last one
def test_level_build_reports_a_product_that_never_completes(emu_bin, tmp_path, grid):
    _, build_word = _run_build(emu_bin, tmp_path, [1000, 1000], 2, 4, grid, stuck=True)
    assert build_word & TIMEOUT_BIT

