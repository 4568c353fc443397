"""Helpers that run the CUDA library and the fp64 oracle on the same seeded inputs.

Comparison rules (the method's acceptance bar):
  * node rows: every row within two bf16 ulps of its largest element, and at most
    1% of elements not bit-identical (counted);
  * selections: the kept node set of every level equals the oracle's, except for
    swaps between candidates whose oracle group scores differ by less than 1e-3;
    such tiles are re-scored by the oracle with the library's selection (which the
    oracle first checks is a top-k up to those near-ties) and counted;
  * outputs: max |diff| <= 2e-2 and mean |diff| <= 5e-3 against the oracle (fp32
    output of bf16 inputs with fp32 accumulation).
"""

from __future__ import annotations

import os

import numpy as np
import torch

import hierarchical_sparse_attention_build_b200 as R
import recsa_inputs as I
from oracle import recsa_oracle as O

MAX_ABS = 2e-2
MEAN_ABS = 5e-3
TIE_TOL = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    return I.bf16_bits(t)


def ordered(b16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> integers whose difference counts ulps (sign-magnitude to two's complement)."""
    b = b16.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    return np.abs(ordered(a_bits) - ordered(b_bits))


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (8 significant bits)."""
    e = np.frexp(np.maximum(np.abs(x), 2.0 ** -126))[1]
    return np.ldexp(1.0, e - 8)


def check_node_rows(got_bits: np.ndarray, want: np.ndarray) -> tuple[int, int]:
    """Library node rows vs oracle rows [n][128].

    Each row must satisfy max|gpu - oracle| <= 2^-7 * max|oracle row| (two bf16 ulps of
    the row's largest element).  Elementwise one-ulp agreement is not a valid bar: the
    library rounds an fp32 value and the oracle an fp64 one, so a row can be one ulp
    apart, and a parent element whose children nearly cancel then moves by several of
    its own ulps.  A wrong child, weight or pooler moves rows by far more than this.
    Returns (elements not bit-identical, total)."""
    got = O.bf16_bits_to_f64(got_bits)
    want = np.asarray(want, dtype=np.float64)
    tol = 2.0 ** -7 * np.abs(want).max(axis=-1, keepdims=True) + 2.0 ** -133
    bad = np.abs(got - want) > tol
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], want[bad][:5])
    return int((got_bits != O.f64_to_bf16_bits(want)).sum()), got_bits.size


class GpuCase:
    """Inputs on the device, a library tree over them and an initialised workspace."""

    def __init__(self, inp: dict, p: R.Params, length: int, device="cuda"):
        self.p = p
        self.inp = inp
        self.k_tok = inp["k_tok"].to(device).contiguous()
        self.v_tok = inp["v_tok"].to(device).contiguous()
        self.pooler = inp["pooler"].to(device).contiguous()
        self.tree = R.RecsaTree(p, self.k_tok, self.v_tok, self.pooler, length)
        self.ws = R.Workspace(p, self.tree.capacity, device)

    def build(self):
        R.build_tree(self.p, self.tree)

    def decode(self, q: torch.Tensor, cluster_size=0, sel_levels=None, fp32=True, kernel=0):
        q = q.to(self.k_tok.device).contiguous()
        B, Q, Hq, _ = q.shape
        out = torch.empty(B, Q, Hq, 128, dtype=torch.float32 if fp32 else torch.bfloat16, device=q.device)
        tiles = B * self.p.num_kv_heads * Q
        sel = None
        lv = sel_levels or max(self.tree.levels, 1)
        if self.p.top_k <= 64 and self.p.top_k >= 1:
            sel = torch.full((tiles, lv, self.p.top_k), -7, dtype=torch.int32, device=q.device)
        ent = torch.zeros(tiles, 2, dtype=torch.int32, device=q.device)
        R.decode(self.p, self.tree, q, out, self.ws, sel_idx=sel, sel_levels=lv, entries=ent,
                 cluster_size=cluster_size, kernel=kernel)
        R.check_device_errors(self.ws)
        torch.cuda.synchronize()
        return out.cpu(), (sel.cpu().numpy() if sel is not None else None), ent.cpu().numpy()

    def prefill(self, k_new, v_new, q, cluster_size=0, fp32=True, sel_levels=None, kernel=0):
        dev = self.k_tok.device
        k_new, v_new, q = k_new.to(dev).contiguous(), v_new.to(dev).contiguous(), q.to(dev).contiguous()
        B, C, Hq, _ = q.shape
        out = torch.empty(B, C, Hq, 128, dtype=torch.float32 if fp32 else torch.bfloat16, device=dev)
        tiles = B * self.p.num_kv_heads * C
        lv = sel_levels or max(self.tree.levels, 1)
        sel = None
        if 1 <= self.p.top_k <= 64:
            sel = torch.full((tiles, lv, self.p.top_k), -7, dtype=torch.int32, device=dev)
        ent = torch.zeros(tiles, 2, dtype=torch.int32, device=dev)
        R.prefill_chunk(self.p, self.tree, k_new, v_new, q, out, self.ws, sel_idx=sel, sel_levels=lv, entries=ent,
                        cluster_size=cluster_size, kernel=kernel)
        R.check_device_errors(self.ws)
        torch.cuda.synchronize()
        return out.cpu(), (sel.cpu().numpy() if sel is not None else None), ent.cpu().numpy()

    def node_bits(self, level: int) -> tuple[np.ndarray, np.ndarray]:
        k, v = self.tree.level_rows(level)
        return bits(k), bits(v)


def gpu_selection(sel: np.ndarray, tile: int, top: int) -> list[list[int]]:
    """Kept node sets of one tile, top level first (levels top .. 1)."""
    out = []
    for lvl in range(top, 0, -1):
        row = sel[tile, lvl - 1]
        out.append(sorted(int(x) for x in row if x >= 0))
    return out


# Every Stats made while a test runs is recorded under that test's id, so the end of the
# session can report tiles, near-tie swaps and errors per configuration.
REPORT: list[tuple[str, "Stats"]] = []


class Stats:
    def __init__(self, label: str | None = None):
        test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" (")[0]
        REPORT.append((label or test or "untitled", self))
        self.tiles = 0
        self.near_ties = 0
        self.max_abs = 0.0
        self.sum_abs = 0.0
        self.count = 0

    def add(self, diff: np.ndarray):
        self.max_abs = max(self.max_abs, float(np.abs(diff).max()) if diff.size else 0.0)
        self.sum_abs += float(np.abs(diff).sum())
        self.count += diff.size

    @property
    def mean_abs(self) -> float:
        return self.sum_abs / max(self.count, 1)

    def assert_ok(self):
        assert self.max_abs <= MAX_ABS, f"max |diff| {self.max_abs}"
        assert self.mean_abs <= MEAN_ABS, f"mean |diff| {self.mean_abs}"

    def __repr__(self):
        return (f"tiles={self.tiles} near_ties={self.near_ties} max_abs={self.max_abs:.3e} "
                f"mean_abs={self.mean_abs:.3e}")


def check_tile(stats: Stats, q_group: np.ndarray, tree: O.Tree, p: int, k: int, causal: bool,
               gpu_out: np.ndarray, gpu_sel: list[list[int]] | None, gpu_entries=None, scale=None):
    """Compare one tile (G query heads of a KV group) with the oracle."""
    tr = O.Trace()
    want = O.attend(q_group, tree, p, k, scale=scale, causal=causal, trace=tr)
    stats.tiles += 1
    if gpu_sel is not None:
        osel = tr.selections()
        assert len(gpu_sel) == len(osel), (gpu_sel, osel)
        if gpu_sel != osel:
            # a near-tie swap: the oracle re-scores with the library's choice after checking it
            want = O.attend(q_group, tree, p, k, scale=scale, causal=causal, selection=gpu_sel, tie_tol=TIE_TOL)
            stats.near_ties += 1
            tr2 = O.Trace()
            O.attend(q_group, tree, p, k, scale=scale, causal=causal, selection=gpu_sel, trace=tr2)
            tr = tr2
    if gpu_entries is not None:
        assert int(gpu_entries[0]) == tr.keys_read and int(gpu_entries[1]) == tr.values_read, (
            gpu_entries, tr.keys_read, tr.values_read)
    stats.add(np.asarray(gpu_out, dtype=np.float64) - want)


def oracle_trees(inp: dict, b: int, length: int, storage="bf16"):
    return O.build_all(bits(inp["k_tok"]), bits(inp["v_tok"]), inp["pooler"].double().numpy(), b, length, storage)
