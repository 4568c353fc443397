"""RecSA oracle: a plain, slow, fp64 CPU restatement of Recursive Sparse Attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA library; the only thing the
two have in common is the seeded input generator (``recsa_inputs``), which holds
none of the method's arithmetic.

Source: "Recursive Sparse Attention: Million-Token Length Extrapolation at
Logarithmic Cost" (arXiv 2611.07232), abstract.  The abstract states:

  (A1) a tree is built over the KV cache, each node summarising its subtree with
       one key and one mean-pooled value;
  (A2) keys come from one pooler per layer, shared by all levels;
  (A3) each level above the tokens selects at most k candidates, so a query reads
       O(log L) entries;
  (A4) the summaries of unselected candidates share one softmax with the exact
       tokens;
  (A5) each entry's RoPE position is its index among the candidates of its level.

The abstract leaves the rest open.  The readings adopted here (each marked R<n>
below and listed with its reason in the design notes) are:

  R1  pooler: parent key = W @ (plain mean of the children's stored pre-RoPE keys),
      W a supplied 128x128 matrix applied at every level.
  R2  storage: in "bf16" mode every node row is rounded to bf16 (nearest, ties to
      even) when stored and the next level reads the stored rows; "exact" mode
      keeps fp64 rows.
  R3  parent value = token-count-weighted mean of its children's values, i.e. the
      plain mean of the subtree's tokens.
  R4  levels: n_0 = L, n_{l+1} = ceil(n_l / b) while n_l > b; the top level T holds
      at most b nodes; L <= b gives T = 0 (plain attention over the tokens).
  R5  candidates of a level are ordered by node index; a candidate's RoPE position
      is its rank in that order; the query's RoPE position is the level's
      candidate count.
  R6  a query at position p sees tokens [0, p): decode queries sit at p = L,
      prefill query i of a chunk appended at L sits at p = L + i.
  R7  RoPE is rotate-half over dims (i, i + 64), angle pos * base^(-2i/128).
  R8  logits are scaled by 1/sqrt(128) unless a scale is given.
  R9  selection ranks candidates by S(c) = sum over the KV group's query heads of the
      scaled logits; the top min(k, #scorable) are kept, ties to the lower node index.
  R10 k = TOPK_ALL keeps every candidate (full expansion).
  R11 the shared softmax adds no bias for a summary's subtree size.
  R12 causal (prefill) mode: at each level the partial trailing node (holding
      tokens both below and at/after p) is not scored, takes no top-k slot, is
      counted among the candidates (so it holds a RoPE position) and is always
      expanded; nodes starting at or after p are not candidates.
  R13 decode mode: a partial last node (L not a multiple of b^l) is an ordinary
      candidate summarising the tokens it holds.
  R14 a query with no visible entry (prefill from an empty cache, query 0) outputs 0.
"""

from __future__ import annotations

import math

import numpy as np

HEAD_DIM = 128
HALF = HEAD_DIM // 2
TOPK_ALL = 0x7FFFFFFF


# ---------------------------------------------------------------------------
# bf16 storage (R2)
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits) -> np.ndarray:
    """Value of raw bf16 bit patterns: a bf16 is the top 16 bits of an IEEE fp32."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def round_to_bf16(x) -> np.ndarray:
    """Nearest bf16 value (ties to even) of each fp64 element, returned as fp64.

    bf16 keeps 8 significant bits and fp32's exponent range.  Writing a normal x
    as m * 2**e with 0.5 <= |m| < 1, the result is round_half_even(m * 2**8) * 2**(e - 8).
    Values below 2**-126 are bf16 subnormals with a fixed spacing of 2**-133."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("round_to_bf16: non-finite input")
    m, e = np.frexp(x)
    normal = np.ldexp(np.round(np.ldexp(m, 8)), e - 8)
    sub = np.ldexp(np.round(np.ldexp(x, 133)), -133)
    out = np.where(np.abs(x) < 2.0 ** -126, sub, normal)
    if np.any(np.abs(out) > 3.3895313892515355e38):
        raise ValueError("round_to_bf16: overflow")
    return out


def f64_to_bf16_bits(x) -> np.ndarray:
    """bf16 bit pattern of round_to_bf16(x)."""
    r = round_to_bf16(x).astype(np.float32)  # exact: r is representable in bf16
    return (r.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Tree structure (A1, R4)
# ---------------------------------------------------------------------------

def level_counts(length: int, b: int) -> list[int]:
    """Node counts per level [n_0 = L, n_1, ..., n_T] under R4."""
    if b < 2:
        raise ValueError("branching must be >= 2")
    n = [int(length)]
    while n[-1] > b:
        n.append(-(-n[-1] // b))
    return n


def subtree_tokens(level: int, node: int, b: int, length: int) -> int:
    """Number of tokens under node `node` of `level` in a cache of `length` tokens."""
    span = b ** level
    return max(0, min(span, length - node * span))


# ---------------------------------------------------------------------------
# Build (A1, A2, R1-R3)
# ---------------------------------------------------------------------------

class Tree:
    """One (sequence, KV head) tree: keys[l], values[l], counts[l] for l = 0..T (level 0 = tokens)."""

    def __init__(self, keys, values, counts, b):
        self.keys = keys
        self.values = values
        self.counts = counts
        self.b = b

    @property
    def length(self) -> int:
        return self.keys[0].shape[0]

    @property
    def top(self) -> int:
        return len(self.keys) - 1


def build_level(kp, vp, cp, pooler, b: int, storage: str = "bf16"):
    """One level above [n_prev] rows kp, vp of token counts cp: node j covers children
    j*b .. j*b+b-1 (the last node fewer), key = W @ mean(children keys) (R1), value = the
    count-weighted mean of the children values (R3), count = the children's sum.  With
    bf16 storage the rows are rounded as stored (R2).  Returns (keys, values, counts)."""
    W = np.asarray(pooler, dtype=np.float64)
    n_prev = kp.shape[0]
    n = -(-n_prev // b)
    kn = np.empty((n, HEAD_DIM))
    vn = np.empty((n, HEAD_DIM))
    cn = np.empty(n)
    for j in range(n):
        c0, c1 = j * b, min((j + 1) * b, n_prev)
        mean_key = kp[c0:c1].sum(axis=0) / (c1 - c0)
        kn[j] = W @ mean_key
        w = cp[c0:c1]
        vn[j] = (w[:, None] * vp[c0:c1]).sum(axis=0) / w.sum()
        cn[j] = w.sum()
    if storage == "bf16":
        kn = round_to_bf16(kn)
        vn = round_to_bf16(vn)
    return kn, vn, cn


def build_tree(k_tok, v_tok, pooler, b: int, storage: str = "bf16") -> Tree:
    """Build the summary tree of one (sequence, KV head).

    k_tok, v_tok: [L][128] fp64 token keys (pre-RoPE) and values.
    pooler: [128][128] W; a parent key is W @ mean(children keys) (R1).
    Parent values are the token-count-weighted mean of the children (R3)."""
    if storage not in ("bf16", "exact"):
        raise ValueError(storage)
    k_tok = np.asarray(k_tok, dtype=np.float64)
    v_tok = np.asarray(v_tok, dtype=np.float64)
    L = k_tok.shape[0]
    ns = level_counts(L, b)
    keys, values, counts = [k_tok], [v_tok], [np.ones(L)]
    for _ in range(1, len(ns)):
        kn, vn, cn = build_level(keys[-1], values[-1], counts[-1], pooler, b, storage)
        keys.append(kn)
        values.append(vn)
        counts.append(cn)
    return Tree(keys, values, counts, b)


# ---------------------------------------------------------------------------
# RoPE at candidate index (A5, R7)
# ---------------------------------------------------------------------------

def rope(x, pos, base: float) -> np.ndarray:
    """Rotate-half RoPE of rows x [..., 128] at integer positions pos (broadcast over rows)."""
    x = np.asarray(x, dtype=np.float64)
    pos = np.asarray(pos, dtype=np.float64)
    inv_freq = float(base) ** (-(2.0 * np.arange(HALF)) / HEAD_DIM)
    ang = pos[..., None] * inv_freq
    c, s = np.cos(ang), np.sin(ang)
    lo, hi = x[..., :HALF], x[..., HALF:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


# ---------------------------------------------------------------------------
# Level-wise attend (A3-A5, R5-R14)
# ---------------------------------------------------------------------------

class Trace:
    """What one query group did at each level (top level first)."""

    def __init__(self):
        self.levels = []  # dicts: level, nodes, forced, qpos, S, kept, gap, n_keys, n_values
        self.weights = None  # [G][E] softmax weights of all entries
        self.entry_positions = []  # RoPE positions of every entry (keys read), for the offset bound

    @property
    def keys_read(self) -> int:
        return sum(d["n_keys"] for d in self.levels)

    @property
    def values_read(self) -> int:
        return sum(d["n_values"] for d in self.levels)

    def selections(self) -> list[list[int]]:
        return [sorted(d["kept"]) for d in self.levels if d["level"] > 0]


def _top_candidates(tree: Tree, p: int, causal: bool, top: int):
    """Candidates of the top level: all nodes (decode) or the visible ones (causal, R12)."""
    if not causal:
        return [(j, False) for j in range(tree.keys[top].shape[0])]
    span = tree.b ** top
    cands = [(j, False) for j in range(p // span)]
    if p % span:
        cands.append((p // span, True))
    return cands


def _children(tree: Tree, level: int, node: int, forced: bool, p: int, causal: bool):
    """Children (next-level candidates) of an expanded node, in node order."""
    b = tree.b
    n_below = tree.keys[level - 1].shape[0]
    out = []
    span_below = b ** (level - 1)
    for c in range(node * b, min((node + 1) * b, n_below)):
        if causal:
            start = c * span_below
            if start >= p:
                break
            out.append((c, forced and (c + 1) * span_below > p))
        else:
            out.append((c, False))
    return out


def attend(q, tree: Tree, p: int, k: int, scale: float | None = None, base: float = 1.0e6,
           causal: bool = False, selection=None, tie_tol: float = 1e-3, trace: Trace | None = None):
    """Output of one KV group's query heads for a query at position p.

    q: [G][128] pre-RoPE query rows of the group.  tree: the group's tree (built over
    at least p tokens).  decode: causal=False and p = tree length.  prefill: causal=True.
    selection: optional replay list (top level first) of the node sets to keep at each
    level above the tokens; each set must be a top-k up to near-ties (|dS| < tie_tol).
    Returns out [G][128] (fp64)."""
    q = np.asarray(q, dtype=np.float64)
    G = q.shape[0]
    scale = 1.0 / math.sqrt(HEAD_DIM) if not scale else float(scale)
    if causal:
        top = len(level_counts(p, tree.b)) - 1
    else:
        if p != tree.length:
            raise ValueError("decode queries sit at p = L")
        top = tree.top
    if top > tree.top:
        raise ValueError("tree has too few levels for p")
    ent_logits, ent_values = [], []
    cands = _top_candidates(tree, p, causal, top) if top > 0 else None
    level_sel = list(selection) if selection is not None else None
    for lvl in range(top, 0, -1):
        nodes = np.array([c for c, _ in cands], dtype=np.int64)
        forced = np.array([f for _, f in cands], dtype=bool)
        n = len(cands)
        qpos = n                                     # R5: query sits at the candidate count
        idx = np.arange(n)                           # R5: RoPE position = rank
        qr = rope(q, np.full(G, qpos), base)
        sc = np.flatnonzero(~forced)                 # scorable candidates (R12)
        kr = rope(tree.keys[lvl][nodes[sc]], idx[sc], base)
        logits = scale * (qr @ kr.T)                 # [G][m]
        S = logits.sum(axis=0)                       # R9
        m = len(sc)
        keep = min(k, m)
        order = np.lexsort((nodes[sc], -S))          # S descending, node ascending (R9)
        kept_pos = set(sc[order[:keep]].tolist())
        gap = float(S[order[keep - 1]] - S[order[keep]]) if 0 < keep < m else None
        if level_sel is not None:
            want = set(int(x) for x in level_sel.pop(0))
            pos_of = {int(nodes[i]): i for i in sc}
            if len(want) != keep or not want <= set(pos_of):
                raise ValueError(f"replayed selection at level {lvl} is not {keep} scorable candidates")
            kept_pos = set(pos_of[x] for x in want)
            s_of = {int(nodes[i]): S[j] for j, i in enumerate(sc)}
            lo = min((s_of[x] for x in want), default=np.inf)
            hi = max((s_of[int(nodes[i])] for i in sc if i not in kept_pos), default=-np.inf)
            if hi - lo >= tie_tol:
                raise ValueError(f"replayed selection at level {lvl} drops a candidate by {hi - lo}")
        n_values = 0
        for j, i in enumerate(sc):
            if i not in kept_pos:                    # A4: unselected summaries join the softmax
                ent_logits.append(logits[:, j])
                ent_values.append(tree.values[lvl][nodes[i]])
                n_values += 1
        if trace is not None:
            trace.levels.append(dict(level=lvl, nodes=nodes.tolist(), forced=forced.tolist(), qpos=qpos,
                                     S=dict(zip(nodes[sc].tolist(), S.tolist())),
                                     kept=sorted(int(nodes[i]) for i in kept_pos), gap=gap,
                                     n_keys=m, n_values=n_values))
            trace.entry_positions.extend((qpos - idx[sc]).tolist())
        nxt = []
        for i in range(n):
            if i in kept_pos or forced[i]:           # A3: expand kept (and forced, R12) nodes
                nxt.extend(_children(tree, lvl, int(nodes[i]), bool(forced[i]), p, causal))
        cands = nxt
    # level 0: exact tokens (A4)
    if top == 0:
        toks = np.arange(p if causal else tree.length, dtype=np.int64)
    else:
        toks = np.array([c for c, _ in cands], dtype=np.int64)
    n0 = len(toks)
    if n0:
        qr = rope(q, np.full(G, n0), base)
        kr = rope(tree.keys[0][toks], np.arange(n0), base)
        logits = scale * (qr @ kr.T)
        ent_logits.extend(logits.T)
        ent_values.extend(tree.values[0][toks])
    if trace is not None:
        trace.levels.append(dict(level=0, nodes=toks.tolist(), forced=[False] * n0, qpos=n0, S={},
                                 kept=[], gap=None, n_keys=n0, n_values=n0))
        trace.entry_positions.extend((n0 - np.arange(n0)).tolist())
    if not ent_logits:                               # R14
        if trace is not None:
            trace.weights = np.zeros((G, 0))
        return np.zeros((G, HEAD_DIM))
    lg = np.stack(ent_logits, axis=1)                # [G][E]
    vals = np.stack(ent_values, axis=0)              # [E][128]
    mx = lg.max(axis=1, keepdims=True)
    e = np.exp(lg - mx)
    wts = e / e.sum(axis=1, keepdims=True)
    if trace is not None:
        trace.weights = wts
    return wts @ vals


def dense_attention(q, keys, values, qpos: int, scale: float | None = None, base: float = 1.0e6):
    """Plain RoPE attention: rows keys/values [n][128] at positions 0..n-1, query at qpos."""
    q = np.asarray(q, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    scale = 1.0 / math.sqrt(HEAD_DIM) if not scale else float(scale)
    n = keys.shape[0]
    if n == 0:
        return np.zeros((q.shape[0], HEAD_DIM))
    qr = rope(q, np.full(q.shape[0], qpos), base)
    kr = rope(keys, np.arange(n), base)
    lg = scale * (qr @ kr.T)
    e = np.exp(lg - lg.max(axis=1, keepdims=True))
    return (e / e.sum(axis=1, keepdims=True)) @ values


# ---------------------------------------------------------------------------
# Whole-call drivers (plain loops over sequences, KV groups and queries)
# ---------------------------------------------------------------------------

def build_all(k_bits, v_bits, pooler, b, length, storage="bf16"):
    """Trees for every (sequence, KV head).  k_bits, v_bits: uint16 [B][Hkv][>=L][128]."""
    B, H = k_bits.shape[:2]
    return [[build_tree(bf16_bits_to_f64(k_bits[bi, h, :length]), bf16_bits_to_f64(v_bits[bi, h, :length]),
                        pooler, b, storage) for h in range(H)] for bi in range(B)]


def decode_all(trees, q_bits, k, scale=None, base=1.0e6, traces=None):
    """Decode outputs [B][Q][Hq][128] (fp64); q_bits uint16 [B][Q][Hq][128]."""
    B, Q, Hq, _ = q_bits.shape
    H = len(trees[0])
    G = Hq // H
    out = np.zeros((B, Q, Hq, HEAD_DIM))
    for bi in range(B):
        for qi in range(Q):
            for h in range(H):
                tr = Trace() if traces is not None else None
                qg = bf16_bits_to_f64(q_bits[bi, qi, h * G:(h + 1) * G])
                out[bi, qi, h * G:(h + 1) * G] = attend(qg, trees[bi][h], trees[bi][h].length, k, scale, base,
                                                        trace=tr)
                if traces is not None:
                    traces[(bi, qi, h)] = tr
    return out


def append_chunk(k_bits, v_bits, knew_bits, vnew_bits, length):
    """Token caches [B][Hkv][length + C][128] after appending a chunk given as [B][C][Hkv][128]."""
    C = knew_bits.shape[1]
    k = np.concatenate([k_bits[:, :, :length], knew_bits.transpose(0, 2, 1, 3)], axis=2)
    v = np.concatenate([v_bits[:, :, :length], vnew_bits.transpose(0, 2, 1, 3)], axis=2)
    assert k.shape[2] == length + C
    return k, v


def prefill_all(k_bits, v_bits, knew_bits, vnew_bits, q_bits, pooler, b, length, k, scale=None, base=1.0e6,
                storage="bf16", queries=None, traces=None):
    """Causal outputs of a prefill chunk (R6, R12): query i sits at p = length + i.

    The chunk [B][C][Hkv][128] is appended to the caches, the trees are built over
    length + C tokens, and each query attends causally.  `queries` optionally limits
    the work to a list of chunk indices (rows not computed stay zero)."""
    B, C, Hq, _ = q_bits.shape
    kc, vc = append_chunk(k_bits, v_bits, knew_bits, vnew_bits, length)
    trees = build_all(kc, vc, pooler, b, length + C, storage)
    H = len(trees[0])
    G = Hq // H
    out = np.zeros((B, C, Hq, HEAD_DIM))
    for bi in range(B):
        for i in (range(C) if queries is None else queries):
            for h in range(H):
                tr = Trace() if traces is not None else None
                qg = bf16_bits_to_f64(q_bits[bi, i, h * G:(h + 1) * G])
                out[bi, i, h * G:(h + 1) * G] = attend(qg, trees[bi][h], length + i, k, scale, base,
                                                       causal=True, trace=tr)
                if traces is not None:
                    traces[(bi, i, h)] = tr
    return out, trees
