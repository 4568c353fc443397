"""Seeded synthetic inputs for the RecSA tree build and level-wise sparse attend.

This module only draws numbers: token keys/values, queries and the pooler matrix.
It holds none of the method's arithmetic, so both the fp64 oracle (``oracle/``) and
the CUDA library's tests and benchmark take their inputs from here.

The shapes follow the attention of Qwen3-4B, the model the RecSA paper
("Recursive Sparse Attention: Million-Token Length Extrapolation at Logarithmic
Cost", abstract) initialises from: 32 query heads, 8 KV heads, head_dim 128,
RoPE base 1e6.  The paper evaluates on RULER at 131K-2M tokens; RULER is not used
here, these seeded random caches stand in for it.

Recipe (every draw is fp32 from a seeded ``torch.Generator`` and is then cast to
bf16 with round-to-nearest-even):

* token keys/values ``[B][Hkv][capacity][128]`` bf16, N(0, 1); slots at or past
  ``length`` are zero;
* ``channel_scaled`` caches multiply K and V by independent per-(KV head, channel)
  scales drawn from U(0.5, 2) before the cast (queries stay unscaled);
* ``needles`` caches overwrite 64 token positions per sequence (uniform, without
  replacement, shared by all KV heads) with keys ``sqrt(128) * (0.9 u + sqrt(0.19) w)``
  where ``u`` is the unit mean direction of the KV group's query vectors and ``w``
  a random unit vector orthogonal to ``u`` (cosine 0.9 with ``u``);
* queries ``[B][Q][Hq][128]`` bf16, N(0, 1);
* the pooler ``W`` is the Q factor of the QR decomposition of an N(0, 1) 128x128
  fp64 matrix with the signs fixed by ``diag(R) > 0``, stored as fp32.

Seeds are ``20260 + n`` for the n-th named workload.  Small workloads are drawn
on the CPU; the large ones are drawn on the device the caller names (the same
seed gives the same numbers on the same device type and torch version).
"""

from __future__ import annotations

import dataclasses

import torch

HEAD_DIM = 128
ROPE_BASE = 1.0e6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    number: int
    batch: int
    length: int
    kv_heads: int
    q_heads: int
    branching: int
    top_k: int
    queries: int = 1  # independent decode queries per sequence
    chunk: int = 0  # prefill chunk length (0 = decode workload)
    dist: str = "normal"  # normal | channel_scaled | needles
    needles: int = 0

    @property
    def seed(self) -> int:
        return 20260 + self.number

    @property
    def capacity(self) -> int:
        return self.length + self.chunk


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_decode", 1, batch=1, length=4096, kv_heads=1, q_heads=4,
                 branching=8, top_k=4, queries=16),
        Workload("decode_131k", 2, batch=8, length=131072, kv_heads=8, q_heads=32,
                 branching=16, top_k=8, dist="channel_scaled"),
        Workload("decode_1m", 3, batch=4, length=1 << 20, kv_heads=8, q_heads=32,
                 branching=16, top_k=8, dist="needles", needles=64),
        Workload("prefill_524k", 4, batch=1, length=524288, kv_heads=8, q_heads=32,
                 branching=16, top_k=8, chunk=8192),
        Workload("build_decode_2m", 5, batch=1, length=1 << 21, kv_heads=8, q_heads=32,
                 branching=16, top_k=8),
    ]
}


def pooler_matrix(seed: int) -> torch.Tensor:
    """Seeded random orthogonal 128x128 pooler, fp32, row-major (CPU)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    a = torch.randn(HEAD_DIM, HEAD_DIM, generator=g, dtype=torch.float64)
    qm, r = torch.linalg.qr(a)
    sign = torch.sign(torch.diagonal(r))
    sign[sign == 0] = 1.0
    return (qm * sign).to(torch.float32).contiguous()


def _normal_bf16(shape, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def token_cache(batch, kv_heads, length, capacity, g, device, dist="normal") -> tuple[torch.Tensor, torch.Tensor]:
    """K and V caches [B][Hkv][capacity][128] bf16 with the first ``length`` slots drawn."""
    k = torch.zeros(batch, kv_heads, capacity, HEAD_DIM, dtype=torch.bfloat16, device=device)
    v = torch.zeros_like(k)
    if dist == "channel_scaled":
        sk = torch.rand(kv_heads, 1, HEAD_DIM, generator=g, device=device) * 1.5 + 0.5
        sv = torch.rand(kv_heads, 1, HEAD_DIM, generator=g, device=device) * 1.5 + 0.5
    for bi in range(batch):
        for t, s in ((k, sk if dist == "channel_scaled" else None), (v, sv if dist == "channel_scaled" else None)):
            x = torch.randn(kv_heads, length, HEAD_DIM, generator=g, device=device, dtype=torch.float32)
            if s is not None:
                x.mul_(s)
            t[bi, :, :length].copy_(x.to(torch.bfloat16))
            del x
    return k, v


def plant_needles(k_tok, q, length, count, kv_heads, q_heads, g) -> torch.Tensor:
    """Overwrite ``count`` key positions per sequence with keys at cosine 0.9 to the group's mean query.

    Returns the planted positions [B][count] (int64, CPU)."""
    device = k_tok.device
    batch = k_tok.shape[0]
    group = q_heads // kv_heads
    positions = []
    for bi in range(batch):
        pos = torch.randperm(length, generator=g, device=device)[:count]
        positions.append(pos.cpu())
        for h in range(kv_heads):
            qg = q[bi, 0, h * group:(h + 1) * group].to(torch.float32)
            u = qg.mean(0)
            u = u / u.norm()
            w = torch.randn(count, HEAD_DIM, generator=g, device=device, dtype=torch.float32)
            w = w - (w @ u)[:, None] * u[None, :]
            w = w / w.norm(dim=1, keepdim=True)
            key = (HEAD_DIM ** 0.5) * (0.9 * u[None, :] + (0.19 ** 0.5) * w)
            k_tok[bi, h, pos] = key.to(torch.bfloat16)
    return torch.stack(positions)


def decode_inputs(w: Workload, device="cpu", capacity: int | None = None) -> dict:
    """Token caches, queries and pooler of a decode workload."""
    g = torch.Generator(device=device).manual_seed(w.seed)
    cap = capacity or w.length
    k, v = token_cache(w.batch, w.kv_heads, w.length, cap, g, device, w.dist)
    q = _normal_bf16((w.batch, w.queries, w.q_heads, HEAD_DIM), g, device)
    out = dict(k_tok=k, v_tok=v, q=q, pooler=pooler_matrix(w.seed).to(device))
    if w.dist == "needles" and w.needles:
        out["needle_positions"] = plant_needles(k, q, w.length, w.needles, w.kv_heads, w.q_heads, g)
    return out


def prefill_inputs(w: Workload, device="cpu") -> dict:
    """Cache of ``length`` tokens (capacity length + chunk), the chunk's K/V and its queries."""
    g = torch.Generator(device=device).manual_seed(w.seed)
    k, v = token_cache(w.batch, w.kv_heads, w.length, w.capacity, g, device, w.dist)
    k_new = _normal_bf16((w.batch, w.chunk, w.kv_heads, HEAD_DIM), g, device)
    v_new = _normal_bf16((w.batch, w.chunk, w.kv_heads, HEAD_DIM), g, device)
    q = _normal_bf16((w.batch, w.chunk, w.q_heads, HEAD_DIM), g, device)
    return dict(k_tok=k, v_tok=v, k_new=k_new, v_new=v_new, q=q, pooler=pooler_matrix(w.seed).to(device))


def random_case(batch, length, kv_heads, q_heads, queries, seed, capacity=None, chunk=0, device="cpu") -> dict:
    """A small N(0, 1) case of any shape, for parity tests and edge cases."""
    g = torch.Generator(device=device).manual_seed(seed)
    cap = capacity or (length + chunk)
    k, v = token_cache(batch, kv_heads, length, cap, g, device)
    q = _normal_bf16((batch, chunk if chunk else queries, q_heads, HEAD_DIM), g, device)
    out = dict(k_tok=k, v_tok=v, q=q, pooler=pooler_matrix(seed).to(device))
    if chunk:
        out["k_new"] = _normal_bf16((batch, chunk, kv_heads, HEAD_DIM), g, device)
        out["v_new"] = _normal_bf16((batch, chunk, kv_heads, HEAD_DIM), g, device)
    return out


def bf16_bits(t: torch.Tensor):
    """Raw bf16 bit patterns of a tensor as a numpy uint16 array (CPU copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
