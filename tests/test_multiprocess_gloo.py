"""The multi-GPU path on CPU: world_size-2 gloo ranks.

The method shards with no exchange: by sequence (every rank runs its own replica and only
the timing is reduced, maximum over ranks) or by KV head (every rank builds and attends its
block of KV heads of every sequence; the blocks' outputs are joined only on request).  These
tests run that host-side logic as gloo processes on 127.0.0.1, with the oracle standing in
for the library where results are compared.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    local = [0.25, 0.5][rank]  # rank 1 is the slower replica
    value, slowest = bench.job_throughput(units_per_rank_step=4, steps=10, local_seconds=local, world=world,
                                          dist_on=True)
    m = bench.max_over_ranks(float(rank + 1), True)
    dist.barrier()
    out[rank] = (value, slowest, m)
    dist.destroy_process_group()


def test_replicas_report_the_slowest_rank_and_the_whole_job():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        value, slowest, m = res[rank]
        assert slowest == 0.5 and m == 2.0
        assert value == pytest.approx(world * 4 * 10 / 0.5)


def test_single_process_is_identity():
    import bench

    value, slowest = bench.job_throughput(4, 10, 0.5, world=1, dist_on=False)
    assert slowest == 0.5 and value == pytest.approx(80.0)


def _shard_worker(rank, world, port, out):
    """One rank of a KV-head-sharded decode: its block of heads, the oracle standing in for
    the library (no GPU here), the blocks joined by the all-gather helper."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import recsa_inputs as I
    from hierarchical_sparse_attention_build_b200 import sharding as S
    from oracle import recsa_oracle as O

    B, L, hkv, G, b, k = 2, 300, 3, 4, 4, 2  # 3 KV heads over 2 ranks: blocks of 2 and 1
    inp = I.random_case(B, L, hkv, hkv * G, 2, seed=11)
    h0, h1 = S.kv_head_range(hkv, rank, world)
    kc, vc = S.shard_cache(inp["k_tok"], h0, h1), S.shard_cache(inp["v_tok"], h0, h1)
    q = S.shard_queries(inp["q"], G, h0, h1)
    trees = O.build_all(I.bf16_bits(kc), I.bf16_bits(vc), inp["pooler"].double().numpy(), b, L)
    block = O.decode_all(trees, I.bf16_bits(q), k)
    full = S.gather_outputs(torch.from_numpy(block), hkv, G)
    out[rank] = (h0, h1, full.numpy())
    dist.destroy_process_group()


def test_kv_head_sharding_joins_to_the_unsharded_decode():
    import recsa_inputs as I
    from oracle import recsa_oracle as O

    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert (res[0][0], res[0][1], res[1][0], res[1][1]) == (0, 2, 2, 3)
    B, L, hkv, G, b, k = 2, 300, 3, 4, 4, 2
    inp = I.random_case(B, L, hkv, hkv * G, 2, seed=11)
    trees = O.build_all(I.bf16_bits(inp["k_tok"]), I.bf16_bits(inp["v_tok"]), inp["pooler"].double().numpy(), b, L)
    want = O.decode_all(trees, I.bf16_bits(inp["q"]), k)
    for rank in range(world):
        assert res[rank][2].shape == want.shape
        assert np.array_equal(res[rank][2], want)  # heads are independent: the same fp64 results


@pytest.mark.parametrize("hkv,world", [(8, 1), (8, 2), (8, 3), (8, 8), (3, 4), (1, 2)])
def test_kv_head_ranges_cover_every_head_once(hkv, world):
    from hierarchical_sparse_attention_build_b200 import sharding as S

    got = [S.kv_head_range(hkv, r, world) for r in range(world)]
    assert got[0][0] == 0 and got[-1][1] == hkv
    for (a0, a1), (b0, b1) in zip(got, got[1:]):
        assert a1 == b0
    sizes = [h1 - h0 for h0, h1 in got]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == hkv


def test_shard_params_keep_everything_but_the_head_counts():
    import hierarchical_sparse_attention_build_b200 as R
    from hierarchical_sparse_attention_build_b200 import sharding as S

    p = R.params(num_kv_heads=8, num_q_heads=32, branching=16, top_k=8)
    q = S.shard_params(p, 1, 3)
    assert (q.num_kv_heads, q.num_q_heads) == (3, 12)
    for name in ("head_dim", "branching", "top_k", "rope_base", "softmax_scale"):
        assert getattr(q, name) == getattr(p, name)
