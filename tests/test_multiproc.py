"""Host logic of the multi-rank benchmark on CPU: two `gloo` ranks.

Layers of a model are independent compression problems (the budget is per
layer), so ranks shard them with no collective on the data path; the only
exchange is the max-over-ranks reduction of the step time.  These tests run
that host logic as two processes on the CPU, with the oracle standing in for
the per-rank work.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from kv_cache_compression_anchorkv_b200.synthetic import CacheSpec, make_layer
from oracle import anchorkv_oracle as O


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = bench.rank_spec(CacheSpec(4, 1, 4, 300, n_dirs=8, seed=3), rank, layers=2)
        # per-rank work: the oracle's compress of this rank's first layer
        K, V, Q = make_layer(spec, 0)
        p = O.Params(n_tokens=spec.n_tokens, n_kv_heads=1, n_q_heads=4, theta=0.3, dtype="bf16", seed=spec.seed)
        res = O.compress_layer(K.double().numpy(), V.double().numpy(), Q.double().numpy(), p)
        n_anchor = int(len(res["anchor_pos"][0]))
        ms = bench.reduce_max(10.0 + rank, world, "cpu")           # rank 1 is the slower one
        value = bench.job_value(spec.n_tokens * spec.n_layers * spec.n_kv_heads, world, ms)
        # replayed-graph time: both ranks timed, then rank 1's capture failed
        g_ok = bench.graph_us_over_ranks(4.0 + rank, 2, world, "cpu")
        g_fail = bench.graph_us_over_ranks(4.0 if rank == 0 else None, 2, world, "cpu")
        out[rank] = (spec.seed, spec.n_layers, ms, value, n_anchor, float(K.float().sum()), g_ok, g_fail)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
        r0, r1 = out[0], out[1]
    # independent caches per rank, layers capped
    assert (r0[0], r1[0]) == (3, 4) and r0[1] == r1[1] == 2
    assert r0[5] != r1[5]
    # both ranks see the slowest rank's time and the same whole-job value
    assert r0[2] == r1[2] == 11.0
    assert r0[3] == r1[3] == pytest.approx(300 * 2 * 1 * 2 / (11.0 / 1e3) / 1e6)
    assert r0[4] == r1[4] == O.layout(O.Params(n_tokens=300, n_kv_heads=1, n_q_heads=4, theta=0.3))["k"]
    # the graph time is the slowest rank's, and a failed capture anywhere is reported everywhere
    assert r0[6] == r1[6] == pytest.approx(1e3 * 5.0 / 2)
    assert r0[7] is None and r1[7] is None


def _compress_layers(spec, ids):
    """Oracle layouts (bytes) of layers `ids` of one seeded cache."""
    res = {}
    for l in ids:
        K, V, Q = make_layer(spec, l)
        p = O.Params(n_tokens=spec.n_tokens, n_kv_heads=spec.n_kv_heads, n_q_heads=spec.n_q_heads, theta=0.3,
                     dtype="bf16", seed=spec.seed, layer=l)
        res[l] = O.compress_layer(K.double().numpy(), V.double().numpy(), Q.double().numpy(), p)["bytes"]
    return res


def _layer_shard_worker(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = bench.rank_spec(CacheSpec(5, 1, 4, 260, n_dirs=8, seed=9), rank, shard="layers")
        ids = bench.rank_layers(spec.n_layers, rank, world, shard="layers")
        out[rank] = (spec.seed, ids, _compress_layers(spec, ids))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_one_model_by_layer():
    """Layer sharding: rank r takes layers l = r (mod 2) of the same seeded
    model; together the ranks cover every layer once, and each layout equals
    the one a single rank computes for that layer, byte for byte (review,
    Referee "Summary": the residual budget is per layer, so layers are
    independent problems)."""
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_layer_shard_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == 9                       # one model: the same seed everywhere
    assert r0[1] == [0, 2, 4] and r1[1] == [1, 3]
    assert sorted(r0[1] + r1[1]) == list(range(5))
    whole = _compress_layers(CacheSpec(5, 1, 4, 260, n_dirs=8, seed=9), range(5))
    for part in (r0[2], r1[2]):
        for l, b in part.items():
            assert np.array_equal(b, whole[l]), l
    assert bench.rank_layers(5, 0, 1, shard="layers") == list(range(5))
    assert bench.rank_layers(5, 1, 2, shard="replicas") == list(range(5))


def test_single_rank_reduce_is_identity():
    assert bench.reduce_max(7.5, 1, "cpu") == 7.5
    assert bench.job_value(1000, 1, 1.0) == pytest.approx(1.0)
    assert bench.graph_us_over_ranks(3.0, 3, 1, "cpu") == pytest.approx(1000.0)
    assert bench.graph_us_over_ranks(None, 3, 1, "cpu") is None
