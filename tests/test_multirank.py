"""Multi-rank host logic on CPU with world size 2 over gloo: the benchmark's
max-over-ranks timing and weak-scaling aggregate, and the decode-context-
parallel exchange the pages describe (each rank attends its own slice of the
KV pages; the partial results are gathered and merged by log-sum-exp)."""
import math
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
        sys.path.insert(0, root)
        import bench
        from oracle import qsa_ref as ref
        out = {}
        # timing: every rank reports its own time, the job time is the max
        ms = bench.max_over_ranks(10.0 + rank, world)
        out["ms"] = ms
        out["rate"] = bench.weak_scaling_rate(128, world, 5, ms)
        out["seed"] = bench.rank_seed(0, rank)
        # DCP: identical inputs on every rank (seed 0), rank r owns split r
        rng = np.random.default_rng(0)
        L, Hq, Hkv, D, P = 700, 8, 2, 16, 16
        qv = rng.standard_normal((Hq, D))
        K = rng.standard_normal((L, Hkv, D))
        V = rng.standard_normal((L, Hkv, D))
        toks = np.sort(rng.choice(L, 300, replace=False))
        o_part, lse_part = ref.split_attention(qv, K, V, toks, 0.25, L, P, world)
        # the library's exchange: this rank's split in, every rank's out
        from sparse_attention_decode_compress_b200.dcp import dcp_exchange
        o_loc = torch.from_numpy(o_part[rank][None].copy())
        l_loc = torch.from_numpy(lse_part[rank][None].copy())
        o_all = torch.empty((world,) + o_loc.shape[1:], dtype=o_loc.dtype)
        l_all = torch.empty((world,) + l_loc.shape[1:], dtype=l_loc.dtype)
        dcp_exchange(o_loc, l_loc, o_all, l_all)
        o_m, lse_m = ref.lse_merge(o_all.numpy(), l_all.numpy())
        o_u, lse_u = ref.attention(qv, K, V, toks, 0.25)
        out["dcp_err"] = float(max(np.abs(o_m - o_u).max(), np.abs(lse_m - lse_u).max()))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_dcp_merge():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r]["ms"] == 11.0                  # max over ranks
        assert math.isclose(res[r]["rate"], 2 * 128 * 5 / 0.011)
        assert res[r]["dcp_err"] < 1e-12             # merged slices == unsplit attention
    assert {res[0]["seed"], res[1]["seed"]} == {0, 1}  # independent replicas
