"""World-size-2 gloo checks of the multi-process path (CPU only).

Each rank takes its shard of a decode batch, runs the FP64 oracle on it, and
the gathered results must equal the single-process run of the whole batch;
the max-over-ranks timing helper must return the largest rank's value.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from long_context_05_b200.parallel import max_over_ranks, rank_seed, shard_batch


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    import torch.distributed as dist

    from long_context_05_b200.inputs import Workload, make_inputs
    from oracle import dsa_oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = Workload("dist_decode", B=5, T=1, S=300, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=32, q_block=1,
                      seed=21, needles=4)
        inp = make_inputs(wl, "cpu")
        first, count = shard_batch(wl.B, world, rank)
        outs = {}
        for b in range(first, first + count):
            d = O.from_inputs(inp, b)
            sc = O.indexer_row(d["qd"][0], d["w"][0], d["kd"], O.query_pos(1, wl.S, 0))
            idx = O.topk_row(sc, wl.k)
            o, lse = O.sparse_attention_row(d["q"][0], d["kv"], idx, wl.d_v, O.default_tau(wl.d_k))
            outs[b] = (idx, o, lse)
        gathered = [None] * world
        dist.all_gather_object(gathered, outs)
        mx = max_over_ranks(10.0 + rank)
        if rank == 0:
            out_q.put((gathered, mx))
    finally:
        dist.destroy_process_group()


def test_shard_batch_covers_once():
    for B in range(0, 40):
        for world in range(1, 9):
            seen = []
            for r in range(world):
                f, c = shard_batch(B, world, r)
                seen.extend(range(f, f + c))
            assert seen == list(range(B))
    assert rank_seed(1004, 3) == 1007


def test_two_rank_gloo_matches_single_process():
    from long_context_05_b200.inputs import Workload, make_inputs
    from oracle import dsa_oracle as O

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    gathered, mx = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert mx == 11.0
    merged = {}
    for part in gathered:
        merged.update(part)
    wl = Workload("dist_decode", B=5, T=1, S=300, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=32, q_block=1,
                  seed=21, needles=4)
    inp = make_inputs(wl, "cpu")
    assert sorted(merged) == list(range(wl.B))
    for b in range(wl.B):
        d = O.from_inputs(inp, b)
        sc = O.indexer_row(d["qd"][0], d["w"][0], d["kd"], O.query_pos(1, wl.S, 0))
        idx = O.topk_row(sc, wl.k)
        o, lse = O.sparse_attention_row(d["q"][0], d["kv"], idx, wl.d_v, O.default_tau(wl.d_k))
        assert np.array_equal(merged[b][0], idx)
        assert np.array_equal(merged[b][1], o) and np.array_equal(merged[b][2], lse)
