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


# ----------------------------------------------------------------- one sequence over ranks

class _OracleRows:
    """prefill_rows' compute on the FP64 oracle (one sequence, whole keys)."""

    def __init__(self, wl, d):
        self.wl, self.d = wl, d

    def prefill_block(self, start, count):
        from oracle import dsa_oracle as O
        wl, d = self.wl, self.d
        res = {}
        for t in range(start, start + count):
            sc, idx, o, lse = O.dsa_row(d["qd"][t], d["w"][t], d["kd"], d["q"][t], d["kv"],
                                         O.query_pos(wl.T, wl.S, t), wl.k, wl.d_v, O.default_tau(wl.d_k))
            res[t] = (idx, o, lse, sc.shape[0])      # sc.shape[0] = indexer pairs of row t
        return res


class _OracleKeySplit:
    """KeySplitDecode's compute on the FP64 oracle: this rank holds keys
    [s0, s0 + cnt) of every sequence."""

    def __init__(self, wl, inp):
        from oracle import dsa_oracle as O
        self.O, self.wl = O, wl
        self.d = [O.from_inputs(inp, b) for b in range(wl.B)]

    def select(self, s0, cnt):
        O, wl = self.O, self.wl
        cs = np.full((wl.B, wl.k), -np.inf)
        ci = np.full((wl.B, wl.k), -1, np.int64)
        for b, d in enumerate(self.d):
            sc = O.indexer_row(d["qd"][0], d["w"][0], d["kd"][s0:s0 + cnt], cnt - 1)   # all keys of the range
            loc = O.topk_row(sc, wl.k)
            ok = loc >= 0
            ci[b, ok] = loc[ok] + s0
            cs[b, ok] = sc[loc[ok]]
        return torch.from_numpy(cs), torch.from_numpy(ci)

    def merge(self, cs_all, ci_all, s0, cnt):
        gidx = np.stack([self.O.topk_merge(cs_all[:, b].numpy(), ci_all[:, b].numpy(), self.wl.k)
                         for b in range(self.wl.B)])
        lidx = np.where((gidx >= s0) & (gidx < s0 + cnt), gidx - s0, -1)
        return torch.from_numpy(gidx), torch.from_numpy(lidx)

    def attend(self, idx_local, s0, cnt):
        O, wl = self.O, self.wl
        os_, ls = [], []
        for b, d in enumerate(self.d):
            sel = idx_local[b].numpy()
            if (sel >= 0).any():
                o, lse = O.sparse_attention_row(d["q"][0], d["kv"][s0:s0 + cnt], sel, wl.d_v,
                                                O.default_tau(wl.d_k))
            else:
                o, lse = np.zeros((wl.H, wl.d_v)), np.full(wl.H, -np.inf)
            os_.append(o)
            ls.append(lse)
        return torch.from_numpy(np.stack(os_)), torch.from_numpy(np.stack(ls))

    def combine(self, o_all, lse_all):
        res = [self.O.combine_partials(o_all[:, b].numpy(), lse_all[:, b].numpy()) for b in range(self.wl.B)]
        return np.stack([r[0] for r in res]), np.stack([r[1] for r in res])


_PREFILL_WL = dict(name="dist_prefill", B=1, T=384, S=384, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=48, q_block=384,
                   seed=22, needles=4)
_SPLIT_WL = dict(name="dist_keysplit", B=2, T=1, S=700, H_I=8, D_I=32, H=8, d_k=80, d_v=64, k=40, q_block=1,
                 seed=23, needles=6)


def _sequence_worker(rank, world, port, out_q):
    import torch.distributed as dist

    from long_context_05_b200.inputs import Workload, make_inputs
    from long_context_05_b200.parallel import KeySplitDecode, prefill_rows, zigzag_blocks
    from oracle import dsa_oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # zig-zag rows of one prefill
        wl = Workload(**_PREFILL_WL)
        d = O.from_inputs(make_inputs(wl, "cpu"))
        blocks = zigzag_blocks(wl.T, world, rank)
        rows = {}
        for _, _, res in prefill_rows(_OracleRows(wl, d), blocks):
            rows.update(res)
        gathered_rows = [None] * world
        dist.all_gather_object(gathered_rows, (blocks, rows))
        # key-split decode of two sequences
        ws = Workload(**_SPLIT_WL)
        inp = make_inputs(ws, "cpu")
        inp.pop("needle_pos", None)

        def all_gather(t):
            parts = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(parts, t.contiguous())
            return torch.stack(parts)

        o, lse, idx = KeySplitDecode(ws.S, world, rank).run(_OracleKeySplit(ws, inp), all_gather)
        if rank == 0:
            out_q.put((gathered_rows, (o, lse, idx.numpy())))
    finally:
        dist.destroy_process_group()


def test_zigzag_blocks_cover_rows_and_balance_pairs():
    from long_context_05_b200.parallel import indexer_pairs, zigzag_blocks
    for T in (7, 100, 512, 131072):
        for world in (1, 2, 3, 4, 8):
            seen = []
            pairs = []
            for r in range(world):
                bl = zigzag_blocks(T, world, r)
                for s, c in bl:
                    seen.extend(range(s, s + c))
                pairs.append(indexer_pairs(bl, T, T))
            assert sorted(seen) == list(range(T))
            assert sum(pairs) == T * (T + 1) // 2
            if T >= 64 * world:
                assert max(pairs) <= 1.05 * min(pairs), (T, world, pairs)


def test_one_sequence_over_two_gloo_ranks():
    """Rows of one prefill in zig-zag blocks and the keys of one decode step
    split over two gloo ranks, each rank computing with the oracle: the union
    of the rows and the merged decode equal the single-process oracle, and the
    ranks' indexer pairs agree within 5%."""
    from long_context_05_b200.inputs import Workload, make_inputs
    from oracle import dsa_oracle as O

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sequence_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    gathered_rows, (o, lse, idx) = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    # prefill rows
    wl = Workload(**_PREFILL_WL)
    d = O.from_inputs(make_inputs(wl, "cpu"))
    union = {}
    pairs = []
    for blocks, rows in gathered_rows:
        assert not set(rows) & set(union)
        union.update(rows)
        pairs.append(sum(v[3] for v in rows.values()))
    assert sorted(union) == list(range(wl.T))
    assert max(pairs) <= 1.05 * min(pairs), pairs
    for t in range(wl.T):
        sc, ix, oo, ll = O.dsa_row(d["qd"][t], d["w"][t], d["kd"], d["q"][t], d["kv"], t, wl.k, wl.d_v,
                                   O.default_tau(wl.d_k))
        assert np.array_equal(union[t][0], ix) and np.array_equal(union[t][1], oo)
    # key-split decode
    ws = Workload(**_SPLIT_WL)
    inp = make_inputs(ws, "cpu")
    for b in range(ws.B):
        db = O.from_inputs(inp, b)
        sc, ix, oo, ll = O.dsa_row(db["qd"][0], db["w"][0], db["kd"], db["q"][0], db["kv"], ws.S - 1, ws.k,
                                   ws.d_v, O.default_tau(ws.d_k))
        assert sorted(idx[b][idx[b] >= 0].tolist()) == sorted(ix[ix >= 0].tolist())
        assert np.max(np.abs(o[b] - oo)) < 1e-12 and np.max(np.abs(lse[b] - ll)) < 1e-12
