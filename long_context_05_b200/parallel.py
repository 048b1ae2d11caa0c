"""Multi-GPU plumbing for the DSA path: one process per GPU.

Three ways the path spreads over ranks:

1. Independent sequences per rank (weak scaling): every rank runs its own
   sequences; the only collectives are the barrier around a timed region and
   the max over ranks of the measured time.

2. One long prefill, its query rows split over ranks.  Query rows are
   independent given the keys; row t's indexer work is t + 1 pairs and its
   attention work min(t + 1, k), so contiguous row ranges would leave the
   last rank with most of the indexer work.  The rows are cut into 2P equal
   blocks and rank r takes blocks r and 2P - 1 - r (zig-zag): each rank pairs
   a short-prefix block with a long-prefix block, so indexer work per rank is
   equal up to one block's slope.  Every rank holds the whole key cache
   (replicated, or one all-gather of k_I and kv: 17 MB + 151 MB at 128K), and
   runs each block as a chunked prefill through dsa_forward (T = block rows,
   seqlens = block end, so pos(t) = block start + t).  No collective on the
   data path.

3. One long decode, its keys split over ranks.  Exact top-k decomposes over
   disjoint key ranges and exact softmax attention over disjoint key subsets
   (log-sum-exp merge), so each rank scores and selects within its own keys,
   the k (score, index) candidates per rank are all-gathered and merged into
   the global top-k, each rank attends over the selected keys it holds, and
   one all-gather of (O_r, LSE_r) plus a combine gives the output.

The orchestration below is written once against a small compute interface,
so the same host logic drives the CUDA library (NCCL all-gathers between
GPUs) and, in the CPU tests, the FP64 oracle (gloo all-gathers).
"""
from __future__ import annotations

import torch


def shard_batch(B: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous block of B items for `rank`: (first, count).  Ranks differ
    by at most one item; every item lands on exactly one rank."""
    base, extra = divmod(B, world)
    first = rank * base + min(rank, extra)
    return first, base + (1 if rank < extra else 0)


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic sequences (independent problems)."""
    return seed + rank


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank measurement (a no-op without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None) -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and torch.device(device).type == "cuda":
            dist.barrier(device_ids=[torch.device(device).index or 0])
        else:
            dist.barrier()


# ------------------------------------------------------------------ prefill rows

def zigzag_blocks(T: int, world: int, rank: int) -> list[tuple[int, int]]:
    """Query-row blocks (start, count) of `rank` when T causal rows are split
    over `world` ranks: 2 * world near-equal blocks, rank r takes blocks r and
    2 * world - 1 - r.  Together the ranks cover every row exactly once."""
    n = 2 * world
    out = []
    for i in (rank, n - 1 - rank):
        s, c = shard_batch(T, n, i)
        if c > 0:
            out.append((s, c))
    return out


def indexer_pairs(blocks, S: int, T: int) -> int:
    """Indexer pairs of the given row blocks of one sequence: sum of pos + 1."""
    off = S - T
    return sum(c * (2 * (off + s) + c + 1) // 2 for s, c in blocks)


def prefill_rows(compute, blocks):
    """Run the rows of `blocks` (one sequence, whole key cache on this rank):
    compute.prefill_block(start, count) -> per-block result.  Returns
    [(start, count, result)]."""
    return [(s, c, compute.prefill_block(s, c)) for s, c in blocks]


# ------------------------------------------------------------------ key-split decode

def key_shard(S: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous key range (first, count) of `rank` in a key-split decode."""
    return shard_batch(S, world, rank)


class KeySplitDecode:
    """One decode step of sequences whose keys are split over ranks.

    The steps are separate methods so that ranks can be driven in lockstep
    (one process per GPU with real all-gathers, or several emulated parts in
    one process).  `compute` supplies the arithmetic:

      select(s0, cnt)             -> (cand_scores [rows, k], cand_idx [rows, k])
                                     this range's top-k as (score, global index)
      merge(cs [P,rows,k], ci, s0, cnt) -> (idx [rows, k] global, idx_local [rows, k])
      attend(idx_local, s0, cnt)  -> (o [rows, H, d_v], lse [rows, H])
      combine(o [P,...], lse [P,...]) -> (o, lse)
    """

    def __init__(self, S: int, world: int, rank: int):
        self.s0, self.cnt = key_shard(S, world, rank)
        self.world = world

    def select(self, compute):
        return compute.select(self.s0, self.cnt)

    def merge(self, compute, cand_scores_all, cand_idx_all):
        return compute.merge(cand_scores_all, cand_idx_all, self.s0, self.cnt)

    def attend(self, compute, idx_local):
        return compute.attend(idx_local, self.s0, self.cnt)

    def run(self, compute, all_gather):
        """The whole step with `all_gather(tensor) -> [world, ...]` between
        the phases.  Returns (o, lse, global idx)."""
        cs, ci = self.select(compute)
        idx, idx_local = self.merge(compute, all_gather(cs), all_gather(ci))
        o, lse = self.attend(compute, idx_local)
        o, lse = compute.combine(all_gather(o), all_gather(lse))
        return o, lse, idx


def nccl_all_gather(t: torch.Tensor) -> torch.Tensor:
    """Stack every rank's copy of `t` (same shape) along a new leading dim."""
    import torch.distributed as dist
    out = torch.empty((dist.get_world_size(),) + tuple(t.shape), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, t.contiguous())
    return out


class DsaKeySplitCompute:
    """KeySplitDecode's arithmetic on this GPU through libdsa.so.

    The part holds, for B decode rows, its key range's caches (k_I, k_scale,
    kv: [B, cnt, ...]) and the queries of every row.  The scratch tensors are
    allocated once here, not per step."""

    def __init__(self, wl, inp_local: dict, S_total: int):
        from long_context_05_b200 import dsa
        self.dsa = dsa
        self.wl = wl                                  # the part's workload (S = its key count)
        self.inp = inp_local
        self.S_total = S_total
        self.shape = dsa.make_shape(wl)
        self.ws = dsa.alloc_workspace(self.shape)
        rows = wl.B * wl.T
        self.ld = (wl.S + 63) // 64 * 64
        self.scores = torch.empty(rows, self.ld, dtype=torch.float32, device="cuda")
        self.idx = torch.empty(wl.B, wl.T, wl.k, dtype=torch.int32, device="cuda")
        self.cs = torch.empty(rows, wl.k, dtype=torch.float32, device="cuda")
        self.ci = torch.empty(rows, wl.k, dtype=torch.int32, device="cuda")
        self.gidx = torch.empty(rows, wl.k, dtype=torch.int32, device="cuda")
        self.lidx = torch.empty(wl.B, wl.T, wl.k, dtype=torch.int32, device="cuda")
        self.o = torch.empty(wl.B, wl.T, wl.H, wl.d_v, dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty(wl.B, wl.T, wl.H, dtype=torch.float32, device="cuda")
        self.out = torch.empty_like(self.o)
        self.out_lse = torch.empty_like(self.lse)
        # the global shape (S = the whole sequence) for the merge and combine
        self.gshape = dsa.make_shape(wl.with_(S=S_total))
        self._topk_ws = self.ws[(rows * self.ld * 4 + 255) // 256 * 256:]

    def select(self, s0, cnt):
        d, i = self.dsa, self.inp
        d.indexer_scores(self.shape, i["q_I"], i["q_scale"], i["w"], i["k_I"], i["k_scale"], 0, self.wl.T,
                         self.scores)
        d.topk(self.shape, self.scores, 0, self.wl.T, self.idx, self.ws)
        d.topk_candidates(self.shape, self.scores, self.idx, s0, self.cs, self.ci)
        return self.cs, self.ci

    def merge(self, cs_all, ci_all, s0, cnt):
        self.dsa.topk_merge(self.gshape, cs_all.contiguous(), ci_all.contiguous(), self.gidx, s0, cnt, self.lidx)
        return self.gidx, self.lidx

    def attend(self, idx_local, s0, cnt):
        self.dsa.sparse_attn(self.shape, self.inp["q"], self.inp["kv"], idx_local, self.o, self.lse, self.ws)
        return self.o, self.lse

    def combine(self, o_all, lse_all):
        self.dsa.attn_combine(self.gshape, o_all.contiguous(), lse_all.contiguous(), self.out, self.out_lse)
        return self.out, self.out_lse


class DsaRowsCompute:
    """prefill_rows' arithmetic on this GPU: block [start, start + count) of
    one sequence (B = 1) as a chunked prefill through dsa_forward, with
    seqlens = start + count so that pos(t) = start + t, over the whole key
    cache (S = the sequence length)."""

    def __init__(self, wl, inp: dict):
        from long_context_05_b200 import dsa
        self.dsa, self.wl, self.inp = dsa, wl, inp
        assert wl.B == 1, "row sharding is per sequence"

    def prefill_block(self, start: int, count: int):
        d, wl, i = self.dsa, self.wl, self.inp
        blk = wl.with_(T=count, q_block=min(wl.q_block, count))
        sl = torch.tensor([start + count], dtype=torch.int32, device="cuda")
        shape = d.make_shape(blk, mode=d.DSA_PREFILL, seqlens=sl)
        rows = slice(start, start + count)
        part = {n: i[n][:, rows].contiguous() for n in ("q_I", "q_scale", "w", "q")}
        part.update({n: i[n] for n in ("k_I", "k_scale", "kv")})
        ws = d.alloc_workspace(shape)
        out = torch.empty(1, count, wl.H, wl.d_v, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(1, count, wl.H, dtype=torch.float32, device="cuda")
        idx = torch.empty(1, count, wl.k, dtype=torch.int32, device="cuda")
        d.forward(shape, part, out, lse, idx, ws)
        return out, lse, idx
