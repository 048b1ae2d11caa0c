"""Seeded synthetic inputs for the DSA hot path.

This module only draws random tensors and packs them into the storage types the
path consumes (FP8 e4m3 bytes with FP32 scales, BF16).  It holds none of the
method's arithmetic: no indexer score, no selection, no attention.  The oracle
and the CUDA path both read what it produces, and nothing else is shared
between them.

Workloads follow the shapes the pages talk about (128K context, k = 2048 per
query, an FP8 indexer with few heads, an MLA-style 576-wide key with a 512-wide
value shared by all heads):

* ouchyi thread on DeepSeek Sparse Attention (web3.ouchyi.pink), "Nasil
  calisiyor" paragraph: indexer in FP8 with few heads, 2,048 tokens kept per
  query whatever the context, the expensive attention over that subset only,
  128K context as the headline length.
* tenelement.pl, "DeepSeek V3.2-Exp Cuts Long-Context Costs ...", section
  "Architektura DeepSeek V3.2-Exp: Od MoE do DSA": FP8 indexer, few heads,
  ReLU, top-k = 2048, MLA with MQA-style KV sharing in decode.

Structure planted so that the selection is not trivial (the pages do not
describe input distributions; sider.ai blog, "Uyarilar" section, only asks for
realistic relevance distributions):

* decode workloads: per sequence, ``needles`` key positions whose indexer key
  has cosine 0.5 with u = unit(sum_j w_j q_I,j), and whose attention latent has
  cosine 0.5 with unit(mean_h q_h[:d_v]);
* prefill workloads: one random direction u per sequence; needle keys carry u
  at cosine 0.5 and every query head carries sign(w) * u at cosine 0.5
  (attention: a second direction in the latent part);
* long prefill: a local-window component p(s), a linear interpolation between
  i.i.d. unit vectors placed every ``local_window`` positions; queries add
  p(t), keys add 0.5 p(s), scaled to the norm of a standard normal vector, so
  keys within about a window of the query are positively correlated with it.

FP8 packing: per (token, head) vector for q_I and per token for k_I,
scale = absmax / 448 and byte = RNE(clamp(x / scale, +-448)) in e4m3.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

E4M3_MAX = 448.0


@dataclass(frozen=True)
class Workload:
    """Shape and distribution of one synthetic DSA workload.

    Query token t of a sequence sits at position (S - T) + t, so a prefill with
    T == S is plain causal self-attention and a decode with T == 1 has its
    single query at S - 1 (it sees all S keys).
    """

    name: str
    B: int          # sequences
    T: int          # query tokens per sequence
    S: int          # keys per sequence
    H_I: int        # indexer heads
    D_I: int        # indexer head dim
    H: int          # attention heads
    d_k: int        # key dim (latent + rope)
    d_v: int        # value dim (the latent)
    k: int          # keys kept per query
    q_block: int    # prefill query block for the score tile
    seed: int
    int_mode: bool = False   # integer-valued FP8 indexer inputs, power-of-two w
    needles: int = 0
    local_window: int = 0

    @property
    def decode(self) -> bool:
        return self.T == 1 and self.S > 1

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # tiny prefill, integer indexer inputs: scores are exact in FP32 and FP64
    "tiny_prefill_256": Workload("tiny_prefill_256", B=1, T=256, S=256, H_I=4, D_I=32,
                                 H=8, d_k=80, d_v=64, k=64, q_block=256, seed=1000,
                                 int_mode=True),
    "decode_32k_b32": Workload("decode_32k_b32", B=32, T=1, S=32768, H_I=64, D_I=128,
                               H=128, d_k=576, d_v=512, k=2048, q_block=1, seed=1001,
                               needles=64),
    "prefill_8k": Workload("prefill_8k", B=1, T=8192, S=8192, H_I=64, D_I=128,
                           H=128, d_k=576, d_v=512, k=2048, q_block=2048, seed=1002,
                           needles=64),
    "decode_128k_b8": Workload("decode_128k_b8", B=8, T=1, S=131072, H_I=64, D_I=128,
                               H=128, d_k=576, d_v=512, k=2048, q_block=1, seed=1003,
                               needles=64),
    "prefill_128k": Workload("prefill_128k", B=1, T=131072, S=131072, H_I=64, D_I=128,
                             H=128, d_k=576, d_v=512, k=2048, q_block=4096, seed=1004,
                             needles=64, local_window=512),
    # the last 512 queries of a 128K prefill (a chunked-prefill step): full
    # 128K score rows at a size small enough for a profiler capture
    "prefill_chunk_128k": Workload("prefill_chunk_128k", B=1, T=512, S=131072, H_I=64, D_I=128,
                                   H=128, d_k=576, d_v=512, k=2048, q_block=512, seed=1005,
                                   needles=64, local_window=512),
}

# rows generated per random draw; fixed so the stream does not depend on memory
_CHUNK_TOKENS = 2048


def _unit(x: torch.Tensor, dim: int = -1) -> torch.Tensor:
    return x / x.norm(dim=dim, keepdim=True).clamp_min(1e-30)


def _cos_half(u: torch.Tensor, g: torch.Tensor) -> torch.Tensor:
    """Vector of norm |g| with cosine 0.5 to the unit vector(s) u.

    u: [..., D] unit, g: [..., D] random.  Returns |g| (0.5 u + sqrt(.75) n),
    n the unit part of g orthogonal to u.
    """
    gn = g.norm(dim=-1, keepdim=True)
    perp = g - (g * u).sum(-1, keepdim=True) * u
    return gn * (0.5 * u + math.sqrt(0.75) * _unit(perp))


def quantize_e4m3(x: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """Pack x [..., D] (float32) into e4m3 bytes with one FP32 scale per vector."""
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    q = (x / scale.unsqueeze(-1)).clamp(-E4M3_MAX, E4M3_MAX)
    return q.to(torch.float8_e4m3fn).view(torch.uint8), scale.float()


def _local_component(pos: torch.Tensor, anchors: torch.Tensor, window: int) -> torch.Tensor:
    """p(pos): linear interpolation between unit anchors placed at window centres."""
    c = (pos.double() - window / 2) / window
    i0 = c.floor().clamp(0, anchors.shape[0] - 1).long()
    i1 = (i0 + 1).clamp(max=anchors.shape[0] - 1)
    f = (c - i0.double()).clamp(0, 1).float().unsqueeze(-1)
    return _unit((1 - f) * anchors[i0] + f * anchors[i1])


def make_inputs(wl: Workload, device="cpu") -> dict:
    """Draw one batch of inputs for ``wl`` on ``device``.

    Returns a dict of tensors (all contiguous):
      q_I     uint8   [B, T, H_I, D_I]  e4m3 bytes
      q_scale float32 [B, T, H_I]
      w       float32 [B, T, H_I]
      k_I     uint8   [B, S, D_I]       e4m3 bytes
      k_scale float32 [B, S]
      q       bfloat16 [B, T, H, d_k]
      kv      bfloat16 [B, S, d_k]      (V = kv[..., :d_v])
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(wl.seed)
    B, T, S, HI, DI, H, dk, dv = wl.B, wl.T, wl.S, wl.H_I, wl.D_I, wl.H, wl.d_k, wl.d_v
    f32 = dict(device=dev, dtype=torch.float32)

    out = {
        "q_I": torch.empty(B, T, HI, DI, dtype=torch.uint8, device=dev),
        "q_scale": torch.empty(B, T, HI, **f32),
        "w": torch.empty(B, T, HI, **f32),
        "k_I": torch.empty(B, S, DI, dtype=torch.uint8, device=dev),
        "k_scale": torch.empty(B, S, **f32),
        "q": torch.empty(B, T, H, dk, dtype=torch.bfloat16, device=dev),
        "kv": torch.empty(B, S, dk, dtype=torch.bfloat16, device=dev),
    }

    if wl.int_mode:
        # integers in [-8, 8] are exact in e4m3; w = +-2^e, e in {-2..2}
        out["q_I"].copy_(torch.randint(-8, 9, (B, T, HI, DI), generator=g, device=dev)
                         .float().to(torch.float8_e4m3fn).view(torch.uint8))
        out["k_I"].copy_(torch.randint(-8, 9, (B, S, DI), generator=g, device=dev)
                         .float().to(torch.float8_e4m3fn).view(torch.uint8))
        out["q_scale"].fill_(1.0)
        out["k_scale"].fill_(1.0)
        e = torch.randint(-2, 3, (B, T, HI), generator=g, device=dev).float()
        sgn = torch.randint(0, 2, (B, T, HI), generator=g, device=dev).float() * 2 - 1
        out["w"].copy_(sgn * torch.exp2(e))
        sd = 1.0 / math.sqrt(dk)
        out["q"].copy_((torch.randn(B, T, H, dk, generator=g, **f32) * sd).bfloat16())
        out["kv"].copy_((torch.randn(B, S, dk, generator=g, **f32) * sd).bfloat16())
        return out

    # per-sequence directions for planted structure
    u_idx = _unit(torch.randn(B, DI, generator=g, **f32))
    u_att = _unit(torch.randn(B, dv, generator=g, **f32))
    nwin = (S + wl.local_window - 1) // wl.local_window + 1 if wl.local_window else 0
    if nwin:
        anchors_i = _unit(torch.randn(B, nwin, DI, generator=g, **f32))
        anchors_a = _unit(torch.randn(B, nwin, dv, generator=g, **f32))

    for b in range(B):
        out["w"][b].copy_(torch.randn(T, HI, generator=g, **f32) / 8.0)
        # queries, in chunks of tokens
        for t0 in range(0, T, _CHUNK_TOKENS):
            t1 = min(T, t0 + _CHUNK_TOKENS)
            n = t1 - t0
            qi = torch.randn(n, HI, DI, generator=g, **f32)
            qa = torch.randn(n, H, dk, generator=g, **f32)
            wsgn = torch.sign(out["w"][b, t0:t1]).unsqueeze(-1)  # [n, HI, 1]
            if wl.needles and not wl.decode:
                qi = _cos_half((wsgn * u_idx[b]).expand(n, HI, DI).contiguous(), qi)
                lat = _cos_half(u_att[b].expand(n, H, dv).contiguous(), qa[..., :dv].contiguous())
                qa[..., :dv] = lat
            if nwin:
                pos = torch.arange(S - T + t0, S - T + t1, device=dev)
                pi = _local_component(pos, anchors_i[b], wl.local_window)      # [n, DI]
                pa = _local_component(pos, anchors_a[b], wl.local_window)      # [n, dv]
                qi = qi + math.sqrt(DI) * wsgn * pi.unsqueeze(1)
                qa[..., :dv] += math.sqrt(dv) * pa.unsqueeze(1)
            q8, qs = quantize_e4m3(qi)
            out["q_I"][b, t0:t1].copy_(q8)
            out["q_scale"][b, t0:t1].copy_(qs)
            out["q"][b, t0:t1].copy_(qa.bfloat16())
        # keys
        for s0 in range(0, S, _CHUNK_TOKENS):
            s1 = min(S, s0 + _CHUNK_TOKENS)
            n = s1 - s0
            ki = torch.randn(n, DI, generator=g, **f32)
            ka = torch.randn(n, dk, generator=g, **f32)
            if nwin:
                pos = torch.arange(s0, s1, device=dev)
                ki = ki + 0.5 * math.sqrt(DI) * _local_component(pos, anchors_i[b], wl.local_window)
                ka[:, :dv] += 0.5 * math.sqrt(dv) * _local_component(pos, anchors_a[b], wl.local_window)
            k8, ks = quantize_e4m3(ki)
            out["k_I"][b, s0:s1].copy_(k8)
            out["k_scale"][b, s0:s1].copy_(ks)
            out["kv"][b, s0:s1].copy_(ka.bfloat16())
        if wl.needles:
            npos = torch.randperm(S, generator=g, device=dev)[: wl.needles]
            gi = torch.randn(wl.needles, DI, generator=g, **f32)
            ga = torch.randn(wl.needles, dv, generator=g, **f32)
            if wl.decode:
                # u = unit(sum_j w_j q_I,j) of the single query, from the packed values
                qf = out["q_I"][b, -1].view(torch.float8_e4m3fn).float() * out["q_scale"][b, -1].unsqueeze(-1)
                ui = _unit((out["w"][b, -1].unsqueeze(-1) * qf).sum(0))
                ua = _unit(out["q"][b, -1, :, :dv].float().mean(0))
            else:
                ui, ua = u_idx[b], u_att[b]
            k8, ks = quantize_e4m3(_cos_half(ui.expand(wl.needles, DI).contiguous(), gi))
            out["k_I"][b, npos] = k8
            out["k_scale"][b, npos] = ks
            kvn = out["kv"][b, npos].float()
            kvn[:, :dv] = _cos_half(ua.expand(wl.needles, dv).contiguous(), ga)
            out["kv"][b, npos] = kvn.bfloat16()
            out.setdefault("needle_pos", torch.empty(B, wl.needles, dtype=torch.long, device=dev))
            out["needle_pos"][b] = npos
    return out



def to_paged(inp: dict, wl: Workload, page_size: int, seed: int):
    """Scatter the key-side arrays of ``inp`` (k_I, k_scale, kv and v when
    present) into page pools, pages in a random order.

    Sequence b's page p (tokens p * page_size .. + page_size - 1) goes to pool
    page table[b, p]; the pool has two spare pages that no sequence maps, and
    the table one extra column of -1 (an unmapped page past each sequence's
    last).  Returns (inputs with the pools in place of the key-side arrays,
    int32 table [B, ppseq + 1] on the inputs' device, number of pool pages).
    """
    import numpy as np

    ppseq = (wl.S + page_size - 1) // page_size
    num_pages = wl.B * ppseq + 2
    perm = np.random.default_rng(seed).permutation(num_pages)[: wl.B * ppseq].reshape(wl.B, ppseq)
    table = np.full((wl.B, ppseq + 1), -1, np.int32)
    table[:, :ppseq] = perm
    dev = inp["kv"].device
    # pool row of every (sequence, token): page base + offset in the page
    rows = (torch.from_numpy(perm).to(dev, torch.int64).unsqueeze(-1) * page_size
            + torch.arange(page_size, device=dev)).reshape(wl.B, -1)[:, : wl.S].reshape(-1)
    out = dict(inp)
    for name in ("k_I", "k_scale", "kv", "v"):
        if name not in inp:
            continue
        x = inp[name]
        pool = torch.zeros((num_pages * page_size,) + tuple(x.shape[2:]), dtype=x.dtype, device=dev)
        pool[rows] = x.reshape((wl.B * wl.S,) + tuple(x.shape[2:]))
        out[name] = pool
    return out, torch.from_numpy(table).to(dev), num_pages
