"""FP64 CPU oracle for the DeepSeek Sparse Attention (DSA) hot path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline / reference arm may import this module.  The product
path never calls it and shares no code with it: the CUDA library computes
everything itself, and this file reads nothing from it.

What DSA computes, as the pages describe it:

* ouchyi thread on DeepSeek Sparse Attention (web3.ouchyi.pink), "Nasil
  calisiyor" paragraph: a light "lightning indexer" scores, for every query,
  how much each context token matters; it has few heads and runs in FP8.  A
  selection step then keeps only the top-k key/value entries, 2,048 per query
  whatever the context length, and the expensive attention runs over that
  subset only.  Complexity goes from O(L^2) to O(L k) with k fixed.
* tenelement.pl, "DeepSeek V3.2-Exp Cuts Long-Context Costs with DeepSeek
  Sparse Attention (DSA) While Maintaining Benchmark Parity", section
  "Architektura DeepSeek V3.2-Exp: Od MoE do DSA": the indexer runs in FP8
  with few heads and computes logits for the context tokens through a ReLU;
  top-k selection keeps 2048 KV entries per query; the core attention sits on
  MLA, used in MQA form (one KV shared by all heads) in decoding.
* degnora.com, "DeepSeekV3, Farki Ne?", section "MLA - Multi-Latent
  Attention": keys and values come from one shared compressed latent, and only
  that latent is cached.

The pages give no formula for the indexer score.  The reading used here (the
plainest one that fits "few FP8 heads through ReLU, one key per token"):

    I[t, s] = sum_j w[t, j] * ReLU( q_I[t, j] . k_I[s] )

with q_I, k_I the dequantised indexer vectors (e4m3 byte times its FP32 scale)
and w a per-query, per-head weight.  The attention key of token s is the whole
cached row kv[s] (latent + rope part); the value is its first d_v columns (the
latent).  Query token t sits at position pos(t) = (S - T) + t and sees keys
s <= pos(t).

Everything here is plain NumPy in float64, from the dequantised inputs, one
query row at a time.  Matrix products use NumPy's matmul (a library primitive
allowed as a step); there is no blocking, fusion or reordering beyond the
definitions above.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------


def e4m3_decode(b) -> np.ndarray:
    """Decode OCP FP8 E4M3 bytes to float64.

    Written from the OCP 8-bit floating point definition (E4M3 variant):
    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
    encodes subnormals m/8 * 2^(1-7); S.1111.111 is NaN; there is no infinity,
    so S.1111.000 .. S.1111.110 are normal numbers up to 448.
    """
    b = np.asarray(b, dtype=np.uint8)
    sign = (b >> 7).astype(np.int64)
    e = ((b >> 3) & 0xF).astype(np.int64)
    m = (b & 0x7).astype(np.float64)
    sub = m / 8.0 * 2.0 ** (1 - 7)
    nor = (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64))
    val = np.where(e == 0, sub, nor)
    val = np.where(sign == 1, -val, val)
    return np.where((e == 15) & (m == 7), np.nan, val)


def bf16_decode(u) -> np.ndarray:
    """Decode bfloat16 bit patterns (uint16) to float64: the top half of an
    IEEE binary32, so bits << 16 reinterpreted as float32 is exact."""
    u = np.asarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dequant_indexer(q_I, q_scale, k_I, k_scale):
    """Dequantise the FP8 indexer operands: byte value times its FP32 scale.

    q_I [B, T, H_I, D_I] bytes, q_scale [B, T, H_I]; k_I [B, S, D_I] bytes,
    k_scale [B, S].  Returns float64 arrays of the same leading shapes.
    """
    q = e4m3_decode(q_I) * np.asarray(q_scale, dtype=np.float64)[..., None]
    k = e4m3_decode(k_I) * np.asarray(k_scale, dtype=np.float64)[..., None]
    return q, k


# ---------------------------------------------------------------------------
# positions
# ---------------------------------------------------------------------------


def query_pos(T: int, S: int, t: int) -> int:
    """Position of query token t when T queries attend over S keys: the queries
    are the last T tokens of the sequence, so pos = S - T + t.  A prefill
    (T == S) gives pos = t; a decode step (T == 1) gives pos = S - 1."""
    return S - T + t


# ---------------------------------------------------------------------------
# step A: lightning indexer
# ---------------------------------------------------------------------------


def indexer_row(qd_t, w_t, kd, pos: int) -> np.ndarray:
    """Scores of one query against keys 0..pos (inclusive).

    qd_t [H_I, D_I] dequantised query heads, w_t [H_I] head weights,
    kd [S, D_I] dequantised keys.  Returns float64 [pos + 1]:
        I[s] = sum_j w_t[j] * max(0, qd_t[j] . kd[s]).
    """
    dots = np.asarray(qd_t, np.float64) @ np.asarray(kd[: pos + 1], np.float64).T  # [H_I, pos+1]
    return np.asarray(w_t, np.float64) @ np.maximum(dots, 0.0)


def indexer_scores(qd, w, kd, S: int | None = None) -> np.ndarray:
    """Full score matrix for one sequence, -inf where the key is not visible.

    qd [T, H_I, D_I], w [T, H_I], kd [S, D_I].  Returns float64 [T, S].
    """
    T = qd.shape[0]
    S = kd.shape[0] if S is None else S
    out = np.full((T, S), -np.inf)
    for t in range(T):
        p = query_pos(T, S, t)
        out[t, : p + 1] = indexer_row(qd[t], w[t], kd, p)
    return out


# ---------------------------------------------------------------------------
# step B: top-k selection
# ---------------------------------------------------------------------------


def topk_row(scores_visible, k: int) -> np.ndarray:
    """Indices of the min(k, n) largest of the n visible scores.

    Ties go to the lower index: candidates are ordered by (score descending,
    index ascending) and the first min(k, n) are kept.  Keys that are not
    visible are never candidates.  Returns int64 [k], padded with -1.
    """
    sv = np.asarray(scores_visible, np.float64)
    n = sv.shape[0]
    order = np.lexsort((np.arange(n), -sv))  # primary: -score, secondary: index
    keep = order[: min(k, n)]
    out = np.full(k, -1, dtype=np.int64)
    out[: keep.shape[0]] = keep
    return out


def topk(scores, k: int, T: int | None = None, S: int | None = None) -> np.ndarray:
    """Top-k for every row of a [T, S] score matrix (row t sees 0..pos(t))."""
    T = scores.shape[0] if T is None else T
    S = scores.shape[1] if S is None else S
    out = np.empty((scores.shape[0], k), dtype=np.int64)
    for t in range(scores.shape[0]):
        p = query_pos(T, S, t)
        out[t] = topk_row(scores[t, : p + 1], k)
    return out


# ---------------------------------------------------------------------------
# step C: sparse MQA/MLA attention over the selected keys
# ---------------------------------------------------------------------------


def sparse_attention_row(q_t, kv, idx_t, d_v: int, tau: float, v=None):
    """Attention of all heads of one query over the selected rows of kv.

    q_t [H, d_k], kv [S, d_k] (one row shared by every head; value = first d_v
    columns), idx_t [k] with -1 for empty slots (skipped; duplicates count as
    often as they appear).  For each head h:
        z_s = tau * q_t[h] . kv[s],   m = max_s z_s,   p_s = exp(z_s - m)
        O[h] = sum_s p_s V[s] / sum_s p_s,             LSE[h] = m + ln sum_s p_s
    with V[s] = kv[s, :d_v] (MLA: the value is the cached latent), or, when a
    separate value array v [S, d_v] is given, V[s] = v[s] (the same formula
    with values kept apart from the keys).
    Returns (O [H, d_v], LSE [H]) in float64.
    """
    sel = np.asarray(idx_t)
    sel = sel[sel >= 0]
    K = np.asarray(kv[sel], np.float64)                       # [n, d_k]
    V = K[:, :d_v] if v is None else np.asarray(v[sel], np.float64)
    z = tau * (np.asarray(q_t, np.float64) @ K.T)             # [H, n]
    m = z.max(axis=1, keepdims=True)
    p = np.exp(z - m)
    l = p.sum(axis=1, keepdims=True)
    O = (p @ V) / l
    lse = (m + np.log(l))[:, 0]
    return O, lse


def sparse_attention(q, kv, idx, d_v: int, tau: float):
    """Sparse attention for every query of one sequence: q [T, H, d_k]."""
    T, H, _ = q.shape
    O = np.empty((T, H, d_v))
    L = np.empty((T, H))
    for t in range(T):
        O[t], L[t] = sparse_attention_row(q[t], kv, idx[t], d_v, tau)
    return O, L


def dense_causal_attention_row(q_t, kv, pos: int, d_v: int, tau: float, v=None):
    """Plain softmax attention of one query over every visible key 0..pos.

    Written without the selection machinery, as the textbook definition:
    weights = exp(z - logsumexp(z)), O = weights @ V, with V = kv[:, :d_v] or
    the separate value array v.  It pins the sparse path (with k >= pos + 1
    every visible key is kept, so DSA must reduce exactly to this) and is the
    reference of the dense short-prefill form.
    """
    V = np.asarray((kv[:, :d_v] if v is None else v)[: pos + 1], np.float64)
    Kf = np.asarray(kv[: pos + 1], np.float64)
    out = np.empty((q_t.shape[0], d_v))
    lse = np.empty(q_t.shape[0])
    for h in range(q_t.shape[0]):
        z = tau * (Kf @ np.asarray(q_t[h], np.float64))
        zmax = np.max(z)
        lse[h] = zmax + np.log(np.sum(np.exp(z - zmax)))
        out[h] = np.exp(z - lse[h]) @ V
    return out, lse


# ---------------------------------------------------------------------------
# one sequence's keys spread over several parts (key-split decode)
# ---------------------------------------------------------------------------


def topk_merge(cand_scores, cand_idx, k: int) -> np.ndarray:
    """Top-k of the union of candidate lists (score, key index), index -1 =
    empty slot: order by (score descending, index ascending), keep the first
    min(k, n).  With disjoint key ranges and each list the top-k of its range
    under the same order, this is the top-k of the whole row (an element of
    the global top-k has fewer than k better elements globally, hence in its
    own range).  Returns int64 [k] padded with -1."""
    cs = np.asarray(cand_scores, np.float64).ravel()
    ci = np.asarray(cand_idx, np.int64).ravel()
    ok = ci >= 0
    cs, ci = cs[ok], ci[ok]
    order = np.lexsort((ci, -cs))
    keep = ci[order[: min(k, ci.shape[0])]]
    out = np.full(k, -1, dtype=np.int64)
    out[: keep.shape[0]] = keep
    return out


def combine_partials(o_parts, lse_parts):
    """Attention over a key set from its results over disjoint subsets:
    with M = max_r LSE_r (parts with LSE = -inf, i.e. no key, are skipped),
        O = sum_r e^(LSE_r - M) O_r / sum_r e^(LSE_r - M),
        LSE = M + ln sum_r e^(LSE_r - M).
    o_parts [P, H, d_v], lse_parts [P, H]; returns (O [H, d_v], LSE [H])."""
    o = np.asarray(o_parts, np.float64)
    ls = np.asarray(lse_parts, np.float64)
    M = ls.max(axis=0)                                      # [H]
    w = np.where(np.isfinite(ls), np.exp(ls - M[None, :]), 0.0)
    den = w.sum(axis=0)
    O = (w[:, :, None] * o).sum(axis=0) / den[:, None]
    return O, M + np.log(den)


# ---------------------------------------------------------------------------
# training the indexer (kernel level)
# ---------------------------------------------------------------------------
#
# tenelement.pl, "DeepSeek V3.2-Exp Cuts Long-Context Costs ...", section
# "Proces Treningu DSA: Od Warm-up do Sparsity": in a short warm-up the
# indexer learns the dense model's attention distribution through a KL
# divergence while the main model is frozen; then a sparse stage trains with
# top-k = 2048, and the indexer's gradients stay separate from the main
# language loss (ouchyi thread, "Nasil calisiyor": the indexer is aligned by
# KL divergence first).  Readings where the pages are silent: the target of
# query t is the main attention's weights summed over heads and divided by H
# (an L1-normalised distribution over keys); the loss is KL(target ||
# softmax(I[t, .])) over the visible keys (warm-up) or over the selected set
# (sparse stage, where both distributions are taken over the set); the target
# is a constant (no gradient flows into the main attention).


def kl_target_row(q_t, kv, pos: int, tau: float, sel=None) -> np.ndarray:
    """Target distribution of query t: p[s] = (1/H) sum_h softmax_s(tau q_h . kv[s])
    over the visible keys 0..pos, or over the selected set `sel` (-1 = empty
    slot) when given.  Returns float64 [pos + 1] (zero outside the set)."""
    keys = np.arange(pos + 1) if sel is None else np.unique(np.asarray(sel)[np.asarray(sel) >= 0])
    K = np.asarray(kv[keys], np.float64)
    z = tau * (np.asarray(q_t, np.float64) @ K.T)               # [H, n]
    z = z - z.max(axis=1, keepdims=True)
    a = np.exp(z)
    a = a / a.sum(axis=1, keepdims=True)
    p = np.zeros(pos + 1)
    p[keys] = a.mean(axis=0)
    return p


def indexer_kl_row(scores_t, p_t, sel=None):
    """KL(p || softmax(I)) of one query row and its gradient with respect to
    the scores.  scores_t, p_t: float64 [n] over keys 0..pos; with `sel`, both
    distributions are over the selected set only.  With q = softmax(I) over
    the set, loss = sum_s p_s (ln p_s - ln q_s) (terms with p_s = 0 are 0) and
    dloss/dI_s = q_s - p_s (zero outside the set).  Returns (loss, grad [n])."""
    I = np.asarray(scores_t, np.float64)
    n = I.shape[0]
    keys = np.arange(n) if sel is None else np.unique(np.asarray(sel)[np.asarray(sel) >= 0])
    z = I[keys] - I[keys].max()
    lq = z - np.log(np.exp(z).sum())
    ps = np.asarray(p_t, np.float64)[keys]
    nz = ps > 0
    loss = float(np.sum(ps[nz] * (np.log(ps[nz]) - lq[nz])))
    g = np.zeros(n)
    g[keys] = np.exp(lq) - ps
    return loss, g


def indexer_grads_row(qd_t, w_t, kd, pos: int, g_t):
    """Chain rule of sum_s g_s I[t, s] back to the indexer's inputs, with
    I[t, s] = sum_j w_j ReLU(q_j . k_s) on the dequantised operands:
        dw_j  = sum_s g_s ReLU(q_j . k_s)
        dq_j  = sum_s g_s w_j [q_j . k_s > 0] k_s
        dk_s  = sum_j g_s w_j [q_j . k_s > 0] q_j      (row t's contribution)
    g_t: float64 [pos + 1].  Returns (dq [H_I, D_I], dw [H_I], dk [pos + 1, D_I])."""
    Q = np.asarray(qd_t, np.float64)
    K = np.asarray(kd[: pos + 1], np.float64)
    w = np.asarray(w_t, np.float64)
    g = np.asarray(g_t, np.float64)
    dots = Q @ K.T                                              # [H_I, n]
    dw = np.maximum(dots, 0.0) @ g
    G = (w[:, None] * (dots > 0)) * g[None, :]                  # [H_I, n]
    return G @ K, dw, G.T @ Q


# ---------------------------------------------------------------------------
# the whole path, and the work it touches
# ---------------------------------------------------------------------------


def default_tau(d_k: int) -> float:
    """Softmax scale 1/sqrt(d_k) (the pages do not state one)."""
    return 1.0 / np.sqrt(d_k)


def dsa_row(qd_t, w_t, kd, q_t, kv, pos: int, k: int, d_v: int, tau: float):
    """One query through all three steps.  Returns (scores, idx, O, LSE)."""
    sc = indexer_row(qd_t, w_t, kd, pos)
    idx = topk_row(sc, k)
    O, lse = sparse_attention_row(q_t, kv, idx, d_v, tau)
    return sc, idx, O, lse


def work_counts(T: int, S: int, k: int) -> dict:
    """Pairs touched by each step for one sequence.

    indexer: every visible (t, s) pair, sum_t (pos(t) + 1);
    attention: sum_t min(pos(t) + 1, k) -- linear in T for fixed k, the
    O(L k) claim of the pages (ouchyi thread; sider.ai blog, "Matematik,
    Minimalist Surum").
    """
    ip = 0
    ap = 0
    for t in range(T):
        v = query_pos(T, S, t) + 1
        ip += v
        ap += min(v, k)
    return {"indexer_pairs": ip, "attention_pairs": ap}


class CountingOracle:
    """Runs the path row by row and counts the pairs each step actually visits.

    The counters come from the arrays the steps touch, not from the closed
    form in :func:`work_counts`, so a test can compare the two.
    """

    def __init__(self):
        self.indexer_pairs = 0
        self.attention_pairs = 0

    def run(self, qd, w, kd, q, kv, k: int, d_v: int, tau: float):
        T = qd.shape[0]
        S = kd.shape[0]
        outs = []
        for t in range(T):
            p = query_pos(T, S, t)
            sc = indexer_row(qd[t], w[t], kd, p)
            self.indexer_pairs += sc.shape[0]
            idx = topk_row(sc, k)
            self.attention_pairs += int((idx >= 0).sum())
            outs.append(sparse_attention_row(q[t], kv, idx, d_v, tau))
        return outs


def from_inputs(inp: dict, b: int = 0) -> dict:
    """Dequantise one sequence of a make_inputs() batch (CPU tensors or arrays)
    into float64 arrays for the functions above."""
    def a(x):
        return x.cpu().numpy() if hasattr(x, "cpu") else np.asarray(x)
    qd, kd = dequant_indexer(a(inp["q_I"][b]), a(inp["q_scale"][b]), a(inp["k_I"][b]), a(inp["k_scale"][b]))
    q = inp["q"][b]
    kv = inp["kv"][b]
    if hasattr(q, "view"):
        import torch  # only to reinterpret bf16 storage as uint16 bits
        q = q.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        kv = kv.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return {"qd": qd, "w": a(inp["w"][b]).astype(np.float64), "kd": kd,
            "q": bf16_decode(q), "kv": bf16_decode(kv)}
