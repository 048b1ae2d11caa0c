"""Pins for the FP64 oracle: values the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a worked
example under tests/golden/, a closed form, an invariant, a library routine
for a special case, or brute force on tiny inputs.  No expected value comes
from the CUDA path.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from long_context_05_b200.inputs import WORKLOADS, make_inputs

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLD, name)) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if line:
                yield line


# ---------------------------------------------------------------- formats

def test_e4m3_table_from_spec():
    for line in _lines("e4m3_table.txt"):
        hx, val = line.split()
        got = float(O.e4m3_decode(np.array([int(hx, 16)], np.uint8))[0])
        if val == "nan":
            assert math.isnan(got), hx
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), hx


def test_e4m3_all_bytes_match_torch():
    # torch's float8_e4m3fn is an independent implementation of the same format
    b = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(b)
    ref = torch.from_numpy(b).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_bf16_decode_matches_torch():
    g = torch.Generator().manual_seed(7)
    x = torch.randn(4096, generator=g).bfloat16()
    bits = x.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.bf16_decode(bits), x.double().numpy())


# ---------------------------------------------------------------- indexer

def _read_indexer_fixture():
    q, qs, w, k, ks, I = {}, {}, {}, {}, {}, {}
    for line in _lines("indexer_tiny.txt"):
        f = line.split()
        if f[0] == "q":
            t, j = int(f[1]), int(f[2])
            q[(t, j)] = [int(x, 16) for x in f[3:5]]
            qs[(t, j)] = float(f[6])
        elif f[0] == "w":
            w[int(f[1])] = [float(x) for x in f[2:]]
        elif f[0] == "k":
            s = int(f[1])
            k[s] = [int(x, 16) for x in f[2:4]]
            ks[s] = float(f[5])
        elif f[0] == "I":
            I[int(f[1])] = [float(x) for x in f[2:]]
    T, HI, D = 3, 2, 2
    qb = np.array([[q[(t, j)] for j in range(HI)] for t in range(T)], np.uint8)
    qsc = np.array([[qs[(t, j)] for j in range(HI)] for t in range(T)])
    kb = np.array([k[s] for s in range(3)], np.uint8)
    ksc = np.array([ks[s] for s in range(3)])
    wa = np.array([w[t] for t in range(T)])
    return qb, qsc, wa, kb, ksc, I


def test_indexer_worked_example():
    qb, qsc, wa, kb, ksc, I = _read_indexer_fixture()
    qd, kd = O.dequant_indexer(qb, qsc, kb, ksc)
    sc = O.indexer_scores(qd, wa, kd)
    for t, row in I.items():
        assert np.array_equal(sc[t, : t + 1], np.array(row)), (t, sc[t])
        assert np.all(np.isneginf(sc[t, t + 1:]))


def test_indexer_closed_form_single_head():
    # one head, w = 1, q = k = a e_1  ->  I = a^2 (and ReLU keeps it)
    for a in [0.5, 3.0, 17.25]:
        qd = np.zeros((1, 1, 8)); qd[0, 0, 0] = a
        kd = np.zeros((1, 8)); kd[0, 0] = a
        assert O.indexer_row(qd[0], np.ones(1), kd, 0)[0] == a * a
        kd[0, 0] = -a  # negative logit is cut by the ReLU
        assert O.indexer_row(qd[0], np.ones(1), kd, 0)[0] == 0.0


def test_indexer_integer_mode_equals_int64_brute_force():
    wl = WORKLOADS["tiny_prefill_256"]
    inp = make_inputs(wl, "cpu")
    d = O.from_inputs(inp)
    sc = O.indexer_scores(d["qd"], d["w"], d["kd"])
    # integer brute force: int64 dots, ReLU, then w = +-2^e applied exactly
    qi = inp["q_I"][0].view(torch.float8_e4m3fn).to(torch.int64).numpy()   # [T, H, D]
    ki = inp["k_I"][0].view(torch.float8_e4m3fn).to(torch.int64).numpy()   # [S, D]
    dots = np.einsum("thd,sd->ths", qi, ki)                                 # exact int64
    w4 = (inp["w"][0].numpy() * 4).astype(np.int64)                          # 4 w is an integer
    assert np.array_equal(w4.astype(np.float64) / 4, inp["w"][0].numpy())
    ref4 = np.einsum("th,ths->ts", w4, np.maximum(dots, 0))
    for t in range(wl.T):
        assert np.array_equal(sc[t, : t + 1] * 4, ref4[t, : t + 1].astype(np.float64))


def test_indexer_scale_homogeneity():
    rng = np.random.default_rng(3)
    qd = rng.standard_normal((5, 4, 16)); w = rng.standard_normal((5, 4)); kd = rng.standard_normal((5, 16))
    a = O.indexer_scores(qd, w, kd)
    b = O.indexer_scores(qd, w, 2 * kd)        # all key scales doubled
    c = O.indexer_scores(3 * qd, w, kd)        # positive query scale
    fin = np.isfinite(a)
    assert np.allclose(b[fin], 2 * a[fin], rtol=1e-14, atol=0)
    assert np.allclose(c[fin], 3 * a[fin], rtol=1e-14, atol=0)


# ---------------------------------------------------------------- top-k

def _is_valid_topk(scores, k, sel):
    """Characterisation of the selected set: right size, and every kept key
    beats every dropped key by (score desc, index asc)."""
    n = len(scores)
    kept = set(int(i) for i in sel if i >= 0)
    if len(kept) != min(k, n) or list(sel).count(-1) != k - min(k, n):
        return False
    for a in kept:
        for b in set(range(n)) - kept:
            if not (scores[a] > scores[b] or (scores[a] == scores[b] and a < b)):
                return False
    return True


def test_topk_worked_examples():
    for line in _lines("topk_tiny.txt"):
        ks, sc, exp, pad = [p.strip() for p in line.split("|")]
        k = int(ks)
        scores = np.array([float(x) for x in sc.split()])
        got = O.topk_row(scores, k)
        assert sorted(int(i) for i in got if i >= 0) == [int(x) for x in exp.split()]
        assert int((got == -1).sum()) == int(pad)


def test_topk_exhaustive_subsets_tiny():
    # brute force over all subsets of size min(k, n): exactly one satisfies the
    # characterisation, and it is the oracle's
    rng = np.random.default_rng(11)
    for _ in range(200):
        n = int(rng.integers(1, 8))
        k = int(rng.integers(1, 9))
        scores = rng.integers(-2, 3, n).astype(np.float64)   # many ties
        good = [c for c in itertools.combinations(range(n), min(k, n))
                if _is_valid_topk(scores, k, list(c) + [-1] * (k - min(k, n)))]
        assert len(good) == 1
        got = O.topk_row(scores, k)
        assert sorted(int(i) for i in got if i >= 0) == list(good[0])


def test_topk_matches_full_sort_large():
    rng = np.random.default_rng(5)
    for n, k in [(5000, 2048), (2000, 2048), (70000, 2048)]:
        s = np.round(rng.standard_normal(n), 2)  # ties
        got = O.topk_row(s, k)
        full = sorted(range(n), key=lambda i: (-s[i], i))[: min(k, n)]
        assert sorted(int(i) for i in got if i >= 0) == sorted(full)


def test_topk_row_causal_visibility():
    sc = np.array([[1.0, 9.0, 9.0], [1.0, 2.0, 9.0], [3.0, 2.0, 1.0]])
    sc_masked = sc.copy()
    for t in range(3):
        sc_masked[t, t + 1:] = -np.inf
    idx = O.topk(sc_masked, 2)
    assert list(idx[0]) == [0, -1]
    assert sorted(idx[1]) == [0, 1]
    assert sorted(idx[2]) == [0, 1]


# ---------------------------------------------------------------- attention

def test_attention_worked_example():
    kv, q, idx, Oe, Le = {}, {}, None, {}, {}
    for line in _lines("attention_tiny.txt"):
        f = line.split()
        if f[0] == "kv":
            kv[int(f[1])] = [float(x) for x in f[2:]]
        elif f[0] == "q":
            q[int(f[1])] = [float(x) for x in f[2:]]
        elif f[0] == "idx":
            idx = np.array([int(x) for x in f[1:]])
        elif f[0] == "O":
            Oe[int(f[1])] = float(f[2])
        elif f[0] == "LSE":
            Le[int(f[1])] = float(f[2])
    kva = np.array([kv[i] for i in range(3)])
    qa = np.array([q[h] for h in range(2)])
    out, lse = O.sparse_attention_row(qa, kva, idx, d_v=1, tau=1.0)
    for h in range(2):
        assert abs(out[h, 0] - Oe[h]) < 1e-14
        assert abs(lse[h] - Le[h]) < 1e-14


def test_attention_single_key_returns_value():
    rng = np.random.default_rng(2)
    kv = rng.standard_normal((10, 12)); q = rng.standard_normal((3, 12))
    out, lse = O.sparse_attention_row(q, kv, np.array([7, -1, -1]), d_v=8, tau=0.3)
    assert np.array_equal(out, np.broadcast_to(kv[7, :8], (3, 8)))
    assert np.allclose(lse, 0.3 * q @ kv[7])


def test_attention_equal_logits_mean():
    rng = np.random.default_rng(4)
    kv = rng.standard_normal((10, 12)); q = np.zeros((2, 12))
    sel = np.array([1, 4, 6, 9])
    out, lse = O.sparse_attention_row(q, kv, sel, d_v=5, tau=1.0)
    assert np.allclose(out, kv[sel, :5].mean(0), rtol=0, atol=1e-15)
    assert np.allclose(lse, np.log(4.0))


def test_attention_separate_values_single_key_and_mean():
    """With values kept apart from the keys, one selected key returns its value
    row exactly and equal logits return the mean of the selected value rows;
    the key rows' own leading columns must play no part."""
    rng = np.random.default_rng(5)
    kv = rng.standard_normal((10, 12)); v = rng.standard_normal((10, 6))
    q = rng.standard_normal((3, 12))
    out, lse = O.sparse_attention_row(q, kv, np.array([-1, 4, -1]), d_v=6, tau=0.5, v=v)
    assert np.array_equal(out, np.broadcast_to(v[4], (3, 6)))
    assert np.allclose(lse, 0.5 * q @ kv[4])
    sel = np.array([0, 3, 3, 8])
    out, lse = O.sparse_attention_row(np.zeros((2, 12)), kv, sel, d_v=6, tau=1.0, v=v)
    assert np.allclose(out, v[sel].mean(0), rtol=0, atol=1e-15)
    assert np.allclose(lse, np.log(4.0))
    od, ld = O.dense_causal_attention_row(np.zeros((2, 12)), kv, 4, 6, 1.0, v=v)
    assert np.allclose(od, v[:5].mean(0), rtol=0, atol=1e-15) and np.allclose(ld, np.log(5.0))


def test_attention_permutation_invariance_and_lse():
    rng = np.random.default_rng(6)
    kv = rng.standard_normal((50, 24)); q = rng.standard_normal((4, 24))
    sel = rng.choice(50, 20, replace=False)
    o1, l1 = O.sparse_attention_row(q, kv, sel, 16, 0.2)
    o2, l2 = O.sparse_attention_row(q, kv, sel[::-1].copy(), 16, 0.2)
    assert np.allclose(o1, o2, atol=1e-14) and np.allclose(l1, l2, atol=1e-14)
    z = 0.2 * q @ kv[sel].T
    assert np.allclose(np.exp(z - l1[:, None]).sum(1), 1.0, atol=1e-14)


def test_topk_merge_of_range_winners_equals_whole_row():
    """The top-k of a row equals the merge of the top-k of its disjoint key
    ranges, ties included (integer scores with large tie groups)."""
    rng = np.random.default_rng(11)
    for n, k, parts in ((1000, 64, 2), (3000, 512, 4), (257, 300, 3)):
        row = rng.integers(-4, 5, n).astype(np.float64)
        ref = O.topk_row(row, k)
        bounds = np.linspace(0, n, parts + 1).astype(int)
        cs, ci = [], []
        for a, b in zip(bounds[:-1], bounds[1:]):
            loc = O.topk_row(row[a:b], k)
            ci.append(np.where(loc >= 0, loc + a, -1))
            cs.append(np.where(loc >= 0, row[a + np.maximum(loc, 0)], 0.0))
        assert np.array_equal(O.topk_merge(np.stack(cs), np.stack(ci), k), ref)


def test_combine_partials_equals_attention_over_the_union():
    rng = np.random.default_rng(12)
    kv = rng.standard_normal((200, 24)); q = rng.standard_normal((3, 24)) * 2
    sel = rng.choice(200, 60, replace=False)
    o_all, l_all = O.sparse_attention_row(q, kv, sel, 16, 0.3)
    parts = [sel[:10], sel[10:45], sel[45:], np.array([-1, -1])]      # the last part is empty
    res = [O.sparse_attention_row(q, kv, s_, 16, 0.3) if (s_ >= 0).any()
           else (np.zeros((3, 16)), np.full(3, -np.inf)) for s_ in parts]
    o, l = O.combine_partials(np.stack([r[0] for r in res]), np.stack([r[1] for r in res]))
    assert np.max(np.abs(o - o_all)) < 1e-12 and np.max(np.abs(l - l_all)) < 1e-12


def test_sparse_equals_dense_when_k_covers_context():
    """k >= visible keys: DSA reduces exactly to dense causal attention
    (ouchyi thread: only the top-k entries are kept -- with k at least the
    context, all are; tenelement.pl, section "Efektywnosc Kosztowa": short
    prefill as masked MHA)."""
    wl = WORKLOADS["tiny_prefill_256"]
    inp = make_inputs(wl, "cpu")
    d = O.from_inputs(inp)
    tau = O.default_tau(wl.d_k)
    sc = O.indexer_scores(d["qd"], d["w"], d["kd"])
    idx = O.topk(sc, wl.S)   # k = S covers every visible key
    for t in [0, 1, 5, 63, 64, 200, 255]:
        o_s, l_s = O.sparse_attention_row(d["q"][t], d["kv"], idx[t], wl.d_v, tau)
        o_d, l_d = O.dense_causal_attention_row(d["q"][t], d["kv"], t, wl.d_v, tau)
        assert np.max(np.abs(o_s - o_d)) < 1e-12
        assert np.max(np.abs(l_s - l_d)) < 1e-12
    # and with the workload's k, rows that see at most k keys are dense too
    idx64 = O.topk(sc, wl.k)
    for t in [0, 30, wl.k - 1]:
        o_s, _ = O.sparse_attention_row(d["q"][t], d["kv"], idx64[t], wl.d_v, tau)
        o_d, _ = O.dense_causal_attention_row(d["q"][t], d["kv"], t, wl.d_v, tau)
        assert np.max(np.abs(o_s - o_d)) < 1e-12


def test_causality_future_keys_do_not_matter():
    wl = WORKLOADS["tiny_prefill_256"].with_(T=40, S=40, k=8)
    inp = make_inputs(wl, "cpu")
    d = O.from_inputs(inp)
    tau = O.default_tau(wl.d_k)
    t = 20
    a = O.dsa_row(d["qd"][t], d["w"][t], d["kd"], d["q"][t], d["kv"], t, wl.k, wl.d_v, tau)
    kd2, kv2 = d["kd"].copy(), d["kv"].copy()
    kd2[t + 1:] *= -3.0
    kv2[t + 1:] += 5.0
    b = O.dsa_row(d["qd"][t], d["w"][t], kd2, d["q"][t], kv2, t, wl.k, wl.d_v, tau)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])


def test_decode_step_equals_prefill_row():
    wl = WORKLOADS["tiny_prefill_256"].with_(T=64, S=64, k=16)
    inp = make_inputs(wl, "cpu")
    d = O.from_inputs(inp)
    tau = O.default_tau(wl.d_k)
    t = 50
    pre = O.dsa_row(d["qd"][t], d["w"][t], d["kd"], d["q"][t], d["kv"], O.query_pos(64, 64, t),
                    wl.k, wl.d_v, tau)
    # a decode step over the first t+1 keys: T = 1 query at position S - 1
    S = t + 1
    dec = O.dsa_row(d["qd"][t], d["w"][t], d["kd"][:S], d["q"][t], d["kv"][:S],
                    O.query_pos(1, S, 0), wl.k, wl.d_v, tau)
    for x, y in zip(pre, dec):
        assert np.array_equal(x, y)


# ---------------------------------------------------------------- complexity

def test_work_counts_o_lk():
    """O(L k) attention pairs vs O(L^2) indexer pairs (ouchyi thread; sider.ai
    blog, "Matematik, Minimalist Surum"): the counters of a real run match the
    closed forms, and attention pairs grow linearly once L > k."""
    rng = np.random.default_rng(9)
    T = S = 48
    k = 6
    qd = rng.standard_normal((T, 2, 4)); w = rng.standard_normal((T, 2)); kd = rng.standard_normal((S, 4))
    q = rng.standard_normal((T, 2, 6)); kv = rng.standard_normal((S, 6))
    c = O.CountingOracle()
    c.run(qd, w, kd, q, kv, k, 4, 0.5)
    wc = O.work_counts(T, S, k)
    assert c.indexer_pairs == wc["indexer_pairs"] == T * (T + 1) // 2
    assert c.attention_pairs == wc["attention_pairs"] == k * (k + 1) // 2 + (T - k) * k
    a1 = O.work_counts(4096, 4096, 2048)["attention_pairs"]
    a2 = O.work_counts(8192, 8192, 2048)["attention_pairs"]
    assert a2 - a1 == 4096 * 2048           # linear in L beyond k
    assert O.work_counts(1, 131072, 2048)["attention_pairs"] == 2048


# ---------------------------------------------------------------- indexer training

def _train_case(seed=21, HI=3, DI=5, S=12, H=4, dk=6):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((HI, DI)), rng.standard_normal(HI), rng.standard_normal((S, DI)),
            rng.standard_normal((H, dk)), rng.standard_normal((S, dk)))


def test_kl_target_is_head_mean_of_dense_attention_weights():
    """p sums to 1 and p @ V equals the mean over heads of the independent
    dense attention output (the target is the heads' weights averaged)."""
    _, _, _, q, kv = _train_case()
    pos, tau, dv = 9, 0.4, 3
    p = O.kl_target_row(q, kv, pos, tau)
    assert abs(p.sum() - 1.0) < 1e-14 and np.all(p >= 0)
    o, _ = O.dense_causal_attention_row(q, kv, pos, dv, tau)
    assert np.allclose(p @ kv[: pos + 1, :dv], o.mean(0), atol=1e-14)
    # over a selected set: zero outside it, and the same identity with the
    # sparse attention
    sel = np.array([7, 2, -1, 5, 9])
    ps = O.kl_target_row(q, kv, pos, tau, sel)
    assert np.all(ps[[0, 1, 3, 4, 6, 8]] == 0) and abs(ps.sum() - 1) < 1e-14
    os_, _ = O.sparse_attention_row(q, kv, sel, dv, tau)
    assert np.allclose(ps @ kv[: pos + 1, :dv], os_.mean(0), atol=1e-14)


def test_indexer_kl_loss_and_score_gradient():
    rng = np.random.default_rng(22)
    I = rng.standard_normal(10)
    p = rng.random(10)
    p /= p.sum()
    loss, g = O.indexer_kl_row(I, p)
    assert loss >= 0
    q = np.exp(I - I.max()); q /= q.sum()
    assert abs(loss - np.sum(p * np.log(p / q))) < 1e-13
    # gradient by central differences
    for s in range(10):
        e = np.zeros(10); e[s] = 1e-6
        fd = (O.indexer_kl_row(I + e, p)[0] - O.indexer_kl_row(I - e, p)[0]) / 2e-6
        assert abs(fd - g[s]) < 1e-8
    # p == softmax(I): no loss, no gradient
    l0, g0 = O.indexer_kl_row(I, q)
    assert abs(l0) < 1e-14 and np.max(np.abs(g0)) < 1e-15
    # over a set: the other keys get no gradient
    sel = np.array([1, 4, 6])
    pset = np.zeros(10); pset[sel] = p[sel] / p[sel].sum()      # a target over the set
    ls, gs = O.indexer_kl_row(I, pset, sel)
    assert np.all(gs[[0, 2, 3, 5, 7, 8, 9]] == 0) and abs(gs.sum()) < 1e-14


def test_indexer_input_gradients_by_finite_differences():
    """dq, dw, dk of the KL loss through the indexer, against central
    differences of the loss as a function of the inputs."""
    Q, w, K, q, kv = _train_case()
    pos, tau = 10, 0.5
    p = O.kl_target_row(q, kv, pos, tau)

    def loss(Q_, w_, K_):
        return O.indexer_kl_row(O.indexer_row(Q_, w_, K_, pos), p)[0]

    _, g = O.indexer_kl_row(O.indexer_row(Q, w, K, pos), p)
    dq, dw, dk = O.indexer_grads_row(Q, w, K, pos, g)
    h = 1e-6
    for (j, d) in [(0, 0), (1, 3), (2, 4)]:
        E = np.zeros_like(Q); E[j, d] = h
        assert abs((loss(Q + E, w, K) - loss(Q - E, w, K)) / (2 * h) - dq[j, d]) < 1e-7
    for j in range(3):
        e = np.zeros(3); e[j] = h
        assert abs((loss(Q, w + e, K) - loss(Q, w - e, K)) / (2 * h) - dw[j]) < 1e-7
    for (s_, d) in [(0, 1), (5, 2), (10, 4)]:
        E = np.zeros_like(K); E[s_, d] = h
        assert abs((loss(Q, w, K + E) - loss(Q, w, K - E)) / (2 * h) - dk[s_, d]) < 1e-7
    # keys past pos play no part
    assert dk.shape[0] == pos + 1
