"""Host-side arithmetic of bench.py (no GPU): the algorithmic work behind the
roofline fractions, and the guard on the captured DRAM traffic."""
import hashlib
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_causal_pairs_closed_forms(bench):
    """Pair counts equal the closed forms of the causal O(L k) work.

    Indexer: sum over queries of pos + 1.  Attention: sum of min(pos + 1, k).
    """
    from long_context_05_b200.inputs import WORKLOADS
    wl = WORKLOADS["prefill_128k"]
    ip, ap = bench.causal_pairs(wl)
    L, k = wl.T, wl.k
    assert ip == L * (L + 1) // 2 == 8_590_000_128
    assert ap == k * (k + 1) // 2 + (L - k) * k == 266_339_328
    dec = WORKLOADS["decode_128k_b8"]
    ip, ap = bench.causal_pairs(dec)
    assert ip == dec.B * dec.S and ap == dec.B * dec.k


def test_algorithmic_flops_per_pair(bench):
    """The roofline's work: 2 H_I D_I FLOP per indexer pair and
    2 H (d_k + d_v) FLOP per attention pair (128K prefill: 1.407e14 and 7.42e13)."""
    from long_context_05_b200.inputs import WORKLOADS
    wl = WORKLOADS["prefill_128k"]
    peaks = {"bf16_tflops": 1000.0, "bf16_tflops_sustained": 1000.0, "hbm_gbs": 1000.0}
    per_kernel = {"indexer": [1000.0], "topk": [1000.0], "sparse_attn": [1000.0]}  # 1 s each
    rep = bench.kernel_report(wl, per_kernel, 1, peaks, "test", sustained=True)
    # the first k rows keep every visible key: they are neither scored nor selected
    scored = 8_590_000_128 - 2048 * 2049 // 2
    assert bench.dense_rows(wl) == 2048 and bench.scored_pairs(wl) == scored
    assert rep["indexer"]["achieved"] == pytest.approx(2 * 64 * 128 * scored / 1e12)
    assert rep["sparse_attn"]["achieved"] == pytest.approx(2 * 128 * (576 + 512) * 266_339_328 / 1e12)
    assert rep["topk"]["achieved"] == pytest.approx(4 * scored / 1e9)


def test_decode_indexer_is_reported_against_hbm(bench):
    """In decode the indexer streams every key once: its roofline is HBM on
    the k_I and k_scale bytes (8 x 131072 x 132 B = 138.4 MB for the 128K decode)."""
    from long_context_05_b200.inputs import WORKLOADS
    dec = WORKLOADS["decode_128k_b8"]
    peaks = {"bf16_tflops": 1000.0, "bf16_tflops_sustained": 1000.0, "hbm_gbs": 1000.0}
    rep = bench.kernel_report(dec, {"indexer": [1.0], "topk": [1.0], "sparse_attn": [1.0]}, 1, peaks, "t", False)
    assert rep["indexer"]["bound"] == "hbm" and rep["indexer"]["unit"] == "GB/s"
    assert rep["indexer"]["work_per_step"] == pytest.approx(8 * 131072 * 132)
    assert rep["sparse_attn"]["bound"] == "hbm"


def test_traffic_reported_only_for_the_captured_source(bench):
    """roofline.traffic is the captured figure only for the captured
    (workload, kernel) and only while the kernel source is unchanged."""
    t = bench.ATTN_TRAFFIC
    with open(os.path.join(ROOT, t["source"]), "rb") as f:
        same = hashlib.sha256(f.read()).hexdigest() == t["sha256"]
    got = bench.measured_traffic("prefill_128k", "sparse_attn")
    assert got == (t["bytes"] if same else None)
    assert bench.measured_traffic("prefill_8k", "sparse_attn") is None
    assert bench.measured_traffic("prefill_128k", "indexer") is None


def test_paged_layout_places_every_token():
    """to_paged (the paged caches of the tests and the bench's paged decode):
    token s of sequence b lands at pool row table[b, s // P] * P + s % P with
    every key-side array moved alike, no two tokens share a pool row, the
    table's extra column is -1, and the spare pool pages stay zero."""
    import torch
    from long_context_05_b200.inputs import Workload, make_inputs, to_paged
    wl = Workload("paged_host", B=3, T=1, S=1000, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=64, q_block=1, seed=21)
    inp = make_inputs(wl, "cpu")
    inp["v"] = torch.randn(wl.B, wl.S, wl.d_v).to(torch.bfloat16)
    P = 64
    pin, table, num_pages = to_paged(inp, wl, P, 22)
    ppseq = (wl.S + P - 1) // P
    assert num_pages == wl.B * ppseq + 2 and tuple(table.shape) == (wl.B, ppseq + 1)
    t = table.numpy()
    assert (t[:, -1] == -1).all()
    assert sorted(t[:, :ppseq].ravel().tolist()) == sorted(set(t[:, :ppseq].ravel().tolist()))
    s = torch.arange(wl.S)
    for b in range(wl.B):
        rows = torch.from_numpy(t[b, (s // P).numpy()]).long() * P + s % P
        for name in ("k_I", "k_scale", "kv", "v"):
            assert torch.equal(pin[name][rows], inp[name][b]), (name, b)
    used = set(t[:, :ppseq].ravel().tolist())
    for pg in set(range(num_pages)) - used:
        assert not pin["kv"][pg * P:(pg + 1) * P].float().abs().any()
