"""GPU parity: the CUDA path through the C ABI against the FP64 oracle.

Every call goes through libdsa.so (ctypes binding); the oracle runs on CPU
copies of the rows it checks.  Sizes: the tiny integer workload in full, small
ragged shapes that span several tiles, the two decode workloads in full (every
row's whole score row element by element too), and the prefill workloads at
full size on stratified samples of about 1,100-1,250 query rows each (the
first 64, k-2..k+1, both sides of every query-block boundary, the last 64 and
1,024 random rows), plus the whole score rows of 32 rows of one 4096-row
block of the 128K prefill.  The sample size is in each test id.
"""
import numpy as np
import pytest
import torch

from long_context_05_b200 import dsa
from long_context_05_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import dsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.lib()
    yield
    torch.cuda.synchronize()


def _tau(wl):
    return float(O.default_tau(wl.d_k))


def _run_forward(wl, inp, entry="dsa_forward"):
    shape = dsa.make_shape(wl)
    ws = dsa.alloc_workspace(shape)
    outs = dsa.alloc_outputs(wl)
    outs.idx.fill_(-7)
    dsa.forward(shape, inp, outs.out, outs.lse, outs.idx, ws, entry=entry)
    st, det = dsa.device_error()
    assert st == 0, f"device error {dsa.STATUS.get(st)} detail {det:#x}"
    return outs


def _scores_for_rows(wl, inp, q_begin, q_count):
    shape = dsa.make_shape(wl)
    ld = (wl.S + 63) // 64 * 64
    sc = torch.full((wl.B * q_count, ld), float("nan"), device="cuda")
    dsa.indexer_scores(shape, inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"],
                       q_begin, q_count, sc)
    return sc


def _check_rows(wl, inp, outs, rows_by_b, exact, tag="", lengths=None, v=None):
    """Oracle on the listed (b -> rows); compare index sets, outputs and LSE.
    lengths: per-sequence key counts (None: all S); v: separate value array
    [B, S, d_v] (float64) or None."""
    tau = _tau(wl)
    idx_gpu = outs.idx.cpu().numpy()
    out_gpu = outs.out.float().cpu().numpy()
    lse_gpu = outs.lse.cpu().numpy()
    stats = P.ErrStats()
    for b, rows in rows_by_b.items():
        seq = P.OracleSeq(inp, b)
        L = None if lengths is None else int(lengths[b])
        for t in rows:
            what = f"{tag} b={b} t={t}"
            sc, idx_o = P.oracle_select(seq, wl, t, L)
            P.check_selection(idx_gpu[b, t], idx_o, sc, exact, what)
            # end to end: oracle attention over the GPU's (validated) selection
            o_g, lse_g = P.oracle_attn(seq, wl, t, tau, idx_gpu[b, t], None if v is None else v[b])
            stats.add(P.check_attention(out_gpu[b, t], o_g, what))
            assert np.allclose(lse_gpu[b, t], lse_g, atol=2e-3, rtol=1e-4), what
    print(stats.line(tag))
    return stats


# ----------------------------------------------------------------- tiny, exact

def test_tiny_integer_workload_bit_exact():
    wl = WORKLOADS["tiny_prefill_256"]
    inp = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    # step A alone: integer mode -> scores exact
    sc = _scores_for_rows(wl, inp, 0, wl.T).cpu().numpy()
    d = O.from_inputs({k: v.cpu() for k, v in inp.items()})
    ref = O.indexer_scores(d["qd"], d["w"], d["kd"])
    for t in range(wl.T):
        assert np.array_equal(sc[t, : t + 1].astype(np.float64), ref[t, : t + 1]), t
    # step B alone on those scores: bit-exact index sets
    shape = dsa.make_shape(wl)
    idx = torch.full((1, wl.T, wl.k), -7, dtype=torch.int32, device="cuda")
    dsa.topk(shape, torch.from_numpy(sc).cuda(), 0, wl.T, idx)
    ref_idx = O.topk(ref, wl.k)
    gi = idx.cpu().numpy()[0]
    for t in range(wl.T):
        assert sorted(gi[t][gi[t] >= 0]) == sorted(ref_idx[t][ref_idx[t] >= 0]), t
        assert (gi[t] < 0).sum() == (ref_idx[t] < 0).sum()
    # step C alone, fed the oracle's indices
    out = torch.empty(1, wl.T, wl.H, wl.d_v, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, wl.T, wl.H, device="cuda")
    dsa.sparse_attn(shape, inp["q"], inp["kv"], torch.from_numpy(ref_idx.astype(np.int32))[None].cuda(), out, lse)
    o_ref, l_ref = O.sparse_attention(d["q"], d["kv"], ref_idx, wl.d_v, _tau(wl))
    P.check_attention(out.float().cpu().numpy()[0], o_ref, "tiny attn")
    assert np.allclose(lse.cpu().numpy()[0], l_ref, atol=1e-3)
    # whole path
    outs = _run_forward(wl, inp)
    assert np.array_equal(np.sort(outs.idx.cpu().numpy()[0], axis=1), np.sort(gi, axis=1))
    P.check_attention(outs.out.float().cpu().numpy()[0], o_ref, "tiny forward")


# ----------------------------------------------------------------- small ragged

SMALL = [
    # ragged prefill: several key tiles, a ragged tail, k < T, blocks of 96
    Workload("ragged_prefill", B=1, T=333, S=333, H_I=64, D_I=128, H=128, d_k=576, d_v=512,
             k=100, q_block=96, seed=7, needles=8),
    # batch of two short prefills, small indexer dims
    Workload("ragged_prefill_b2", B=2, T=200, S=200, H_I=8, D_I=64, H=16, d_k=576, d_v=512,
             k=64, q_block=64, seed=8),
    # chunked prefill: T < S, the queries are the last T positions
    Workload("chunked_prefill", B=1, T=130, S=700, H_I=16, D_I=128, H=64, d_k=576, d_v=512,
             k=128, q_block=128, seed=9, needles=4),
    # decode, S not a multiple of any tile, k > S for one configuration
    Workload("decode_small", B=3, T=1, S=1000, H_I=64, D_I=128, H=128, d_k=576, d_v=512,
             k=256, q_block=1, seed=10, needles=16),
    Workload("decode_k_covers_all", B=2, T=1, S=777, H_I=32, D_I=32, H=8, d_k=80, d_v=64,
             k=2048, q_block=1, seed=11),
    # decode with fewer than 128 heads on the MLA row (the decode kernel's
    # masked head rows) and a selection that ends inside its last split
    Workload("decode_h64_ragged_k", B=2, T=1, S=3000, H_I=16, D_I=128, H=64, d_k=576, d_v=512,
             k=1000, q_block=1, seed=12, needles=8),
]


@pytest.mark.parametrize("wl", SMALL, ids=[w.name for w in SMALL])
def test_small_shapes_full(wl):
    inp = make_inputs(wl, "cuda")
    outs = _run_forward(wl, inp)
    _check_rows(wl, inp, outs, {b: list(range(wl.T)) for b in range(wl.B)}, exact=False, tag=wl.name)
    # scores of step A for a block of rows
    q0, qc = max(0, wl.T - 50), min(50, wl.T)
    sc = _scores_for_rows(wl, inp, q0, qc).cpu().numpy()
    for b in range(wl.B):
        seq = P.OracleSeq(inp, b)
        for i in range(0, qc, 7):
            t = q0 + i
            qd, w, _ = seq.query(t)
            pos = O.query_pos(wl.T, wl.S, t)
            ref = O.indexer_row(qd, w, seq.kd, pos)
            P.check_scores(sc[b * qc + i], ref, P.score_abs_scale(seq, wl, t), False, f"{wl.name} b={b} t={t}")
            assert np.all(np.isnan(sc[b * qc + i, pos + 1: wl.S])), "wrote past the causal limit"


def test_prefill_and_decode_entry_points_agree():
    wl = Workload("agree", B=1, T=1, S=900, H_I=64, D_I=128, H=128, d_k=576, d_v=512, k=300,
                  q_block=1, seed=12, needles=8)
    inp = make_inputs(wl, "cuda")
    a = _run_forward(wl, inp, "dsa_decode")
    b = _run_forward(wl, inp, "dsa_prefill")
    assert np.array_equal(np.sort(a.idx.cpu().numpy(), -1), np.sort(b.idx.cpu().numpy(), -1))
    P.check_attention(a.out.float().cpu().numpy(), b.out.double().cpu().numpy(), "decode vs prefill")


def test_attention_padding_and_duplicates():
    wl = Workload("dup", B=1, T=4, S=64, H_I=4, D_I=32, H=128, d_k=576, d_v=512, k=16, q_block=4, seed=13)
    inp = make_inputs(wl, "cuda")
    idx = np.full((1, 4, 16), -1, np.int32)
    idx[0, 0, :3] = [60, 5, 5]                 # duplicate counted twice
    idx[0, 1, 7] = 61                          # single key, rest empty
    idx[0, 2, :] = np.arange(16)[::-1] * 3     # permuted
    idx[0, 3, ::2] = np.arange(8) + 40
    shape = dsa.make_shape(wl)
    out = torch.empty(1, 4, wl.H, wl.d_v, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, 4, wl.H, device="cuda")
    dsa.sparse_attn(shape, inp["q"], inp["kv"], torch.from_numpy(idx).cuda(), out, lse)
    assert dsa.device_error()[0] == 0
    d = O.from_inputs({k: v.cpu() for k, v in inp.items()})
    o_ref, l_ref = O.sparse_attention(d["q"], d["kv"], idx[0], wl.d_v, _tau(wl))
    P.check_attention(out.float().cpu().numpy()[0], o_ref, "dup/pad")
    assert np.allclose(lse.cpu().numpy()[0], l_ref, atol=2e-3)


# ----------------------------------------------------------------- full workloads

@pytest.mark.parametrize("name", ["decode_32k_b32", "decode_128k_b8"])
def test_decode_workloads_full(name):
    wl = WORKLOADS[name]
    inp = make_inputs(wl, "cuda")
    outs = _run_forward(wl, inp)
    _check_rows(wl, inp, outs, {b: [0] for b in range(wl.B)}, exact=False, tag=name)


@pytest.mark.parametrize("name", ["decode_32k_b32", "decode_128k_b8"])
def test_decode_indexer_scores_every_row_in_full(name):
    """Every decode row's whole score row (32768 or 131072 entries), element by
    element, in the launch configuration dsa_forward uses for decode (short key
    runs per work item, double-buffered query tiles)."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, "cuda")
    sc = _scores_for_rows(wl, inp, 0, 1).cpu().numpy()
    for b in range(wl.B):
        seq = P.OracleSeq(inp, b)
        qd, w, _ = seq.query(0)
        ref = O.indexer_row(qd, w, seq.kd, wl.S - 1)
        P.check_scores(sc[b], ref, P.score_abs_scale(seq, wl, 0), False, f"{name} b={b}")


# stratified samples of the prefill workloads: about 1.1-1.3K rows each
PREFILL_SAMPLES = {name: P.sample_rows(WORKLOADS[name], 1024) for name in ("prefill_8k", "prefill_128k")}


@pytest.mark.parametrize("name", list(PREFILL_SAMPLES),
                         ids=[f"{n}-{len(r)}rows" for n, r in PREFILL_SAMPLES.items()])
def test_prefill_workloads_sampled(name):
    wl = WORKLOADS[name]
    inp = make_inputs(wl, "cuda")
    outs = _run_forward(wl, inp)
    rows = PREFILL_SAMPLES[name]
    assert len(rows) >= 1000
    _check_rows(wl, inp, outs, {0: rows}, exact=False, tag=name)
    # rows with fewer visible keys than k keep all of them (dense)
    idx = outs.idx[0, : wl.k].cpu().numpy()
    for t in (0, 1, 100, wl.k - 1):
        assert sorted(idx[t][idx[t] >= 0]) == list(range(t + 1))


def test_prefill_128k_indexer_block_scores():
    """Whole score rows of 32 rows of one 4096-row query block of the 128K
    prefill (the launch configuration of the benchmark: a full block, paired
    key tiles, 16-query items), element by element: the first and last rows
    of the block, rows on both sides of item (16-row) boundaries, random
    rows."""
    wl = WORKLOADS["prefill_128k"]
    inp = make_inputs(wl, "cuda")
    q0 = 16 * wl.q_block                   # rows 65536 .. 69631
    sc = _scores_for_rows(wl, inp, q0, wl.q_block)
    rng = np.random.default_rng(3)
    picks = sorted(set([0, 1, 15, 16, 17, 2047, 2048, wl.q_block - 2, wl.q_block - 1] +
                       rng.integers(0, wl.q_block, 23).tolist()))
    seq = P.OracleSeq(inp, 0)
    for i in picks:
        t = q0 + i
        row = sc[i].cpu().numpy()
        qd, w, _ = seq.query(t)
        ref = O.indexer_row(qd, w, seq.kd, t)
        P.check_scores(row, ref, P.score_abs_scale(seq, wl, t), False, f"prefill_128k block t={t}")
        assert np.all(np.isnan(row[t + 1: wl.S])), "wrote past the causal limit"
    assert len(picks) >= 30


# ----------------------------------------------------------------- errors

def test_argument_errors_are_reported():
    wl = WORKLOADS["tiny_prefill_256"]
    shape = dsa.make_shape(wl, H=12)       # H % 8 != 0
    assert dsa.workspace_size(shape) == 0
    inp = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    outs = dsa.alloc_outputs(wl)
    good = dsa.make_shape(wl)
    ws = dsa.alloc_workspace(good)
    with pytest.raises(dsa.DsaError) as e:
        dsa.forward(shape, inp, outs.out, outs.lse, outs.idx, ws)
    assert e.value.code == 2
    with pytest.raises(dsa.DsaError) as e:
        dsa.forward(good, inp, outs.out, outs.lse, outs.idx, ws[:16])
    assert e.value.code == 3
    bad = dsa.make_shape(wl, T=wl.S + 1)
    with pytest.raises(dsa.DsaError) as e:
        dsa.forward(bad, inp, outs.out, outs.lse, outs.idx, ws)
    assert e.value.code == 1


def test_out_of_range_index_is_reported_not_read():
    wl = Workload("oob", B=1, T=2, S=64, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=4, q_block=2, seed=14)
    inp = make_inputs(wl, "cuda")
    idx = torch.tensor([[[0, 1, 64 + 5, -1], [3, -1, -1, -1]]], dtype=torch.int32, device="cuda")
    out = torch.empty(1, 2, wl.H, wl.d_v, dtype=torch.bfloat16, device="cuda")
    dsa.sparse_attn(dsa.make_shape(wl), inp["q"], inp["kv"], idx, out)
    st, det = dsa.device_error()
    assert st == 6 and (det & 0xF0) == 0x30
    assert dsa.device_error()[0] == 0   # cleared by the read


def test_bounded_wait_reports_timeout():
    """A wait that can never be satisfied gives up after the configured limit
    and reports DSA_ERR_TIMEOUT; the context stays usable afterwards."""
    import time
    dsa.set_wait_timeout_us(20000)            # 20 ms
    try:
        t0 = time.perf_counter()
        dsa.selftest_wait_timeout()
        st, det = dsa.device_error()
        dt = time.perf_counter() - t0
    finally:
        dsa.set_wait_timeout_us(0)           # back to the default
    assert st == 5 and (det & 0xFF) == 0x50
    assert dt < 5.0
    assert dsa.device_error()[0] == 0
    # the library still works after the timeout
    wl = WORKLOADS["tiny_prefill_256"]
    inp = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    _run_forward(wl, inp)
