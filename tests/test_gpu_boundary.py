"""GPU parity of the boundary's generalisations, through the C ABI, against
the FP64 oracle:

* per-sequence lengths (dsa_shape.seqlens): a ragged decode batch whose
  sequences hold 777, 5000, 32768 and 131072 keys, and chunked prefills over
  contexts of different lengths; the oracle runs each sequence on its own
  length;
* values kept apart from the keys (dsa_inputs.v / v_or_null);
* paged key caches (block_table, page sizes 16, 64 and 256): scores must equal
  the contiguous run's bit for bit, selections and outputs the oracle's;
* the dense form (dsa_dense_attn, and dsa_forward's rows whose visible keys
  all fit in k) against the oracle's dense causal attention;
* lengths and block-table entries out of range are reported on the device,
  never read.
"""
import numpy as np
import pytest
import torch

from long_context_05_b200 import dsa
from long_context_05_b200.inputs import Workload, make_inputs, to_paged
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


def _forward(wl, inp, shape):
    ws = dsa.alloc_workspace(shape)
    outs = dsa.alloc_outputs(wl)
    outs.idx.fill_(-7)
    outs.out.fill_(7.0)
    dsa.forward(shape, inp, outs.out, outs.lse, outs.idx, ws)
    st, det = dsa.device_error()
    assert st == 0, f"device error {dsa.STATUS.get(st)} detail {det:#x}"
    return outs


def _check_all_rows(wl, inp, outs, lengths=None, v=None, tag=""):
    tau = _tau(wl)
    idx_gpu = outs.idx.cpu().numpy()
    out_gpu = outs.out.float().cpu().numpy()
    lse_gpu = outs.lse.cpu().numpy()
    vd = None if v is None else O.bf16_decode(P.u16(v))
    stats = P.ErrStats()
    for b in range(wl.B):
        seq = P.OracleSeq(inp, b)
        L = wl.S if lengths is None else int(lengths[b])
        for t in range(wl.T):
            what = f"{tag} b={b} L={L} t={t}"
            sc, idx_o = P.oracle_select(seq, wl, t, L)
            P.check_selection(idx_gpu[b, t], idx_o, sc, False, what)
            o_g, l_g = P.oracle_attn(seq, wl, t, tau, idx_gpu[b, t], None if vd is None else vd[b])
            stats.add(P.check_attention(out_gpu[b, t], o_g, what))
            assert np.allclose(lse_gpu[b, t], l_g, atol=2e-3, rtol=1e-4), what
    print(stats.line(tag))


# ----------------------------------------------------------------- lengths

def test_ragged_decode_batch_against_each_sequence_alone():
    lengths = [777, 5000, 32768, 131072]
    wl = Workload("ragged_decode", B=4, T=1, S=131072, H_I=64, D_I=128, H=128, d_k=576, d_v=512, k=2048,
                  q_block=1, seed=31, needles=64)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    sl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    shape = dsa.make_shape(wl, seqlens=sl)
    outs = _forward(wl, inp, shape)
    _check_all_rows(wl, inp, outs, lengths, tag="ragged decode")
    # every row's whole score row, and nothing written at or past its length
    ld = (wl.S + 63) // 64 * 64
    sc = torch.full((wl.B, ld), float("nan"), device="cuda")
    dsa.indexer_scores(shape, inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], 0, 1, sc)
    assert dsa.device_error()[0] == 0
    sc = sc.cpu().numpy()
    for b, L in enumerate(lengths):
        seq = P.OracleSeq(inp, b)
        qd, w, _ = seq.query(0)
        ref = O.indexer_row(qd, w, seq.kd, L - 1)
        P.check_scores(sc[b], ref, P.score_abs_scale(seq, wl, 0, L), False, f"ragged scores b={b}")
        assert np.all(np.isnan(sc[b, L:wl.S])), f"b={b}: scores written at or past the length"


def test_ragged_chunked_prefill():
    """T = 100 new queries per sequence over contexts of 100, 1500 and 3000
    keys (pos = L_b - T + t), in 64-row query blocks."""
    lengths = [100, 1500, 3000]
    wl = Workload("ragged_chunk", B=3, T=100, S=3000, H_I=16, D_I=64, H=64, d_k=576, d_v=512, k=256,
                  q_block=64, seed=32, needles=8)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    sl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    outs = _forward(wl, inp, dsa.make_shape(wl, seqlens=sl))
    _check_all_rows(wl, inp, outs, lengths, tag="ragged chunked prefill")


def test_length_out_of_range_is_reported():
    wl = Workload("badlen", B=2, T=1, S=1000, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=64, q_block=1, seed=33)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    sl = torch.tensor([500, 1001], dtype=torch.int32, device="cuda")   # 1001 > S
    shape = dsa.make_shape(wl, seqlens=sl)
    ws = dsa.alloc_workspace(shape)
    outs = dsa.alloc_outputs(wl)
    dsa.forward(shape, inp, outs.out, outs.lse, outs.idx, ws)
    st, det = dsa.device_error()
    assert st == 6 and (det >> 8) & 0xFF == 0xB0, (st, hex(det))
    assert dsa.device_error()[0] == 0


# ----------------------------------------------------------------- separate V

SEPV = [
    Workload("sepv_prefill", B=1, T=300, S=300, H_I=64, D_I=128, H=128, d_k=576, d_v=512, k=100,
             q_block=128, seed=34, needles=8),
    Workload("sepv_decode", B=3, T=1, S=4000, H_I=32, D_I=128, H=128, d_k=576, d_v=512, k=512,
             q_block=1, seed=35, needles=16),
    Workload("sepv_small_dims", B=2, T=90, S=90, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=40, q_block=90,
             seed=36),
]


@pytest.mark.parametrize("wl", SEPV, ids=[w.name for w in SEPV])
def test_separate_values(wl):
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    g = torch.Generator(device="cuda")
    g.manual_seed(wl.seed + 100)
    inp["v"] = torch.randn(wl.B, wl.S, wl.d_v, generator=g, device="cuda").bfloat16()
    outs = _forward(wl, inp, dsa.make_shape(wl))
    _check_all_rows(wl, inp, outs, v=inp["v"], tag=wl.name)
    # step C alone, fed the GPU's selection, agrees with the whole path
    out2 = torch.empty_like(outs.out)
    shape = dsa.make_shape(wl)
    dsa.sparse_attn(shape, inp["q"], inp["kv"], outs.idx, out2, None, dsa.alloc_workspace(shape), v=inp["v"])
    assert dsa.device_error()[0] == 0
    P.check_attention(out2.float().cpu().numpy(), outs.out.double().cpu().numpy(), wl.name + " step C")


# ----------------------------------------------------------------- paged caches

def _paged(inp, wl, page_size, seed):
    """Key-side arrays in page pools, a random page order, spare pages and -1
    past each sequence's pages."""
    return to_paged(inp, wl, page_size, seed)


PAGED = [
    (Workload("paged_decode", B=3, T=1, S=5000, H_I=64, D_I=128, H=128, d_k=576, d_v=512, k=512, q_block=1,
              seed=37, needles=16), 64),
    (Workload("paged_decode_p16", B=2, T=1, S=3000, H_I=16, D_I=64, H=64, d_k=576, d_v=512, k=256,
              q_block=1, seed=38, needles=8), 16),
    (Workload("paged_chunk_p256", B=2, T=64, S=1200, H_I=8, D_I=128, H=32, d_k=576, d_v=512, k=200,
              q_block=32, seed=39, needles=8), 256),
]


@pytest.mark.parametrize("wl,page", PAGED, ids=[w.name for w, _ in PAGED])
def test_paged_caches(wl, page):
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    lengths = [wl.S - 37 * b for b in range(wl.B)]          # ragged too
    sl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    pin, table, num_pages = _paged(inp, wl, page, wl.seed)
    flat = dsa.make_shape(wl, seqlens=sl)
    paged = dsa.make_shape(wl, seqlens=sl, block_table=table, page_size=page, num_pages=num_pages)
    # step A: identical scores from the pool
    ld = (wl.S + 63) // 64 * 64
    a = torch.full((wl.B * wl.T, ld), float("nan"), device="cuda")
    b = torch.full((wl.B * wl.T, ld), float("nan"), device="cuda")
    dsa.indexer_scores(flat, inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], 0, wl.T, a)
    dsa.indexer_scores(paged, pin["q_I"], pin["q_scale"], pin["w"], pin["k_I"], pin["k_scale"], 0, wl.T, b)
    assert dsa.device_error()[0] == 0
    assert torch.equal(torch.nan_to_num(a, nan=-1e30), torch.nan_to_num(b, nan=-1e30))
    # the whole path: oracle on the logical (unpaged) arrays
    outs = _forward(wl, pin, paged)
    _check_all_rows(wl, inp, outs, lengths, tag=wl.name)


def test_unmapped_page_is_reported_not_read():
    wl = Workload("badpage", B=1, T=1, S=256, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=32, q_block=1, seed=40)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    pin, table, num_pages = _paged(inp, wl, 64, 1)
    table[0, 2] = num_pages + 5                               # a page that holds keys, out of range
    shape = dsa.make_shape(wl, block_table=table, page_size=64, num_pages=num_pages)
    ws = dsa.alloc_workspace(shape)
    outs = dsa.alloc_outputs(wl)
    dsa.forward(shape, pin, outs.out, outs.lse, outs.idx, ws)
    st, det = dsa.device_error()
    assert st == 6, (st, hex(det))
    assert dsa.device_error()[0] == 0


# ----------------------------------------------------------------- dense form

DENSE = [
    Workload("dense_prefill", B=1, T=700, S=700, H_I=4, D_I=32, H=128, d_k=576, d_v=512, k=64, q_block=700,
             seed=41),
    Workload("dense_prefill_small", B=2, T=150, S=150, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=16, q_block=150,
             seed=42),
    Workload("dense_decode_long", B=2, T=1, S=20000, H_I=4, D_I=32, H=128, d_k=576, d_v=512, k=64,
             q_block=1, seed=43),
]


@pytest.mark.parametrize("wl", DENSE, ids=[w.name for w in DENSE])
def test_dense_attention_entry_point(wl):
    """dsa_dense_attn: every visible key, whatever k, against the oracle's
    textbook dense causal attention."""
    inp = make_inputs(wl, "cuda")
    shape = dsa.make_shape(wl)
    out = torch.full((wl.B, wl.T, wl.H, wl.d_v), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(wl.B, wl.T, wl.H, device="cuda")
    dsa.dense_attn(shape, inp["q"], inp["kv"], out, lse, dsa.alloc_workspace(shape))
    assert dsa.device_error()[0] == 0
    tau = _tau(wl)
    og, lg = out.float().cpu().numpy(), lse.cpu().numpy()
    stats = P.ErrStats()
    rows = range(wl.T) if wl.T <= 200 else sorted(set(list(range(70)) + list(range(wl.T - 70, wl.T)) +
                                                       list(range(70, wl.T - 70, 9))))
    for b in range(wl.B):
        d = O.from_inputs({k: v[b:b + 1].cpu() for k, v in inp.items() if k != "needle_pos"})
        for t in rows:
            pos = O.query_pos(wl.T, wl.S, t)
            o_ref, l_ref = O.dense_causal_attention_row(d["q"][t], d["kv"], pos, wl.d_v, tau)
            stats.add(P.check_attention(og[b, t], o_ref, f"{wl.name} b={b} t={t}"))
            assert np.allclose(lg[b, t], l_ref, atol=2e-3, rtol=1e-4)
    print(stats.line(wl.name))


def test_forward_rows_within_k_skip_indexer():
    """A prefill of 1500 tokens with k = 2048: every row keeps all its visible
    keys, so dsa_forward writes idx = 0..pos without running steps A and B
    (two launches: the index fill and the attention) and the output is dense
    causal attention."""
    wl = Workload("short_prefill", B=1, T=1500, S=1500, H_I=64, D_I=128, H=128, d_k=576, d_v=512, k=2048,
                  q_block=512, seed=44, needles=8)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    n0 = dsa.launch_count()
    outs = _forward(wl, inp, dsa.make_shape(wl))
    assert dsa.launch_count() - n0 == 2
    idx = outs.idx.cpu().numpy()[0]
    for t in range(wl.T):
        assert np.array_equal(np.sort(idx[t][idx[t] >= 0]), np.arange(t + 1)), t
    d = O.from_inputs({k: v.cpu() for k, v in inp.items()})
    og = outs.out.float().cpu().numpy()[0]
    stats = P.ErrStats()
    for t in list(range(0, wl.T, 11)) + [wl.T - 1]:
        o_ref, _ = O.dense_causal_attention_row(d["q"][t], d["kv"], t, wl.d_v, _tau(wl))
        stats.add(P.check_attention(og[t], o_ref, f"short prefill t={t}"))
    print(stats.line("short prefill"))


def test_prefill_in_query_blocks_equals_one_call():
    """A prefill run as one dsa_forward call per query block (each a chunked
    prefill over the whole key cache with seqlens = the block's end, as the
    bench's end-to-end measurement runs it) selects the same keys for every
    row as one call over all rows, and its outputs agree."""
    wl = Workload("blocked_prefill", B=1, T=3000, S=3000, H_I=64, D_I=128, H=128, d_k=576, d_v=512, k=512,
                  q_block=1024, seed=45, needles=8)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    ref = _forward(wl, inp, dsa.make_shape(wl))
    got = dsa.alloc_outputs(wl)
    for s0 in range(0, wl.T, wl.q_block):
        c = min(wl.q_block, wl.T - s0)
        end = torch.tensor([s0 + c], dtype=torch.int32, device="cuda")
        shape = dsa.make_shape(wl.with_(T=c, q_block=c), mode=dsa.DSA_PREFILL, seqlens=end)
        part = {n: inp[n][:, s0:s0 + c] for n in ("q_I", "q_scale", "w", "q")}
        part.update({n: inp[n] for n in ("k_I", "k_scale", "kv")})
        dsa.forward(shape, part, got.out[:, s0:s0 + c], got.lse[:, s0:s0 + c], got.idx[:, s0:s0 + c],
                    dsa.alloc_workspace(shape))
    st, det = dsa.device_error()
    assert st == 0, (st, hex(det))
    a, b = got.idx.cpu().numpy()[0], ref.idx.cpu().numpy()[0]
    for t in range(wl.T):
        assert np.array_equal(np.sort(a[t][a[t] >= 0]), np.sort(b[t][b[t] >= 0])), t
    # the same sets, possibly in another slot order: outputs agree to FP32
    # summation order, LSE to 1e-4
    assert torch.allclose(got.out.float(), ref.out.float(), atol=2e-2, rtol=2e-2)
    assert torch.allclose(got.lse, ref.lse, atol=1e-4, rtol=1e-5)


def test_indexer_single_query_launch_equals_full_launch():
    """dsa_indexer_scores for one query row of a prefill (the one-query form:
    N = 64 sub-tiles, two CTAs per SM) gives that row's scores bit for bit as
    a launch over all rows does (the same FP8 products, K order and head
    order), on every visible key."""
    wl = Workload("one_row", B=2, T=40, S=5000, H_I=64, D_I=128, H=8, d_k=80, d_v=64, k=256, q_block=40, seed=47)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    shape = dsa.make_shape(wl)
    ld = (wl.S + 63) // 64 * 64
    full = torch.full((wl.B * wl.T, ld), float("nan"), device="cuda")
    dsa.indexer_scores(shape, inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], 0, wl.T, full)
    for t in (0, 17, wl.T - 1):
        one = torch.full((wl.B, ld), float("nan"), device="cuda")
        dsa.indexer_scores(shape, inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], t, 1, one)
        st, det = dsa.device_error()
        assert st == 0, (st, hex(det))
        n = wl.S - wl.T + t + 1
        for b in range(wl.B):
            a = one[b, :n].cpu().numpy()
            r = full[b * wl.T + t, :n].cpu().numpy()
            assert np.array_equal(a, r), (t, b, np.max(np.abs(a - r)))
