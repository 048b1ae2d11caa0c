"""dsa_select: steps A and B without the score tile, through the C ABI.

In prefill over long contexts the selection keeps only candidates at or
above a per-row threshold taken from a key sample, and rows the candidates
cannot settle are repaired from a fully scored row.  The scores of either way
are the same FP32 numbers (the same MMAs and epilogue), so the selection must
equal the materialised path's (dsa_indexer_scores + dsa_topk) exactly; rows
are also checked against the FP64 oracle.  Two adversarial inputs force the
repair: every key equal (the candidate list overflows) and keys that score
zero except the sampled ones (too few candidates).
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


def _materialised(wl, inp, shape, q0, cnt):
    ld = (wl.S + 63) // 64 * 64
    sc = torch.empty(wl.B * cnt, ld, device="cuda")
    dsa.indexer_scores(shape, inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], q0, cnt, sc)
    idx = torch.full((wl.B, wl.T, wl.k), -7, dtype=torch.int32, device="cuda")
    dsa.topk(shape, sc, q0, cnt, idx)
    return idx


def _fused(wl, inp, shape, q0, cnt):
    idx = torch.full((wl.B, wl.T, wl.k), -9, dtype=torch.int32, device="cuda")
    dsa.select(shape, inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], q0, cnt, idx,
               dsa.alloc_workspace(shape, fused=True))
    st, det = dsa.device_error()
    assert st == 0, (st, hex(det))
    return idx


def _same_sets(a, b, rows):
    a, b = a.cpu().numpy(), b.cpu().numpy()
    for bb in range(a.shape[0]):
        for t in rows:
            x, y = a[bb, t], b[bb, t]
            assert (x < 0).sum() == (y < 0).sum(), (bb, t)
            assert np.array_equal(np.sort(x[x >= 0]), np.sort(y[y >= 0])), (bb, t)


def test_fused_selection_equals_materialised_128k_rows():
    wl = WORKLOADS["prefill_chunk_128k"]                 # the last 512 queries of a 128K prefill
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    shape = dsa.make_shape(wl)
    ref = _materialised(wl, inp, shape, 0, wl.T)
    got = _fused(wl, inp, shape, 0, wl.T)
    _same_sets(got, ref, range(wl.T))
    # and against the oracle on a few full rows
    seq = P.OracleSeq(inp, 0)
    g = got.cpu().numpy()[0]
    for t in (0, 1, 255, 256, wl.T - 1):
        sc, idx_o = P.oracle_select(seq, wl, t)
        P.check_selection(g[t], idx_o, sc, False, f"fused t={t}")


def test_forward_takes_the_fused_selection_in_a_small_workspace():
    """dsa_forward given dsa_select_workspace_size bytes (no room for the
    score tile) selects through the fused path: the same selection and the
    same output as with the full workspace."""
    wl = WORKLOADS["prefill_chunk_128k"]
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    shape = dsa.make_shape(wl)
    small, full = dsa.alloc_workspace(shape, fused=True), dsa.alloc_workspace(shape)
    assert small.numel() < full.numel() // 2        # 108 MiB instead of the 256 MiB score tile
    a, b = dsa.alloc_outputs(wl), dsa.alloc_outputs(wl)
    dsa.forward(shape, inp, a.out, a.lse, a.idx, small)
    dsa.forward(shape, inp, b.out, b.lse, b.idx, full)
    st, det = dsa.device_error()
    assert st == 0, (st, hex(det))
    _same_sets(a.idx, b.idx, range(wl.T))
    # the same sets in another slot order: outputs agree to FP32 summation order
    assert torch.allclose(a.out.float(), b.out.float(), atol=2e-2, rtol=2e-2)
    with pytest.raises(dsa.DsaError):
        dsa.forward(shape, inp, a.out, a.lse, a.idx, small[: small.numel() - 256])


def test_fused_selection_block_of_128k_prefill():
    wl = WORKLOADS["prefill_128k"]
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    shape = dsa.make_shape(wl)
    q0 = 20 * wl.q_block
    ref = _materialised(wl, inp, shape, q0, wl.q_block)
    got = _fused(wl, inp, shape, q0, wl.q_block)
    _same_sets(got, ref, range(q0, q0 + wl.q_block))


def _adversarial(kind):
    wl = Workload(f"select_{kind}", B=1, T=64, S=32768, H_I=8, D_I=64, H=8, d_k=80, d_v=64, k=2048, q_block=64,
                  seed=61)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    if kind == "all_equal":
        inp["k_I"][:] = inp["k_I"][:, :1].clone()             # one key row everywhere: every score ties
        inp["k_scale"][:] = inp["k_scale"][:, :1].clone()
    else:
        keep = torch.zeros(wl.S, dtype=torch.bool, device="cuda")
        keep[::32] = True                                     # the rows the 32-stride sample reads
        inp["k_I"][:, ~keep] = 0                              # score exactly 0 elsewhere
    return wl, inp


@pytest.mark.parametrize("kind", ["all_equal", "sample_only"])
def test_fused_selection_repairs_rows(kind):
    wl, inp = _adversarial(kind)
    shape = dsa.make_shape(wl)
    got = _fused(wl, inp, shape, 0, wl.T)
    ref = _materialised(wl, inp, shape, 0, wl.T)
    _same_sets(got, ref, range(wl.T))
    seq = P.OracleSeq(inp, 0)
    g = got.cpu().numpy()[0]
    for t in (0, 31, wl.T - 1):
        sc, idx_o = P.oracle_select(seq, wl, t)
        P.check_selection(g[t], idx_o, sc, kind == "all_equal", f"{kind} t={t}")
    if kind == "all_equal":
        # every score ties: the lowest indices win
        assert np.array_equal(np.sort(g[0]), np.arange(wl.k))
