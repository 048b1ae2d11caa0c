"""One sequence over several parts, on one GPU, through the C ABI.

The parts of a key-split decode and the zig-zag row blocks of a prefill are
run one after another in this process (the all-gathers become stacking), with
the same host orchestration (long_context_05_b200.parallel) that drives one
process per GPU.  No kernel waits on another part's kernel, so emulating the
parts on one device is exact.  Checks:

* key-split decode with 2 and 4 parts: the merged selection equals the
  unsplit dsa_forward's selection exactly (each part's scores are the same
  FP32 numbers), and the combined output matches the FP64 oracle;
* zig-zag prefill blocks of one sequence over 2 parts: the union of rows
  equals the unsplit run's selection and matches the oracle.
"""
import numpy as np
import pytest
import torch

from long_context_05_b200 import dsa
from long_context_05_b200.inputs import Workload, make_inputs
from long_context_05_b200.parallel import DsaKeySplitCompute, DsaRowsCompute, KeySplitDecode, prefill_rows, \
    zigzag_blocks
from oracle import dsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.lib()


def _unsplit(wl, inp):
    shape = dsa.make_shape(wl)
    ws = dsa.alloc_workspace(shape)
    outs = dsa.alloc_outputs(wl)
    dsa.forward(shape, inp, outs.out, outs.lse, outs.idx, ws)
    assert dsa.device_error()[0] == 0
    return outs


@pytest.mark.parametrize("parts", [2, 4])
def test_key_split_decode(parts):
    wl = Workload("keysplit", B=4, T=1, S=40000, H_I=64, D_I=128, H=128, d_k=576, d_v=512, k=2048, q_block=1,
                  seed=51, needles=64)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    ref = _unsplit(wl, inp)
    runs, computes = [], []
    for r in range(parts):
        ks = KeySplitDecode(wl.S, parts, r)
        loc = {n: inp[n] for n in ("q_I", "q_scale", "w", "q")}
        loc.update({n: inp[n][:, ks.s0:ks.s0 + ks.cnt].contiguous() for n in ("k_I", "k_scale", "kv")})
        runs.append(ks)
        computes.append(DsaKeySplitCompute(wl.with_(S=ks.cnt), loc, wl.S))
    # phases in lockstep, stacking in place of the all-gathers
    cand = [ks.select(c) for ks, c in zip(runs, computes)]
    cs = torch.stack([c[0].clone() for c in cand])
    ci = torch.stack([c[1].clone() for c in cand])
    merged = [ks.merge(c, cs, ci) for ks, c in zip(runs, computes)]
    att = [ks.attend(c, m[1]) for ks, c, m in zip(runs, computes, merged)]
    o_all = torch.stack([a[0].clone() for a in att])
    l_all = torch.stack([a[1].clone() for a in att])
    out, lse = computes[0].combine(o_all, l_all)
    st, det = dsa.device_error()
    assert st == 0, (st, hex(det))
    # every part merges to the same selection (as sets: slot order is free)
    gidx = merged[0][0].cpu().numpy()
    for m in merged[1:]:
        assert torch.equal(torch.sort(m[0], dim=-1).values, torch.sort(merged[0][0], dim=-1).values)
    ref_idx = ref.idx.cpu().numpy()[:, 0]
    og, lg = out.float().cpu().numpy()[:, 0], lse.cpu().numpy()[:, 0]
    stats = P.ErrStats()
    for b in range(wl.B):
        assert sorted(gidx[b][gidx[b] >= 0].tolist()) == sorted(ref_idx[b][ref_idx[b] >= 0].tolist()), b
        seq = P.OracleSeq(inp, b)
        sc, idx_o = P.oracle_select(seq, wl, 0)
        P.check_selection(gidx[b], idx_o, sc, False, f"keysplit b={b}")
        o_ref, l_ref = P.oracle_attn(seq, wl, 0, float(O.default_tau(wl.d_k)), gidx[b])
        stats.add(P.check_attention(og[b], o_ref, f"keysplit/{parts} b={b}"))
        assert np.allclose(lg[b], l_ref, atol=2e-3, rtol=1e-4)
    print(stats.line(f"key-split decode over {parts} parts"))


def test_zigzag_prefill_rows():
    wl = Workload("zigzag", B=1, T=3000, S=3000, H_I=64, D_I=128, H=128, d_k=576, d_v=512, k=512,
                  q_block=1024, seed=52, needles=16)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    ref = _unsplit(wl, inp)
    comp = DsaRowsCompute(wl, inp)
    got = {}
    for r in range(2):
        for s, c, (out, lse, idx) in prefill_rows(comp, zigzag_blocks(wl.T, 2, r)):
            for i in range(c):
                got[s + i] = (idx[0, i].cpu().numpy(), out[0, i].float().cpu().numpy())
    assert dsa.device_error()[0] == 0
    assert sorted(got) == list(range(wl.T))
    ref_idx = ref.idx.cpu().numpy()[0]
    seq = P.OracleSeq(inp, 0)
    stats = P.ErrStats()
    for t in range(wl.T):
        assert sorted(got[t][0][got[t][0] >= 0].tolist()) == sorted(ref_idx[t][ref_idx[t] >= 0].tolist()), t
    for t in list(range(0, wl.T, 37)) + [wl.T - 1]:
        o_ref, _ = P.oracle_attn(seq, wl, t, float(O.default_tau(wl.d_k)), got[t][0])
        stats.add(P.check_attention(got[t][1], o_ref, f"zigzag t={t}"))
    print(stats.line("zig-zag prefill rows over 2 parts"))
