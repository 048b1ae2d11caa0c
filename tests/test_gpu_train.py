"""Indexer training kernels, through the C ABI, against the FP64 oracle.

Warm-up (dense): the target is the main attention's weights over every
visible key, averaged over heads; the loss is KL(target || softmax(I)).
Sparse stage: the same over the selected set.  Checked: the target rows, the
per-row loss and dL/dI, and dL/dw, dL/dq_I, dL/dk_I (on the dequantised
operands) against the oracle's chain rule, with tolerances from FP32
accumulation: target and dL/dI 1e-5 absolute (entries are probabilities),
loss 1e-4 relative, input gradients 1e-3 of the gradient's largest entry
(sums of a few thousand FP32 terms).
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


def _close(g, r, tol, what):
    err = np.max(np.abs(g - r)) if r.size else 0.0
    scale = max(np.max(np.abs(r)), 1e-30)
    assert err <= tol * scale, f"{what}: max err {err:.3e} vs scale {scale:.3e}"


@pytest.mark.parametrize("sparse", [False, True], ids=["warmup_dense", "sparse_set"])
def test_indexer_training_step(sparse):
    # integer-valued FP8 indexer operands with unit scales: every dot product
    # q_j . k_s is an exact integer on both sides, so the ReLU's mask [dot > 0]
    # is the same decision in FP32 and FP64 and only summation order differs
    wl = Workload("train", B=1, T=256, S=1024, H_I=64, D_I=128, H=128, d_k=576, d_v=512, k=128, q_block=256,
                  seed=71, int_mode=True)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    shape = dsa.make_shape(wl)
    ws = dsa.alloc_workspace(shape)
    rows = wl.B * wl.T
    ld = (wl.S + 63) // 64 * 64
    # main attention over the same keys (its lse feeds the target)
    out = torch.empty(1, wl.T, wl.H, wl.d_v, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, wl.T, wl.H, device="cuda")
    idx = None
    if sparse:
        outs = dsa.alloc_outputs(wl)
        dsa.forward(shape, inp, outs.out, outs.lse, outs.idx, ws)
        idx, lse = outs.idx, outs.lse
    else:
        dsa.dense_attn(shape, inp["q"], inp["kv"], out, lse, ws)
    scores = torch.zeros(rows, ld, device="cuda")
    dsa.indexer_scores(shape, inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], 0, wl.T, scores)
    target = torch.zeros(rows, ld, device="cuda")
    dsa.kl_target(shape, inp["q"], inp["kv"], lse, 0, wl.T, target, idx)
    grad = torch.zeros(rows, ld, device="cuda")
    loss = torch.zeros(rows, device="cuda")
    dsa.indexer_kl(shape, scores, target, 0, wl.T, grad, loss, idx)
    dq = torch.zeros(1, wl.T, wl.H_I, wl.D_I, device="cuda")
    dw = torch.zeros(1, wl.T, wl.H_I, device="cuda")
    dk = torch.zeros(1, wl.S, wl.D_I, device="cuda")
    dsa.indexer_backward(shape, inp["q_I"], inp["q_scale"], inp["w"], inp["k_I"], inp["k_scale"], grad, 0, wl.T,
                         dq, dw, dk, idx)
    st, det = dsa.device_error()
    assert st == 0, (st, hex(det))
    tg, gg, lg = target.cpu().numpy(), grad.cpu().numpy(), loss.cpu().numpy()
    dqg, dwg, dkg = dq.cpu().numpy()[0], dw.cpu().numpy()[0], dk.cpu().numpy()[0]
    idx_np = None if idx is None else idx.cpu().numpy()[0]
    d = O.from_inputs({k_: v.cpu() for k_, v in inp.items()})
    tau = float(O.default_tau(wl.d_k))
    dk_ref = np.zeros((wl.S, wl.D_I))
    for t in range(wl.T):
        pos = O.query_pos(wl.T, wl.S, t)
        sel = None if idx_np is None else idx_np[t]
        p = O.kl_target_row(d["q"][t], d["kv"], pos, tau, sel)
        keys = np.arange(pos + 1) if sel is None else sel[sel >= 0]
        assert np.max(np.abs(tg[t, keys] - p[keys])) < 1e-5, f"target t={t}"
        # the oracle's loss and dL/dI over the GPU's own scores (FP32, checked
        # element-wise against the oracle elsewhere) and the oracle's target
        I = scores[t, : pos + 1].double().cpu().numpy()
        l_ref, g_ref = O.indexer_kl_row(I, p, sel)
        assert abs(lg[t] - l_ref) <= 1e-4 * max(abs(l_ref), 1e-3), f"loss t={t}: {lg[t]} vs {l_ref}"
        assert np.max(np.abs(gg[t, : pos + 1] - g_ref)) < 1e-5, f"dL/dI t={t}"
        dq_r, dw_r, dk_r = O.indexer_grads_row(d["qd"][t], d["w"][t], d["kd"], pos, g_ref)
        _close(dqg[t], dq_r, 1e-3, f"dq t={t}")
        _close(dwg[t], dw_r, 1e-3, f"dw t={t}")
        dk_ref[: pos + 1] += dk_r
    _close(dkg, dk_ref, 1e-3, "dk")


# ----------------------------------------------------------------- backward alone, several shapes

BWD_CASES = [
    # name, B, T, S, H_I, k (None: every visible key), page size, ragged lengths
    ("dense_b2_ragged_8tiles", 2, 24, 900, 64, None, 0, True),
    ("sparse_k300_h32_paged64", 2, 16, 1100, 32, 300, 64, False),
    ("dense_h16_one_query_block", 1, 8, 700, 16, None, 0, False),
    ("sparse_k2048_h64_16tiles", 1, 4, 2600, 64, 2048, 0, False),
]


@pytest.mark.parametrize("name,B,T,S,H_I,k,page,ragged", BWD_CASES, ids=[c[0] for c in BWD_CASES])
def test_indexer_backward_shapes(name, B, T, S, H_I, k, page, ragged):
    """dsa_indexer_backward fed a random dL/dI, against the oracle's chain
    rule.  Integer FP8 bytes with power-of-two scales keep every dot product
    exact on both sides, so the ReLU mask is the same decision; the
    tolerance, 2e-5 of the largest entry, is FP32 accumulation over a few
    thousand terms (a gradient carried in plain BF16 would miss it by far)."""
    wl = Workload(name, B=B, T=T, S=S, H_I=H_I, D_I=128, H=8, d_k=80, d_v=64, k=k or 64, q_block=T, seed=90,
                  int_mode=True)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    gen = torch.Generator(device="cuda").manual_seed(91)
    inp["q_scale"] = torch.exp2(torch.randint(-3, 4, inp["q_scale"].shape, device="cuda", generator=gen).float())
    inp["k_scale"] = torch.exp2(torch.randint(-3, 4, inp["k_scale"].shape, device="cuda", generator=gen).float())
    lengths = [S - 37 * b if ragged else S for b in range(B)]
    sl = torch.tensor(lengths, dtype=torch.int32, device="cuda") if ragged else None
    ld = (S + 63) // 64 * 64
    rows = B * T
    grad = torch.randn(rows, ld, device="cuda", generator=gen)
    idx = None
    rng = np.random.default_rng(92)
    if k is not None:
        sel = np.full((B, T, k), -1, np.int32)
        for b in range(B):
            for t in range(T):
                n = lengths[b] - T + t + 1
                keys = rng.choice(n, size=min(k, n), replace=False)
                slots = rng.permutation(k)[: keys.size]         # valid keys anywhere in the row
                sel[b, t, slots] = keys
        idx = torch.from_numpy(sel).cuda()
    key_inp = inp
    if page:
        key_inp, table, num_pages = to_paged(inp, wl, page, 93)
        shape = dsa.make_shape(wl, seqlens=sl, block_table=table, page_size=page, num_pages=num_pages)
        dk = torch.zeros(num_pages * page, wl.D_I, device="cuda")
    else:
        shape = dsa.make_shape(wl, seqlens=sl)
        dk = torch.zeros(B, S, wl.D_I, device="cuda")
    dq = torch.zeros(B, T, H_I, wl.D_I, device="cuda")
    dw = torch.zeros(B, T, H_I, device="cuda")
    dsa.indexer_backward(shape, inp["q_I"], inp["q_scale"], inp["w"], key_inp["k_I"], key_inp["k_scale"], grad, 0, T,
                         dq, dw, dk, idx)
    st, det = dsa.device_error()
    assert st == 0, (st, hex(det))
    g_np = grad.cpu().double().numpy()
    dq_np, dw_np, dk_np = dq.cpu().numpy(), dw.cpu().numpy(), dk.cpu().numpy()
    for b in range(B):
        d = O.from_inputs({k_: v.cpu() for k_, v in inp.items()}, b)
        dk_ref = np.zeros((S, wl.D_I))
        for t in range(T):
            pos = lengths[b] - T + t
            g = g_np[b * T + t, : pos + 1].copy()
            if idx is not None:
                keep = np.zeros(pos + 1, bool)
                s_ = sel[b, t]
                keep[s_[s_ >= 0]] = True
                g[~keep] = 0.0
            dq_r, dw_r, dk_r = O.indexer_grads_row(d["qd"][t], d["w"][t], d["kd"], pos, g)
            _close(dq_np[b, t], dq_r, 2e-5, f"dq b={b} t={t}")
            _close(dw_np[b, t], dw_r, 2e-5, f"dw b={b} t={t}")
            dk_ref[: pos + 1] += dk_r
        if page:
            tb = table.cpu().numpy()
            s_all = np.arange(S)
            got = dk_np[tb[b, s_all // page] * page + s_all % page]
        else:
            got = dk_np[b]
        _close(got, dk_ref, 2e-5, f"dk b={b}")


@pytest.mark.parametrize("sparse", [False, True], ids=["dense", "sparse"])
def test_kl_target_paged_ragged(sparse):
    """dsa_kl_target over page pools (page 64, random order) with ragged
    lengths, against the oracle's target rows; the dense stage reads every
    visible key, the sparse one a random set with empty slots anywhere.  The
    lse fed in is the oracle's own (natural log over the same keys), so only
    the target's arithmetic is under test: 1e-5 absolute (entries are
    probabilities)."""
    wl = Workload("kl_paged", B=2, T=6, S=900, H_I=8, D_I=64, H=128, d_k=576, d_v=512, k=200, q_block=6, seed=95)
    inp = make_inputs(wl, "cuda")
    inp.pop("needle_pos", None)
    lengths = [wl.S, wl.S - 123]
    sl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    pin, table, num_pages = to_paged(inp, wl, 64, 96)
    shape = dsa.make_shape(wl, seqlens=sl, block_table=table, page_size=64, num_pages=num_pages)
    rng = np.random.default_rng(97)
    tau = float(O.default_tau(wl.d_k))
    sel = None
    if sparse:
        sel = np.full((wl.B, wl.T, wl.k), -1, np.int32)
        for b in range(wl.B):
            for t in range(wl.T):
                n = lengths[b] - wl.T + t + 1
                keys = rng.choice(n, size=min(wl.k, n) - 7, replace=False)
                sel[b, t, rng.permutation(wl.k)[: keys.size]] = keys
    lse = np.zeros((wl.B, wl.T, wl.H), np.float32)
    refs = {}
    for b in range(wl.B):
        d = O.from_inputs({k_: v.cpu() for k_, v in inp.items()}, b)
        for t in range(wl.T):
            pos = lengths[b] - wl.T + t
            keys = np.arange(pos + 1) if sel is None else np.unique(sel[b, t][sel[b, t] >= 0])
            z = tau * (d["q"][t] @ d["kv"][keys].T)
            m = z.max(axis=1)
            lse[b, t] = m + np.log(np.exp(z - m[:, None]).sum(axis=1))
            refs[(b, t)] = O.kl_target_row(d["q"][t], d["kv"], pos, tau, None if sel is None else sel[b, t])
    ld = (wl.S + 63) // 64 * 64
    target = torch.zeros(wl.B * wl.T, ld, device="cuda")
    idx = None if sel is None else torch.from_numpy(sel).cuda()
    dsa.kl_target(shape, pin["q"], pin["kv"], torch.from_numpy(lse).cuda(), 0, wl.T, target, idx)
    st, det = dsa.device_error()
    assert st == 0, (st, hex(det))
    tg = target.cpu().numpy()
    for (b, t), p in refs.items():
        pos = lengths[b] - wl.T + t
        keys = np.arange(pos + 1) if sel is None else np.unique(sel[b, t][sel[b, t] >= 0])
        assert np.max(np.abs(tg[b * wl.T + t, keys] - p[keys])) < 1e-5, (b, t)
