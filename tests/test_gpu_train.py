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
from long_context_05_b200.inputs import Workload, make_inputs
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
