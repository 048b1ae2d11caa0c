"""GPU parity of step B (dsa_topk) on adversarial score rows.

Rows are fed straight to the C ABI, so the selection is checked apart from
the indexer: heavy ties (all equal, huge tie groups at the k-th key that do
not fit the shared-memory candidate buffer), signed zeros, sorted rows and
random rows.  Index sets must equal the oracle's exactly (the scores are
FP32 values, so both sides compare the same numbers).
"""
import numpy as np
import pytest
import torch

from long_context_05_b200 import dsa
from oracle import dsa_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.lib()


def _rows(n, rng):
    r = []
    r.append(rng.standard_normal(n).astype(np.float32))                       # random
    r.append(np.zeros(n, np.float32))                                         # all equal
    z = np.where(rng.random(n) < 0.5, np.float32(-0.0), np.float32(0.0))
    z[rng.choice(n, min(100, n // 8), replace=False)] = 1.0
    r.append(z.astype(np.float32))                                            # signed zeros
    big = np.full(n, 0.5, np.float32)                                         # huge tie at the k-th key
    big[rng.choice(n, min(1000, n // 8), replace=False)] = 2.0
    big[rng.choice(n, min(3000, n // 4), replace=False)] = -1.0
    r.append(big)
    r.append(rng.integers(-3, 4, n).astype(np.float32))                       # few levels
    r.append(np.linspace(1, -1, n).astype(np.float32))                        # decreasing
    r.append(np.linspace(-1, 1, n).astype(np.float32))                        # increasing
    d = np.round(rng.standard_normal(n), 1).astype(np.float32)                # many duplicates
    r.append(d)
    return np.stack(r)


@pytest.mark.parametrize("S,k,use_ws", [(20000, 2048, True), (20000, 2048, False), (3000, 2048, False),
                                        (131072, 2048, True), (700, 64, False)])
def test_topk_adversarial_rows(S, k, use_ws):
    rng = np.random.default_rng(S + k)
    rows = _rows(S, rng)
    B = rows.shape[0]
    shape = dsa.make_shape(None, mode=dsa.DSA_DECODE, B=B, T=1, S=S, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=k,
                           q_block=1)
    ld = (S + 63) // 64 * 64
    sc = torch.full((B, ld), float("nan"), device="cuda")
    sc[:, :S] = torch.from_numpy(rows).cuda()
    idx = torch.full((B, 1, k), -7, dtype=torch.int32, device="cuda")
    ws = dsa.alloc_workspace(shape) if use_ws else None
    dsa.topk(shape, sc, 0, 1, idx, ws)
    st, det = dsa.device_error()
    assert st == 0, (st, det)
    got = idx.cpu().numpy()[:, 0]
    for b in range(B):
        ref = O.topk_row(rows[b].astype(np.float64), k)
        g = got[b]
        assert (g == -1).sum() == (ref == -1).sum(), b
        assert sorted(g[g >= 0].tolist()) == sorted(ref[ref >= 0].tolist()), f"row pattern {b}"
