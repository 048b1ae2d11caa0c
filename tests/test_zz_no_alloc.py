"""dsa_topk_static: the allocation-free top-k entry point.

It must select exactly what dsa_topk selects (integer index sets, so the
tolerance is equality of the sorted sets), on two calls in a row: the second
call reuses the library's fixed histogram array after the first, so any count
left behind by the first call would change its answer.  Rows of each call are
also checked against the FP64 oracle's selection (the scores are FP32 values
that both sides compare as they are), including the few-levels rows whose
tie group at the k-th key is larger than the shared-memory candidate buffer.
The file is named to run last, after the other GPU tests have used the
library on the same device.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_05_b200 import dsa
from oracle import dsa_oracle as O

DSA_ERR_WORKSPACE = 3
MAX_ROWS = 64  # DSA_TOPK_STATIC_MAX_ROWS in include/dsa.h


def _shape(B, T, S, k):
    return dsa.make_shape(None, mode=dsa.DSA_DECODE if T == 1 else dsa.DSA_PREFILL, B=B, T=T, S=S, H_I=4,
                          D_I=32, H=8, d_k=80, d_v=64, k=k, q_block=T)


def test_static_topk_rejects_rows_beyond_limit():
    """Host-side check: more than the fixed array's rows is refused before any launch."""
    from long_context_05_b200 import build
    build.build()
    shape = _shape(B=MAX_ROWS + 1, T=1, S=4096, k=2048)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    code = dsa.lib().dsa_topk_static(ctypes.byref(shape), fake, 4096, 0, 1, fake, None)
    assert code == DSA_ERR_WORKSPACE


def _scores(g, rows, S, ld, kind):
    sc = torch.full((rows, ld), float("nan"), device="cuda")
    if kind == "normal":
        sc[:, :S] = torch.randn(rows, S, generator=g, device="cuda")
    else:  # few levels: large tie groups around the k-th key
        sc[:, :S] = torch.randint(-3, 4, (rows, S), generator=g, device="cuda").float()
    return sc


def _sets(idx):
    a = idx.cpu().numpy().reshape(-1, idx.shape[-1])
    return [sorted(r.tolist()) for r in a]


@pytest.mark.gpu
@pytest.mark.parametrize("B,T,S,q_begin,q_count,k", [
    (8, 1, 131072, 0, 1, 2048),      # decode rows, eight sequences of 128K keys
    (2, 40, 20000, 8, 32, 2048),     # a ragged prefill block: 64 rows, causal lengths 19969..20000
    (1, 3, 1500, 0, 3, 2048),        # every row shorter than k: indices 0..pos, then -1
])
def test_static_topk_matches_topk_twice(B, T, S, q_begin, q_count, k):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    shape = _shape(B, T, S, k)
    ld = (S + 63) // 64 * 64
    rows = B * q_count
    g = torch.Generator(device="cuda")
    g.manual_seed(S + rows)
    ws = dsa.alloc_workspace(shape)
    for call, kind in enumerate(("normal", "levels")):
        sc = _scores(g, rows, S, ld, kind)
        ref = torch.full((B, T, k), -7, dtype=torch.int32, device="cuda")
        got = torch.full((B, T, k), -9, dtype=torch.int32, device="cuda")
        dsa.topk(shape, sc, q_begin, q_count, ref, ws)
        dsa.topk_static(shape, sc, q_begin, q_count, got)
        st, det = dsa.device_error()
        assert st == 0, (call, st, det)
        r, o = ref[:, q_begin:q_begin + q_count], got[:, q_begin:q_begin + q_count]
        assert _sets(o) == _sets(r), f"call {call}"
        # rows outside [q_begin, q_begin + q_count) are left alone
        assert bool((got[:, :q_begin] == -9).all()) and bool((got[:, q_begin + q_count:] == -9).all())
        n = S - T + q_begin + np.arange(q_count) + 1
        filled = (o.cpu().numpy() >= 0).sum(-1)
        assert (filled == np.minimum(n, k)[None, :]).all(), f"call {call}"
        # against the oracle: the first, a middle and the last row of the call
        og = o.cpu().numpy()
        scn = sc.cpu().numpy()
        for r in sorted({0, rows // 2, rows - 1}):
            b, i = divmod(r, q_count)
            ref = O.topk_row(scn[r, : n[i]].astype(np.float64), k)
            assert sorted(og[b, i][og[b, i] >= 0].tolist()) == sorted(ref[ref >= 0].tolist()), (call, r)
