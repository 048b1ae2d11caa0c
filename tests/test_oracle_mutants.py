"""The pins catch plausible mistakes in the oracle.

Each case swaps one oracle function for a copy with a planted mistake (a
dropped term, a wrong sign or index, a transposed operand, a wrong tie rule)
and checks that at least one pin of tests/test_oracle.py fails on it.  The
mistakes are planted in the CPU oracle only.
"""
import numpy as np
import pytest

from oracle import dsa_oracle as O
import tests.test_oracle as P


def _indexer_no_relu(qd_t, w_t, kd, pos):
    return np.asarray(w_t) @ (np.asarray(qd_t) @ np.asarray(kd[: pos + 1]).T)


def _indexer_exclusive(qd_t, w_t, kd, pos):
    r = np.asarray(w_t) @ np.maximum(np.asarray(qd_t) @ np.asarray(kd[: pos + 1]).T, 0)
    r[-1] = -np.inf if pos > 0 else r[-1]
    return r


def _indexer_relu_after_sum(qd_t, w_t, kd, pos):
    return np.maximum(np.asarray(w_t) @ (np.asarray(qd_t) @ np.asarray(kd[: pos + 1]).T), 0)


def _e4m3_bias8(b):
    b = np.asarray(b, np.uint8)
    s = (b >> 7).astype(np.int64); e = ((b >> 3) & 15).astype(np.int64); m = (b & 7).astype(np.float64)
    v = np.where(e == 0, m / 8 * 2.0 ** -7, (1 + m / 8) * np.exp2((e - 8).astype(np.float64)))
    v = np.where(s == 1, -v, v)
    return np.where((e == 15) & (m == 7), np.nan, v)


def _topk_ties_high(sv, k):
    sv = np.asarray(sv, np.float64)
    n = sv.shape[0]
    order = np.lexsort((-np.arange(n), -sv))
    out = np.full(k, -1, np.int64)
    keep = order[: min(k, n)]
    out[: keep.shape[0]] = keep
    return out


def _topk_no_pad_limit(sv, k):
    sv = np.asarray(sv, np.float64)
    order = np.argsort(-sv, kind="stable")
    out = np.full(k, -1, np.int64)
    keep = order[: k - 1 if k > 1 else 1]   # off by one
    out[: keep.shape[0]] = keep
    return out


def _attn_wrong_value_cols(q_t, kv, idx_t, d_v, tau):
    sel = np.asarray(idx_t); sel = sel[sel >= 0]
    K = np.asarray(kv[sel], np.float64)
    z = tau * (q_t @ K.T); m = z.max(1, keepdims=True); p = np.exp(z - m); l = p.sum(1, keepdims=True)
    return (p @ K[:, -d_v:]) / l, (m + np.log(l))[:, 0]


def _attn_lse_no_max(q_t, kv, idx_t, d_v, tau):
    sel = np.asarray(idx_t); sel = sel[sel >= 0]
    K = np.asarray(kv[sel], np.float64)
    z = tau * (q_t @ K.T); m = z.max(1, keepdims=True); p = np.exp(z - m); l = p.sum(1, keepdims=True)
    return (p @ K[:, :d_v]) / l, np.log(l)[:, 0]



MUTANTS = [
    ("indexer_row", _indexer_no_relu),
    ("indexer_row", _indexer_exclusive),
    ("indexer_row", _indexer_relu_after_sum),
    ("e4m3_decode", _e4m3_bias8),
    ("topk_row", _topk_ties_high),
    ("topk_row", _topk_no_pad_limit),
    ("sparse_attention_row", _attn_wrong_value_cols),
    ("sparse_attention_row", _attn_lse_no_max),
]

PINS = [name for name in dir(P) if name.startswith("test_")]


def _run_pins():
    failed = []
    for name in PINS:
        fn = getattr(P, name)
        try:
            fn()
        except Exception:
            failed.append(name)
    return failed


@pytest.mark.parametrize("target,mutant", MUTANTS, ids=[m[1].__name__ for m in MUTANTS])
def test_pins_catch_mutant(monkeypatch, target, mutant):
    monkeypatch.setattr(O, target, mutant)
    failed = _run_pins()
    assert failed, f"no pin caught mutant {mutant.__name__} of {target}"
