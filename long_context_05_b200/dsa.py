"""Thin ctypes binding of libdsa.so (include/dsa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors must be CUDA tensors on the current device, contiguous, of
the dtype stated; the work is enqueued on torch's current stream.  There is
no CPU fallback: if the library is missing, importing the functions raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

DSA_PREFILL = 0
DSA_DECODE = 1

STATUS = {
    0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_WORKSPACE",
    4: "DSA_ERR_CUDA", 5: "DSA_ERR_TIMEOUT", 6: "DSA_ERR_DEVICE_BOUNDS",
}

EXPORTS = [
    "dsa_version", "dsa_status_string", "dsa_workspace_size", "dsa_indexer_scores", "dsa_topk",
    "dsa_sparse_attn", "dsa_forward", "dsa_prefill", "dsa_decode", "dsa_get_device_error",
    "dsa_set_wait_timeout_us", "dsa_launch_count", "dsa_selftest_wait_timeout", "dsa_topk_static",
]


class DsaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [
        ("mode", ctypes.c_int), ("B", ctypes.c_int), ("T", ctypes.c_int), ("S", ctypes.c_int),
        ("H_I", ctypes.c_int), ("D_I", ctypes.c_int), ("H", ctypes.c_int), ("d_k", ctypes.c_int),
        ("d_v", ctypes.c_int), ("k", ctypes.c_int), ("q_block", ctypes.c_int),
        ("softmax_scale", ctypes.c_float),
    ]


class Inputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("q_I", "q_scale", "w", "k_I", "k_scale", "q", "kv")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libdsa.so (built in-tree by long_context_05_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m long_context_05_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        sp = ctypes.POINTER(Shape)
        L.dsa_version.restype = i
        L.dsa_status_string.restype = ctypes.c_char_p
        L.dsa_status_string.argtypes = [i]
        L.dsa_workspace_size.restype = sz
        L.dsa_workspace_size.argtypes = [sp]
        L.dsa_indexer_scores.restype = i
        L.dsa_indexer_scores.argtypes = [sp, vp, vp, vp, vp, vp, i, i, vp, i64, vp]
        L.dsa_topk.restype = i
        L.dsa_topk.argtypes = [sp, vp, i64, i, i, vp, vp, sz, vp]
        L.dsa_topk_static.restype = i
        L.dsa_topk_static.argtypes = [sp, vp, i64, i, i, vp, vp]
        L.dsa_sparse_attn.restype = i
        L.dsa_sparse_attn.argtypes = [sp, vp, vp, vp, vp, vp, vp, sz, vp]
        for fn in ("dsa_forward", "dsa_prefill", "dsa_decode"):
            getattr(L, fn).restype = i
            getattr(L, fn).argtypes = [sp, ctypes.POINTER(Inputs), vp, vp, vp, vp, sz, vp]
        L.dsa_get_device_error.restype = i
        L.dsa_get_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
        L.dsa_launch_count.restype = ctypes.c_ulonglong
        L.dsa_launch_count.argtypes = []
        L.dsa_selftest_wait_timeout.restype = i
        L.dsa_selftest_wait_timeout.argtypes = [vp]
        L.dsa_set_wait_timeout_us.restype = None
        L.dsa_set_wait_timeout_us.argtypes = [ctypes.c_longlong]
        _lib = L
    return _lib


def make_shape(wl=None, mode=None, **kw) -> Shape:
    """Shape from a Workload (long_context_05_b200.inputs) and/or keywords."""
    f = {n: 0 for n, _ in Shape._fields_}
    f["softmax_scale"] = 0.0
    if wl is not None:
        for n in ("B", "T", "S", "H_I", "D_I", "H", "d_k", "d_v", "k", "q_block"):
            f[n] = getattr(wl, n)
        f["mode"] = DSA_DECODE if wl.decode else DSA_PREFILL
    if mode is not None:
        f["mode"] = mode
    f.update(kw)
    return Shape(**f)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, dtype, name):
    if not (t.is_cuda and t.is_contiguous() and t.dtype == dtype):
        raise ValueError(f"{name}: need a contiguous CUDA tensor of {dtype}, got {t.dtype} "
                         f"{'cuda' if t.is_cuda else 'cpu'} contiguous={t.is_contiguous()}")


def _check(fn, code):
    if code != 0:
        raise DsaError(fn, code)


def workspace_size(shape: Shape) -> int:
    return int(lib().dsa_workspace_size(ctypes.byref(shape)))


def alloc_workspace(shape: Shape) -> torch.Tensor:
    n = workspace_size(shape)
    if n == 0:
        raise DsaError("dsa_workspace_size", 1)
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def indexer_scores(shape: Shape, q_I, q_scale, w, k_I, k_scale, q_begin: int, q_count: int,
                   scores: torch.Tensor) -> torch.Tensor:
    """Step A into scores [B * q_count, ld] (float32, ld = scores.shape[1])."""
    for t, d, n in ((q_I, torch.uint8, "q_I"), (q_scale, torch.float32, "q_scale"), (w, torch.float32, "w"),
                    (k_I, torch.uint8, "k_I"), (k_scale, torch.float32, "k_scale"),
                    (scores, torch.float32, "scores")):
        _need(t, d, n)
    _check("dsa_indexer_scores", lib().dsa_indexer_scores(
        ctypes.byref(shape), _p(q_I), _p(q_scale), _p(w), _p(k_I), _p(k_scale), q_begin, q_count,
        _p(scores), scores.shape[-1], _stream()))
    return scores


def topk(shape: Shape, scores: torch.Tensor, q_begin: int, q_count: int, idx: torch.Tensor,
         ws: torch.Tensor | None = None) -> torch.Tensor:
    """Step B: rows of `scores` -> idx [B, T, k] int32 rows q_begin.. q_begin+q_count."""
    _need(scores, torch.float32, "scores")
    _need(idx, torch.int32, "idx")
    _check("dsa_topk", lib().dsa_topk(
        ctypes.byref(shape), _p(scores), scores.shape[-1], q_begin, q_count, _p(idx),
        _p(ws), 0 if ws is None else ws.numel(), _stream()))
    return idx


def topk_static(shape: Shape, scores: torch.Tensor, q_begin: int, q_count: int,
                idx: torch.Tensor) -> torch.Tensor:
    """Step B with the library's fixed histogram array (no workspace, no allocation)."""
    _need(scores, torch.float32, "scores")
    _need(idx, torch.int32, "idx")
    _check("dsa_topk_static", lib().dsa_topk_static(
        ctypes.byref(shape), _p(scores), scores.shape[-1], q_begin, q_count, _p(idx), _stream()))
    return idx


def sparse_attn(shape: Shape, q, kv, idx, out, lse=None, ws=None):
    """Step C: out [B, T, H, d_v] bf16 (+ lse [B, T, H] fp32)."""
    _need(q, torch.bfloat16, "q")
    _need(kv, torch.bfloat16, "kv")
    _need(idx, torch.int32, "idx")
    _need(out, torch.bfloat16, "out")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    _check("dsa_sparse_attn", lib().dsa_sparse_attn(
        ctypes.byref(shape), _p(q), _p(kv), _p(idx), _p(out), _p(lse), _p(ws),
        0 if ws is None else ws.numel(), _stream()))
    return out, lse


def _inputs(inp: dict) -> Inputs:
    for n, d in (("q_I", torch.uint8), ("q_scale", torch.float32), ("w", torch.float32),
                 ("k_I", torch.uint8), ("k_scale", torch.float32), ("q", torch.bfloat16),
                 ("kv", torch.bfloat16)):
        _need(inp[n], d, n)
    return Inputs(*(inp[n].data_ptr() for n in ("q_I", "q_scale", "w", "k_I", "k_scale", "q", "kv")))


def forward(shape: Shape, inp: dict, out, lse, idx, ws, entry: str = "dsa_forward"):
    """The whole path through dsa_forward (or dsa_prefill / dsa_decode)."""
    ins = _inputs(inp)
    _need(out, torch.bfloat16, "out")
    _need(idx, torch.int32, "idx")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    _check(entry, getattr(lib(), entry)(
        ctypes.byref(shape), ctypes.byref(ins), _p(out), _p(lse), _p(idx), _p(ws), ws.numel(), _stream()))
    return out, lse, idx


def device_error() -> tuple[int, int]:
    """Synchronise the current stream; return (status, detail) of the device error word."""
    d = ctypes.c_int(0)
    st = lib().dsa_get_device_error(_stream(), ctypes.byref(d))
    return int(st), int(d.value)


def launch_count() -> int:
    return int(lib().dsa_launch_count())


def selftest_wait_timeout() -> None:
    _check("dsa_selftest_wait_timeout", lib().dsa_selftest_wait_timeout(_stream()))


def set_wait_timeout_us(us: int) -> None:
    lib().dsa_set_wait_timeout_us(int(us))


@dataclass
class Outputs:
    out: torch.Tensor
    lse: torch.Tensor
    idx: torch.Tensor


def alloc_outputs(wl) -> Outputs:
    dev = "cuda"
    return Outputs(torch.empty(wl.B, wl.T, wl.H, wl.d_v, dtype=torch.bfloat16, device=dev),
                   torch.empty(wl.B, wl.T, wl.H, dtype=torch.float32, device=dev),
                   torch.empty(wl.B, wl.T, wl.k, dtype=torch.int32, device=dev))
