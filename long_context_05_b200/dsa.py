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
    "dsa_version", "dsa_status_string", "dsa_workspace_size", "dsa_select_workspace_size", "dsa_indexer_scores",
    "dsa_topk",
    "dsa_sparse_attn", "dsa_forward", "dsa_prefill", "dsa_decode", "dsa_get_device_error",
    "dsa_set_wait_timeout_us", "dsa_launch_count", "dsa_selftest_wait_timeout", "dsa_topk_static",
    "dsa_dense_attn", "dsa_topk_candidates", "dsa_topk_merge", "dsa_attn_combine", "dsa_select",
    "dsa_kl_target", "dsa_indexer_kl", "dsa_indexer_backward",
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
        ("softmax_scale", ctypes.c_float), ("seqlens", ctypes.c_void_p), ("page_size", ctypes.c_int),
        ("pages_per_seq", ctypes.c_int), ("num_pages", ctypes.c_int), ("block_table", ctypes.c_void_p),
    ]


INPUT_NAMES = ("q_I", "q_scale", "w", "k_I", "k_scale", "q", "kv", "v")


class Inputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in INPUT_NAMES]


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
        L.dsa_select_workspace_size.restype = sz
        L.dsa_select_workspace_size.argtypes = [sp]
        L.dsa_indexer_scores.restype = i
        L.dsa_indexer_scores.argtypes = [sp, vp, vp, vp, vp, vp, i, i, vp, i64, vp]
        L.dsa_topk.restype = i
        L.dsa_topk.argtypes = [sp, vp, i64, i, i, vp, vp, sz, vp]
        L.dsa_topk_static.restype = i
        L.dsa_topk_static.argtypes = [sp, vp, i64, i, i, vp, vp]
        L.dsa_sparse_attn.restype = i
        L.dsa_sparse_attn.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.dsa_dense_attn.restype = i
        L.dsa_dense_attn.argtypes = [sp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.dsa_kl_target.restype = i
        L.dsa_kl_target.argtypes = [sp, vp, vp, vp, vp, i, i, vp, i64, vp]
        L.dsa_indexer_kl.restype = i
        L.dsa_indexer_kl.argtypes = [sp, vp, vp, i64, vp, i, i, vp, vp, vp]
        L.dsa_indexer_backward.restype = i
        L.dsa_indexer_backward.argtypes = [sp, vp, vp, vp, vp, vp, vp, i64, vp, i, i, vp, vp, vp, vp]
        L.dsa_select.restype = i
        L.dsa_select.argtypes = [sp, vp, vp, vp, vp, vp, i, i, vp, vp, sz, vp]
        L.dsa_topk_candidates.restype = i
        L.dsa_topk_candidates.argtypes = [sp, vp, i64, vp, ctypes.c_int32, vp, vp, vp]
        L.dsa_topk_merge.restype = i
        L.dsa_topk_merge.argtypes = [sp, i, vp, vp, vp, ctypes.c_int32, ctypes.c_int32, vp, vp]
        L.dsa_attn_combine.restype = i
        L.dsa_attn_combine.argtypes = [sp, i, vp, vp, vp, vp, vp]
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


def make_shape(wl=None, mode=None, seqlens=None, block_table=None, page_size=0, num_pages=0, **kw) -> Shape:
    """Shape from a Workload (long_context_05_b200.inputs) and/or keywords.

    seqlens: int32 CUDA tensor [B] of per-sequence key counts (or None).
    block_table: int32 CUDA tensor [B, pages_per_seq] for paged caches, with
    page_size and num_pages.  The shape keeps references to both tensors, so
    their device pointers stay valid while the shape is alive."""
    f = {n: 0 for n, _ in Shape._fields_}
    f["softmax_scale"] = 0.0
    f["seqlens"] = None
    f["block_table"] = None
    if wl is not None:
        for n in ("B", "T", "S", "H_I", "D_I", "H", "d_k", "d_v", "k", "q_block"):
            f[n] = getattr(wl, n)
        f["mode"] = DSA_DECODE if wl.decode else DSA_PREFILL
    if mode is not None:
        f["mode"] = mode
    keep = []
    if seqlens is not None:
        _need(seqlens, torch.int32, "seqlens")
        f["seqlens"] = seqlens.data_ptr()
        keep.append(seqlens)
    f["page_size"] = page_size
    f["num_pages"] = num_pages
    if isinstance(block_table, int):        # a raw device address (pages_per_seq in kw)
        f["block_table"] = block_table
    elif block_table is not None:
        _need(block_table, torch.int32, "block_table")
        f["block_table"] = block_table.data_ptr()
        f["pages_per_seq"] = block_table.shape[-1]
        keep.append(block_table)
    f.update(kw)
    sh = Shape(**f)
    sh._keep = keep
    return sh


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


def select_workspace_size(shape: Shape) -> int:
    return int(lib().dsa_select_workspace_size(ctypes.byref(shape)))


def alloc_workspace(shape: Shape, fused: bool = False) -> torch.Tensor:
    """dsa_workspace_size bytes, or with fused=True dsa_select_workspace_size
    (dsa_select's size; a prefill forward given it takes the fused selection)."""
    n = select_workspace_size(shape) if fused else workspace_size(shape)
    if n == 0:
        raise DsaError("dsa_select_workspace_size" if fused else "dsa_workspace_size", 1)
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


def select(shape: Shape, q_I, q_scale, w, k_I, k_scale, q_begin: int, q_count: int, idx: torch.Tensor,
           ws: torch.Tensor) -> torch.Tensor:
    """Steps A and B for queries [q_begin, q_begin + q_count) -> idx [B, T, k]."""
    for t, d, n in ((q_I, torch.uint8, "q_I"), (q_scale, torch.float32, "q_scale"), (w, torch.float32, "w"),
                    (k_I, torch.uint8, "k_I"), (k_scale, torch.float32, "k_scale"), (idx, torch.int32, "idx")):
        _need(t, d, n)
    _check("dsa_select", lib().dsa_select(
        ctypes.byref(shape), _p(q_I), _p(q_scale), _p(w), _p(k_I), _p(k_scale), q_begin, q_count, _p(idx),
        _p(ws), ws.numel(), _stream()))
    return idx


def topk_static(shape: Shape, scores: torch.Tensor, q_begin: int, q_count: int,
                idx: torch.Tensor) -> torch.Tensor:
    """Step B with the library's fixed histogram array (no workspace, no allocation)."""
    _need(scores, torch.float32, "scores")
    _need(idx, torch.int32, "idx")
    _check("dsa_topk_static", lib().dsa_topk_static(
        ctypes.byref(shape), _p(scores), scores.shape[-1], q_begin, q_count, _p(idx), _stream()))
    return idx


def sparse_attn(shape: Shape, q, kv, idx, out, lse=None, ws=None, v=None):
    """Step C: out [B, T, H, d_v] bf16 (+ lse [B, T, H] fp32).  v: separate
    values [.., d_v] bf16, or None for V = kv[..., :d_v]."""
    _need(q, torch.bfloat16, "q")
    _need(kv, torch.bfloat16, "kv")
    _need(idx, torch.int32, "idx")
    _need(out, torch.bfloat16, "out")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    if v is not None:
        _need(v, torch.bfloat16, "v")
    _check("dsa_sparse_attn", lib().dsa_sparse_attn(
        ctypes.byref(shape), _p(q), _p(kv), _p(v), _p(idx), _p(out), _p(lse), _p(ws),
        0 if ws is None else ws.numel(), _stream()))
    return out, lse


def dense_attn(shape: Shape, q, kv, out, lse=None, ws=None, v=None):
    """Dense causal attention over every visible key (no selection)."""
    _need(q, torch.bfloat16, "q")
    _need(kv, torch.bfloat16, "kv")
    _need(out, torch.bfloat16, "out")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    if v is not None:
        _need(v, torch.bfloat16, "v")
    _check("dsa_dense_attn", lib().dsa_dense_attn(
        ctypes.byref(shape), _p(q), _p(kv), _p(v), _p(out), _p(lse), _p(ws),
        0 if ws is None else ws.numel(), _stream()))
    return out, lse


def topk_candidates(shape: Shape, scores, idx, part_begin: int, cand_scores, cand_idx):
    """(score, global index) pairs of a part's selection (key-split rows)."""
    _need(scores, torch.float32, "scores")
    _need(idx, torch.int32, "idx")
    _need(cand_scores, torch.float32, "cand_scores")
    _need(cand_idx, torch.int32, "cand_idx")
    _check("dsa_topk_candidates", lib().dsa_topk_candidates(
        ctypes.byref(shape), _p(scores), scores.shape[-1], _p(idx), part_begin, _p(cand_scores), _p(cand_idx),
        _stream()))
    return cand_scores, cand_idx


def topk_merge(shape: Shape, cand_scores, cand_idx, idx, local_begin: int = 0, local_count: int = 0,
               idx_local=None):
    """Global top-k of [nparts, B*T, k] candidate lists (+ this part's local indices)."""
    _need(cand_scores, torch.float32, "cand_scores")
    _need(cand_idx, torch.int32, "cand_idx")
    _need(idx, torch.int32, "idx")
    if idx_local is not None:
        _need(idx_local, torch.int32, "idx_local")
    _check("dsa_topk_merge", lib().dsa_topk_merge(
        ctypes.byref(shape), cand_scores.shape[0], _p(cand_scores), _p(cand_idx), _p(idx), local_begin,
        local_count, _p(idx_local), _stream()))
    return idx, idx_local


def attn_combine(shape: Shape, o_parts, lse_parts, out, lse=None):
    """Merge [nparts, ...] attention results over disjoint key subsets."""
    _need(o_parts, torch.bfloat16, "o_parts")
    _need(lse_parts, torch.float32, "lse_parts")
    _need(out, torch.bfloat16, "out")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    _check("dsa_attn_combine", lib().dsa_attn_combine(
        ctypes.byref(shape), o_parts.shape[0], _p(o_parts), _p(lse_parts), _p(out), _p(lse), _stream()))
    return out, lse


def kl_target(shape: Shape, q, kv, lse, q_begin: int, q_count: int, target, idx=None):
    """Indexer-training target rows [B * q_count, ld] from the main attention's lse."""
    _need(q, torch.bfloat16, "q")
    _need(kv, torch.bfloat16, "kv")
    _need(lse, torch.float32, "lse")
    _need(target, torch.float32, "target")
    if idx is not None:
        _need(idx, torch.int32, "idx")
    _check("dsa_kl_target", lib().dsa_kl_target(
        ctypes.byref(shape), _p(q), _p(kv), _p(lse), _p(idx), q_begin, q_count, _p(target), target.shape[-1],
        _stream()))
    return target


def indexer_kl(shape: Shape, scores, target, q_begin: int, q_count: int, grad, loss, idx=None):
    """KL loss per row and its gradient with respect to the indexer scores."""
    for t, n in ((scores, "scores"), (target, "target"), (grad, "grad"), (loss, "loss")):
        _need(t, torch.float32, n)
    if idx is not None:
        _need(idx, torch.int32, "idx")
    _check("dsa_indexer_kl", lib().dsa_indexer_kl(
        ctypes.byref(shape), _p(scores), _p(target), scores.shape[-1], _p(idx), q_begin, q_count, _p(grad),
        _p(loss), _stream()))
    return grad, loss


def indexer_backward(shape: Shape, q_I, q_scale, w, k_I, k_scale, grad, q_begin: int, q_count: int, dq, dw, dk,
                     idx=None):
    """Gradients of the indexer's inputs (dequantised, FP32); dk accumulates."""
    for t, d, n in ((q_I, torch.uint8, "q_I"), (q_scale, torch.float32, "q_scale"), (w, torch.float32, "w"),
                    (k_I, torch.uint8, "k_I"), (k_scale, torch.float32, "k_scale"), (grad, torch.float32, "grad"),
                    (dq, torch.float32, "dq"), (dw, torch.float32, "dw"), (dk, torch.float32, "dk")):
        _need(t, d, n)
    if idx is not None:
        _need(idx, torch.int32, "idx")
    _check("dsa_indexer_backward", lib().dsa_indexer_backward(
        ctypes.byref(shape), _p(q_I), _p(q_scale), _p(w), _p(k_I), _p(k_scale), _p(grad), grad.shape[-1], _p(idx),
        q_begin, q_count, _p(dq), _p(dw), _p(dk), _stream()))
    return dq, dw, dk


def _inputs(inp: dict) -> Inputs:
    """Inputs struct from a dict of tensors; "v" is optional (None = MLA form)."""
    for n, d in (("q_I", torch.uint8), ("q_scale", torch.float32), ("w", torch.float32),
                 ("k_I", torch.uint8), ("k_scale", torch.float32), ("q", torch.bfloat16),
                 ("kv", torch.bfloat16)):
        _need(inp[n], d, n)
    v = inp.get("v")
    if v is not None:
        _need(v, torch.bfloat16, "v")
    return Inputs(*(inp[n].data_ptr() for n in INPUT_NAMES[:-1]), None if v is None else v.data_ptr())


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
