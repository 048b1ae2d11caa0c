"""The C-ABI library builds, loads and exports every symbol include/dsa.h
declares; host-side argument checks answer without a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

from long_context_05_b200 import dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    return sorted(set(re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def libpath():
    from long_context_05_b200 import build
    return build.build()


def test_header_declarations_match_binding():
    assert _declared() == sorted(dsa.EXPORTS)


def test_library_exports_every_declared_symbol(libpath):
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(dsa_\w+)", out))
    missing = set(_declared()) - exported
    assert not missing, missing
    L = ctypes.CDLL(libpath)
    for name in _declared():
        assert hasattr(L, name)


def test_host_side_calls_without_gpu(libpath):
    L = dsa.lib()
    assert L.dsa_version() >= 100
    assert L.dsa_status_string(3) == b"workspace missing or too small"
    # invalid shapes are rejected before touching the device
    bad = dsa.make_shape(None, B=1, T=4, S=2, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=4, q_block=4)
    assert dsa.workspace_size(bad) == 0                     # T > S
    uns = dsa.make_shape(None, B=1, T=4, S=8, H_I=4, D_I=48, H=8, d_k=80, d_v=64, k=4, q_block=4)
    assert dsa.workspace_size(uns) == 0                     # D_I unsupported
    assert L.dsa_forward(None, None, None, None, None, None, 0, None) == 1
    assert L.dsa_indexer_scores(ctypes.byref(bad), None, None, None, None, None, 0, 1, None, 8, None) == 1
    assert L.dsa_sparse_attn(ctypes.byref(uns), None, None, None, None, None, None, None, 0, None) == 2
    assert L.dsa_dense_attn(ctypes.byref(uns), None, None, None, None, None, None, 0, None) == 2
    assert L.dsa_version() >= 200
    # paged caches: the page size must be a multiple of 16 and the block table
    # must cover S keys per sequence
    paged = dict(B=2, T=1, S=1000, H_I=4, D_I=32, H=8, d_k=80, d_v=64, k=64, q_block=1, mode=dsa.DSA_DECODE)
    fake_table = 1 << 20                                    # never dereferenced on the host
    ok = dsa.make_shape(None, **paged, page_size=64, pages_per_seq=16, num_pages=40, block_table=fake_table)
    assert dsa.workspace_size(ok) > 0
    assert dsa.workspace_size(dsa.make_shape(None, **paged, page_size=40, pages_per_seq=25, num_pages=60,
                                             block_table=fake_table)) == 0      # not a multiple of 16
    assert dsa.workspace_size(dsa.make_shape(None, **paged, page_size=64, pages_per_seq=15, num_pages=40,
                                             block_table=fake_table)) == 0      # 15 * 64 < S
    assert dsa.workspace_size(dsa.make_shape(None, **paged, page_size=64, pages_per_seq=16, num_pages=40)) == 0
    # the fused selection's workspace: about a third of the 4096 x 131072 FP32
    # score tile (2 GiB) for a 128K prefill block; the score tile's size where
    # the fused selection does not apply (decode, short contexts)
    from long_context_05_b200.inputs import WORKLOADS
    big = dsa.make_shape(WORKLOADS["prefill_128k"])
    tile = 4096 * 131072 * 4
    assert dsa.workspace_size(big) >= tile
    assert 0 < dsa.select_workspace_size(big) < tile // 3
    for name in ("decode_128k_b8", "prefill_8k"):
        sh = dsa.make_shape(WORKLOADS[name])
        assert dsa.select_workspace_size(sh) == dsa.workspace_size(sh) > 0
    assert dsa.select_workspace_size(bad) == 0
    assert L.dsa_launch_count() == 0


def test_build_entry_compiles(libpath):
    import __graft_entry__ as ge
    ge.build()
    assert os.path.exists(dsa.LIB_PATH)
