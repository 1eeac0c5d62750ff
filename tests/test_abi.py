"""The C-ABI library without a GPU: it loads, exports every entry point the header declares, and
its host-side argument checks reject bad calls before anything is launched."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jssa.h")


@pytest.fixture(scope="module")
def lib():
    from token_level_sparse_fp8_b200 import build, _lib
    build.build()
    return _lib.load()


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"JSSA_API\s+[\w\s\*]+?\b(jssa_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ["jssa_calibrate_accumulate", "jssa_compute_basis", "jssa_store", "jssa_score_topk",
              "jssa_indexed_attend", "jssa_decode", "jssa_dense_decode"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    from token_level_sparse_fp8_b200 import _lib
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (jssa_\w+)", out))
    assert set(_declared()) <= exported
    assert set(_declared()) == set(_lib.SIGNATURES)
    for n in _declared():
        assert hasattr(lib, n)


def test_built_for_sm100a():
    # the build compiles for sm_100a only (no PTX for other targets, no other architectures)
    from token_level_sparse_fp8_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings_and_version(lib):
    from token_level_sparse_fp8_b200 import _lib
    assert lib.jssa_version() >= 100
    assert _lib.status_string(0) == "ok"
    for code in range(-7, 0):
        assert _lib.status_string(code) != "unknown status"


def test_workspace_sizes_are_host_only(lib):
    from token_level_sparse_fp8_b200 import api, _lib
    assert api.workspace_size(_lib.FN_COMPUTE_BASIS, 0, 1, 8, 128, 0, 1, 0) == 8 * 128 * 128 * 8
    n = api.workspace_size(_lib.FN_DECODE, 16, 32, 8, 128, 8192, 16, 2048)
    n_score = api.workspace_size(_lib.FN_SCORE_TOPK, 16, 32, 8, 128, 8192, 16, 2048)
    n_attend = api.workspace_size(_lib.FN_INDEXED_ATTEND, 16, 32, 8, 128, 8192, 16, 2048)
    assert n >= n_score + n_attend > 0
    assert n_score >= 16 * 8 * 131072 * 8  # candidate keys + positions for every position
    full = api.workspace_size(_lib.FN_DENSE_DECODE, 16, 32, 8, 128, 8192, 16, 0)
    windowed = api.workspace_size(_lib.FN_DENSE_DECODE, 16, 32, 8, 128, 8192, 16, 1024)
    assert full > windowed
    with pytest.raises(_lib.JSSAError):
        api.workspace_size(_lib.FN_DECODE, 1, 30, 8, 128, 64, 16, 64)  # h_q not a multiple of h_kv


def test_mla_workspace_and_budget_limit(lib):
    from token_level_sparse_fp8_b200 import api, _lib
    # one sequence, 128 heads: a single split needs no partials; many splits need
    # (tickets +) 128 rows x 132 floats per (head block, value quarter, split)
    assert api.workspace_size(_lib.FN_MLA_ATTEND, 64, 128, 1, 576, 2048, 64, 1024) == 0
    n = api.workspace_size(_lib.FN_MLA_ATTEND, 1, 128, 1, 576, 2048, 64, 2048)
    assert n >= 4 * 2 * 128 * 132 * 4
    big = api.workspace_size(_lib.FN_MLA_ATTEND, 1, 128, 1, 576, 8192, 64, 256 * 1024)
    assert big > n
    with pytest.raises(_lib.JSSAError):
        api.workspace_size(_lib.FN_MLA_ATTEND, 1, 128, 1, 576, 8192, 64, 256 * 1024 + 1)
    with pytest.raises(_lib.JSSAError):
        api.workspace_size(_lib.FN_MLA_ATTEND, 1, 100, 1, 576, 2048, 64, 2048)  # h_q % 16
    # the entry refuses the same budget before touching any pointer
    st = lib.jssa_mla_attend(None, None, 64 * 576, 576, None, 16, None, None, 1, 128,
                             256 * 1024 + 1, 10, 64, ctypes.c_float(0.1), None, None, 0, None)
    assert st == -3
    # an output 8- but not 16-byte aligned (the kernel writes 16-byte pieces of each row)
    st = lib.jssa_mla_attend(0x10000, 0x20000, 64 * 576, 576, 0x30000, 16, 0x40000, 0x50000, 1,
                             128, 2048, 10, 64, ctypes.c_float(0.1), 0x60008, 0x70000, 1 << 30,
                             None)
    assert st == -4


def test_argument_checks_reject_before_launch(lib):
    from token_level_sparse_fp8_b200 import _lib
    # NULL inputs, unsupported shapes and bad alignment are refused on the host
    st = lib.jssa_score_topk(None, None, None, None, 16, None, 1, 8, 2, 128, 32, 10, 16, 128,
                             None, None, None, 0, None)
    assert st == -1
    st = lib.jssa_score_topk(None, None, None, None, 16, None, 1, 8, 2, 96, 32, 10, 16, 128,
                             None, None, None, 0, None)
    assert st == -3  # no d = 96 instance
    st = lib.jssa_score_topk(None, None, None, None, 16, None, 1, 8, 3, 128, 32, 10, 16, 128,
                             None, None, None, 0, None)
    assert st == -2  # 8 query heads over 3 KV heads
    st = lib.jssa_store(8, 1024, 32, 1, 2, 128, 32, 48, 32, 10, 16, None)
    assert st == -4  # misaligned key pointer
    # queries 4- but not 16-byte aligned (the prep reads query rows with 16-byte loads)
    st = lib.jssa_score_topk(0x1004, 0x2000, 0x3000, 0x4000, 16, 0x5000, 1, 8, 2, 128, 32, 10, 16,
                             128, 0x6000, 0x7000, 0x8000, 1 << 30, None)
    assert st == -4
    st = lib.jssa_indexed_attend(16, 16, 16, 4096, 256, 128, 16, 8, 16, 16, 1, 64, 2, 128, 128,
                                 10, 16, ctypes.c_float(0.1), 16, None, 0, None)
    assert st == -3  # G = 32 query heads per KV head is beyond the m16 tile
    st = lib.jssa_decode(None, None, None, None, None, 0, 0, 0, None, None, None, 1, None, 0, 8, 2,
                         128, 32, 1, 16, 128, ctypes.c_float(0.1), None, None, None, None, 0, None)
    assert st == 0  # batch 0 is a no-op
    st = lib.jssa_compute_basis(16, 16, 2, 128, 32, 16, None, 16, 100, None)
    assert st == -5  # workspace too small
    # host-buffer decode: NULL host buffers, a lone new K row, and a workspace without room for
    # the two staging sets are refused before any copy or stream is created
    args = (0x1000, 0x2000, 16 * 2 * 128, 2 * 128, 128, 0x4000, 0x5000, 0x6000, 16, 0x7000, 2, 8,
            2, 128, 32, 10, 16, 128, ctypes.c_float(0.1), 0x8000, 0x9000)
    st = lib.jssa_decode_host(None, None, None, *args, 0xA000, 0xB000, 1 << 30, None)
    assert st == -1
    st = lib.jssa_decode_host(0xC000, 0xD000, None, *args, 0xA000, 0xB000, 1 << 30, None)
    assert st == -1
    need = _lib_ws(lib, 8, 2, 8, 2, 128, 16, 16, 128)
    st = lib.jssa_decode_host(0xC000, None, None, *args, 0xA000, 0xB000, need - 1, None)
    assert st == -5
    assert need >= _lib_ws(lib, 4, 2, 8, 2, 128, 16, 16, 128) + 2 * 2 * (2 * 8 * 128 * 2)
    assert lib.jssa_decode_host_join(None, None) == -1


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    # sizes whose split-K scratch exceeds the library's fixed array are refused before any launch
    # (the pointers are never dereferenced: host-side check only)
    from token_level_sparse_fp8_b200 import api, _lib
    limit = 4 << 20
    batch, h_q, h_kv, d, budget = 64, 32, 8, 128, 4096
    need = api.workspace_size(_lib.FN_INDEXED_ATTEND, batch, h_q, h_kv, d, 1024, 16, budget)
    assert need > limit
    st = lib.jssa_indexed_attend_noalloc(0x10000, 0x20000, 0x30000, 16 * h_kv * d, h_kv * d, d,
                                         0x40000, 1024, 0x50000, 0x60000, batch, h_q, h_kv, d,
                                         budget, 100000, 16, ctypes.c_float(0.1), 0x70000, None)
    assert st == -7
    assert _lib.status_string(st) != "unknown status"
    # a size that fits is not refused by that check (it fails later only for want of a GPU)
    small = api.workspace_size(_lib.FN_INDEXED_ATTEND, 1, 8, 2, 128, 16, 16, 256)
    assert small <= limit


def _lib_ws(lib, fn, batch, h_q, h_kv, d, max_pages, page_size, budget):
    n = ctypes.c_size_t(0)
    assert lib.jssa_workspace_size(fn, batch, h_q, h_kv, d, max_pages, page_size, budget,
                                   ctypes.byref(n)) == 0
    return n.value
