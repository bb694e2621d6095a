"""CPU checks of the C ABI: the library loads, exports every entry point include/iskv.h declares,
and rejects bad arguments on the host before any CUDA call (no GPU needed)."""

import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "iskv.h")


def _lib():
    from kv_cache_online_b200 import build
    build.build()
    from kv_cache_online_b200 import _lib as L
    return L, L.load()


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"\b(iskv_[a-z_]+)\s*\(", src)))


def test_header_declarations_are_all_bound_and_exported():
    L, lib = _lib()
    declared = _declared()
    assert len(declared) >= 15
    assert set(declared) == set(L.SIGNATURES), "binding must mirror the header exactly"
    nm = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True,
                        text=True, check=True).stdout
    exported = set(re.findall(r"\b(iskv_[a-z_]+)\b", nm))
    missing = [n for n in declared if n not in exported]
    assert not missing, f"not exported: {missing}"
    for n in declared:
        getattr(lib, n)


def test_status_strings_and_version():
    L, lib = _lib()
    assert lib.iskv_abi_version() == 1
    for code in range(9):
        assert lib.iskv_status_string(code)
    assert lib.iskv_status_string(99) == b"unknown status"


def test_workspace_queries_are_consistent():
    L, lib = _lib()
    one = lib.iskv_fold_workspace_size(1, 1024, 256, 64)
    two = lib.iskv_fold_workspace_size(2, 1024, 256, 64)
    assert one > 1024 * 256 * 4 and two > one
    assert lib.iskv_fold_workspace_size(0, 1024, 256, 64) == 0
    assert lib.iskv_reorth_workspace_size(1, 1024, 256, 16384) > 16 * 256 * 256 * 4
    assert lib.iskv_reconstruct_workspace_size(1, 1024, 256) >= 1024 * 256 * 2
    assert lib.iskv_select_workspace_size(65536, 8, 8) > 65536 * 8


def _fake_handle(L, d=1024, r=256, storage=1, base=0x10000):
    return L.IskvLowRank(d, r, 4096, storage, 0, base, base + 0x1000, base + 0x2000,
                         base + 0x3000, base + 0x4000)


def test_host_side_argument_errors():
    L, lib = _lib()
    h = _fake_handle(L)
    F = ctypes.c_void_p(0x20000)
    P = ctypes.c_void_p(0x30000)
    ws = ctypes.c_void_p(0x40000)
    big = 1 << 40
    # null handle
    assert lib.iskv_fold_block(None, F, 1, 64, P, 0.0, ws, big, None) == 1
    # bad block size (not a multiple of 8 / too large)
    assert lib.iskv_fold_block(ctypes.byref(h), F, 1, 12, P, 0.0, ws, big, None) == 2
    assert lib.iskv_fold_block(ctypes.byref(h), F, 1, 256, P, 0.0, ws, big, None) == 2
    assert b"b" in lib.iskv_last_error()
    # bad dtype
    assert lib.iskv_fold_block(ctypes.byref(h), F, 7, 64, P, 0.0, ws, big, None) == 1
    # workspace too small / misaligned
    assert lib.iskv_fold_block(ctypes.byref(h), F, 1, 64, P, 0.0, ws, 10, None) == 8
    assert lib.iskv_fold_block(ctypes.byref(h), F, 1, 64, P, 0.0, ctypes.c_void_p(0x40001),
                               big, None) == 8
    # misaligned history pointer
    hb = _fake_handle(L, base=0x10008)
    assert lib.iskv_fold_block(ctypes.byref(hb), F, 1, 64, P, 0.0, ws, big, None) == 1
    # r_max > d, r_max not a multiple of 16
    assert lib.iskv_fold_block(ctypes.byref(_fake_handle(L, d=128, r=256)), F, 1, 64, P, 0.0, ws,
                               big, None) == 2
    assert lib.iskv_fold_block(ctypes.byref(_fake_handle(L, r=250)), F, 1, 64, P, 0.0, ws, big,
                               None) == 2
    # reconstruction: d != heads * head_dim, odd head_dim
    out = ctypes.c_void_p(0x50000)
    assert lib.iskv_reconstruct(ctypes.byref(h), None, 1, None, 0, 100, 8, 64, 1, 5e5, out, 1,
                                ws, big, None) == 2
    assert lib.iskv_reconstruct(ctypes.byref(h), None, 1, None, 0, 100, 8, 127, 1, 5e5, out, 1,
                                ws, big, None) == 2
    # selection: L out of range, head_dim odd, null output
    k = ctypes.c_void_p(0x60000)
    o = ctypes.c_void_p(0x70000)
    assert lib.iskv_select_prompt_blocks(k, 1, 0, 8, 128, 8, 128, 4, 32, o, o, o, o, ws, big,
                                         None) == 2
    assert lib.iskv_select_prompt_blocks(k, 1, 100, 8, 127, 8, 128, 4, 32, o, o, o, o, ws, big,
                                         None) == 2
    assert lib.iskv_select_prompt_blocks(k, 1, 100, 8, 128, 8, 128, 4, 32, None, o, o, o, ws, big,
                                         None) == 1
    # reorth: batched histories must agree
    arr = (L.IskvLowRank * 2)(_fake_handle(L), _fake_handle(L, r=128))
    assert lib.iskv_reorth(arr, 2, ws, big, None) == 2


def test_python_binding_fails_loudly_without_library(tmp_path):
    from kv_cache_online_b200 import _lib as L
    with pytest.raises(RuntimeError, match="not found"):
        L.load(str(tmp_path / "missing.so"))
