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
    # the cache step reuses one workspace for its append, folds, eviction and reorth in turn
    step = lib.iskv_cache_step_workspace_size(64, 1024, 256, 64, 17000, 0)
    assert step == max(lib.iskv_fold_workspace_size(64, 1024, 256, 64),
                       lib.iskv_reorth_workspace_size(64, 1024, 256, 17000))
    refit = lib.iskv_cache_step_workspace_size(64, 1024, 128, 64, 17000, 128)
    assert refit >= lib.iskv_fold_workspace_size(64, 1024, 128, 128) > \
        lib.iskv_fold_workspace_size(64, 1024, 128, 64)
    # a refit larger than one fold takes runs as b-row folds: no extra workspace
    assert lib.iskv_cache_step_workspace_size(64, 1024, 256, 64, 17000, 192) == step
    assert lib.iskv_cache_step_workspace_size(0, 1024, 256, 64, 17000, 0) == 0


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
    # allocation-free selection: each refusal leaves its own reason, a later one replaces it
    assert lib.iskv_select_prompt_blocks_noalloc(k, 1, 1 << 20, 8, 128, 8, 128, 4, 32, o, o, o, o,
                                                 None) == 8
    assert b"scratch" in lib.iskv_last_error()
    assert lib.iskv_select_prompt_blocks_noalloc(k, 1, 100, 8, 127, 8, 128, 4, 32, o, o, o, o,
                                                 None) == 2
    assert b"head_dim" in lib.iskv_last_error()
    assert lib.iskv_select_prompt_blocks_noalloc(k, 1, 100, 8, 128, 8, 128, 4, 32, None, o, o, o,
                                                 None) == 1
    assert b"null" in lib.iskv_last_error()
    # reorth: batched histories must agree
    arr = (L.IskvLowRank * 2)(_fake_handle(L), _fake_handle(L, r=128))
    assert lib.iskv_reorth(arr, 2, ws, big, None) == 2


def test_python_binding_fails_loudly_without_library(tmp_path):
    from kv_cache_online_b200 import _lib as L
    with pytest.raises(RuntimeError, match="not found"):
        L.load(str(tmp_path / "missing.so"))


def _fake_table(L, live, d=1024, window=128, block=64, cap_e=1024, dtype=1, base=0x80000):
    return L.IskvExactTable(d, window, block, 256, dtype, 0, cap_e, base, base + 0x100000,
                            ctypes.cast(live, ctypes.POINTER(ctypes.c_int32)), window + block,
                            0, 0, -1, 0, 0, 1)


def test_cache_policy_host_side_errors():
    """The cache-policy entry points refuse bad tables on the host and leave the mirror unchanged."""
    L, lib = _lib()
    live = (ctypes.c_int32 * 512)()
    ws = ctypes.c_void_p(0x40000)
    big = 1 << 40
    X = ctypes.c_void_p(0x20000)
    P = ctypes.c_void_p(0x30000)
    n = ctypes.c_int64()
    t = _fake_table(L, live)
    # initial window longer than the window; protected + window rows beyond the capacity
    assert lib.iskv_cache_prefill(ctypes.byref(t), X, 1, 1000, P, 10, 129, X, P, ctypes.byref(n),
                                  ws, big, None) == 1
    small = _fake_table(L, live, cap_e=100)
    assert lib.iskv_cache_prefill(ctypes.byref(small), X, 1, 1000, P, 10, 128, X, P,
                                  ctypes.byref(n), ws, big, None) == 4
    # live_cap below window + block
    bad = _fake_table(L, live)
    bad.live_cap = 100
    assert lib.iskv_cache_prefill(ctypes.byref(bad), X, 1, 1000, P, 10, 0, X, P, ctypes.byref(n),
                                  ws, big, None) == 2

    h = _fake_handle(L)
    tp = (ctypes.POINTER(L.IskvExactTable) * 1)(ctypes.pointer(t))
    hp = (ctypes.POINTER(L.IskvLowRank) * 1)(ctypes.pointer(h))
    rows = ctypes.c_void_p(0x90000)
    assert lib.iskv_cache_step(tp, hp, 0, rows, 1, 0.0, None, None, ws, big, None) == 2
    # a full table
    t.n_prot, t.n_live = 1000, 24
    assert lib.iskv_cache_step(tp, hp, 1, rows, 1, 0.0, None, None, ws, big, None) == 4
    # a fold is due (window 0: the new row makes 8 pending) but the history has no room
    t2 = _fake_table(L, live, window=0, block=8)
    for i in range(7):
        live[i] = i
    t2.n_live, t2.last, t2.hist_rows = 7, 6, 4090
    tp2 = (ctypes.POINTER(L.IskvExactTable) * 1)(ctypes.pointer(t2))
    assert lib.iskv_cache_step(tp2, hp, 1, rows, 1, 0.0, None, None, ws, big, None) == 4
    assert b"no room" in lib.iskv_last_error()
    assert (t2.n_live, t2.last, t2.hist_rows) == (7, 6, 4090)
    # a block the fold does not take; tables that disagree on d
    t3 = _fake_table(L, live, block=12)
    tp3 = (ctypes.POINTER(L.IskvExactTable) * 1)(ctypes.pointer(t3))
    assert lib.iskv_cache_step(tp3, hp, 1, rows, 1, 0.0, None, None, ws, big, None) == 2
    # a refit that is not a multiple of the block; a refit due on a non-empty history that neither
    # one fold nor a wide history of rank r_max + refit_rows - block <= 512 takes
    t5 = _fake_table(L, live, window=0, block=8)
    t5.refit_rows, t5.refit_done, t5.live_cap = 12, 0, 12
    tp5 = (ctypes.POINTER(L.IskvExactTable) * 1)(ctypes.pointer(t5))
    assert lib.iskv_cache_step(tp5, hp, 1, rows, 1, 0.0, None, None, ws, big, None) == 2
    t6 = _fake_table(L, live, window=0, block=8)
    t6.refit_rows, t6.refit_done, t6.live_cap = 280, 0, 280   # 256 + 280 - 8 > 512
    for i in range(279):
        live[i] = i
    t6.n_live, t6.last, t6.hist_rows = 279, 278, 100
    tp6 = (ctypes.POINTER(L.IskvExactTable) * 1)(ctypes.pointer(t6))
    assert lib.iskv_cache_step(tp6, hp, 1, rows, 1, 0.0, None, None, ws, big, None) == 2
    assert b"wide history" in lib.iskv_last_error()
    ta, tb = _fake_table(L, live), _fake_table(L, live, d=512)
    tp4 = (ctypes.POINTER(L.IskvExactTable) * 2)(ctypes.pointer(ta), ctypes.pointer(tb))
    hp4 = (ctypes.POINTER(L.IskvLowRank) * 2)(ctypes.pointer(h), ctypes.pointer(h))
    assert lib.iskv_cache_step(tp4, hp4, 2, rows, 1, 0.0, None, None, ws, big, None) == 2


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "iskv.h"

/* A plain C caller: the ABI version, a status string, a workspace query, and the cache step's
   schedule dry run on a host-only table (keys, empty prompt, W = 4, b = 8). */
int main(void) {
  int32_t live[12];
  iskv_exact_table t;
  iskv_exact_table *tabs[1];
  int32_t folded = 0, first = -1, pos;
  memset(&t, 0, sizeof t);
  t.d = 64; t.window = 4; t.block = 8; t.dtype = ISKV_BF16; t.cap_e = 64;
  t.rows = (void *)0x100000; t.pos = (int32_t *)0x200000;   /* never dereferenced by the dry run */
  t.live_host = live; t.live_cap = 12; t.last = -1; t.refit_done = 1;
  tabs[0] = &t;
  for (pos = 0; pos < 16; ++pos) {
    if (iskv_cache_plan(tabs, 1, 16, 64, 1, &folded, NULL) != ISKV_OK) return 2;
    if (folded && first < 0) first = pos;
  }
  printf("%d %s %d %lld %lld\n", (int)iskv_abi_version(), iskv_status_string(ISKV_ERR_CAPACITY),
         first, (long long)t.n_live, (long long)t.hist_rows);
  return iskv_fold_workspace_size(1, 1024, 256, 64) > 0 ? 0 : 3;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    """include/iskv.h compiles as strict C99 and a C program linked against libiskv.so runs the
    host-side entry points (no GPU needed)."""
    L, lib = _lib()
    src = tmp_path / "caller.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(L.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir,
                    "-liskv", f"-Wl,-rpath,{libdir}"], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    # first fold with position W + b - 1 = 11; after 16 positions: 8 folded, 8 live
    assert out == ["1", "history", "capacity", "exceeded", "11", "8", "8"]
