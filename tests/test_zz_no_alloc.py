"""The allocation-free selection entry point, called through the C ABI.

iskv_select_prompt_blocks_noalloc serves callers that cannot allocate device memory: a plugin
inside a host framework that owns all device memory and hands over only inputs and outputs, or a
latency-critical path where cudaMalloc could synchronise the device. Its scratch is a fixed array
inside the library, shared by every call on the device. This test makes two calls in a row (the
second runs on scratch that still holds the first call's contents) and checks each result against
the workspace form, bit for bit, plus the refusal of a size that does not fit the scratch.

This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from gpu_util import kv
import synth

pytestmark = pytest.mark.gpu


def _noalloc(m, keys, block=8, per_head=128, suffix=4, radius=32):
    lib = m._lib.load()
    L, H, hd = keys.shape
    dev = keys.device
    pk = torch.full((L,), -7, dtype=torch.int32, device=dev)
    pv = torch.full((L,), -7, dtype=torch.int32, device=dev)
    hb = torch.full((H, per_head), -7, dtype=torch.int32, device=dev)
    cnt = torch.full((2 + H,), -7, dtype=torch.int64, device=dev)
    st = lib.iskv_select_prompt_blocks_noalloc(
        keys.data_ptr(), m._dt(keys), L, H, hd, block, per_head, suffix, radius, pk.data_ptr(),
        pv.data_ptr(), hb.data_ptr(), cnt.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return st, {"P_K": pk, "P_V": pv, "head_blocks": hb, "counts": cnt}


def _same(a, b, H):
    ca, cb = a["counts"].cpu().numpy(), b["counts"].cpu().numpy()
    assert np.array_equal(ca, cb)
    assert np.array_equal(a["P_K"][:ca[0]].cpu().numpy(), b["P_K"][:cb[0]].cpu().numpy())
    assert np.array_equal(a["P_V"][:ca[1]].cpu().numpy(), b["P_V"][:cb[1]].cpu().numpy())
    for h in range(H):
        n = int(ca[2 + h])
        assert np.array_equal(a["head_blocks"][h][:n].cpu().numpy(),
                              b["head_blocks"][h][:n].cpu().numpy())


def test_noalloc_selection_matches_workspace_form_on_two_calls():
    m = kv()
    cases = [synth.outlier_prompt_keys(65536, 8, 128, seed=21)[0],
             synth.outlier_prompt_keys(4096 + 5, 8, 128, seed=22)[0]]
    keys = [torch.as_tensor(k, dtype=torch.float32).cuda().to(torch.bfloat16) for k in cases]
    outs = []
    for k in keys:                          # two calls in a row on the shared scratch
        st, out = _noalloc(m, k)
        assert st == 0
        outs.append(out)
    torch.cuda.synchronize()
    for k, out in zip(keys, outs):
        ref = m.select_prompt_blocks(k, 8, 128, 4, 32)
        torch.cuda.synchronize()
        _same(out, ref, 8)


def test_noalloc_small_call_then_larger_calls():
    """A small prompt first, then a 16 times longer one with the same per-head budget, then a
    prompt whose tail is not a whole block: each later call runs on scratch that the earlier,
    smaller calls left partly written, and each must still equal the workspace form bit for bit."""
    m = kv()
    cases = [synth.outlier_prompt_keys(4101, 8, 128, seed=23)[0],
             synth.outlier_prompt_keys(65536, 8, 128, seed=24)[0],
             synth.outlier_prompt_keys(30000 + 3, 8, 128, seed=25)[0]]
    for k in cases:
        kt = torch.as_tensor(k, dtype=torch.float32).cuda().to(torch.bfloat16)
        st, out = _noalloc(m, kt)
        assert st == 0
        ref = m.select_prompt_blocks(kt, 8, 128, 4, 32)
        torch.cuda.synchronize()
        _same(out, ref, 8)


def test_noalloc_refuses_sizes_beyond_its_scratch():
    m = kv()
    lib = m._lib.load()
    limit = lib.iskv_select_workspace_size(1 << 20, 8, 8)
    assert limit > (4 << 20)
    dummy = ctypes.c_void_p(0x1000)
    st = lib.iskv_select_prompt_blocks_noalloc(dummy, 1, 1 << 20, 8, 128, 8, 128, 4, 32, dummy,
                                               dummy, dummy, dummy, None)
    assert st == 8   # ISKV_ERR_WORKSPACE, nothing launched
    assert b"scratch" in lib.iskv_last_error()
    st = lib.iskv_select_prompt_blocks_noalloc(dummy, 7, 4096, 8, 128, 8, 128, 4, 32, dummy,
                                               dummy, dummy, dummy, None)
    assert st == 1   # ISKV_ERR_ARG: bad key dtype
    assert b"float32 or bf16" in lib.iskv_last_error()
