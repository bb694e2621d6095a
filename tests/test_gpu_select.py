"""GPU prompt-block selection (Algorithm 1 steps 2-4) against the oracle: indices bit-exact."""

import numpy as np
import pytest
import torch

from gpu_util import kv
from oracle import select as osel
import synth

pytestmark = pytest.mark.gpu


def _run(m, keys_np, dtype, per_head=128, block=8, suffix=4, radius=32):
    kt = torch.as_tensor(keys_np, dtype=dtype, device="cuda").contiguous()
    seen = kt.to(torch.float64).cpu().numpy()
    ref = osel.select_prompt_blocks(seen, block, per_head, suffix, radius)
    out = m.select_prompt_blocks(kt, block, per_head, suffix, radius)
    torch.cuda.synchronize()
    return ref, {k: v.cpu().numpy() for k, v in out.items()}


def _check(ref, out, H, per_head):
    c = out["counts"]
    assert c[0] == len(ref["P_K"]) and np.array_equal(out["P_K"][:c[0]], ref["P_K"])
    assert c[1] == len(ref["P_V"]) and np.array_equal(out["P_V"][:c[1]], ref["P_V"])
    for h in range(H):
        nh = len(ref["head_blocks"][h])
        assert c[2 + h] == nh
        assert np.array_equal(out["head_blocks"][h][:nh], ref["head_blocks"][h])
        assert np.all(out["head_blocks"][h][nh:per_head] == -1)


def _margin_ok(ref, per_head):
    for sc in ref["scores"]:
        if sc.size > per_head:
            s = np.sort(sc)
            if s[per_head] - s[per_head - 1] < 1e-9:
                return False
    return True


@pytest.mark.parametrize("L,H,hd,dtype,seed", [
    (4096, 8, 128, torch.float32, 0),
    (4096 + 5, 8, 128, torch.bfloat16, 1),
    (16384, 8, 128, torch.bfloat16, 2),
    (2000, 2, 64, torch.float32, 3),
])
def test_selection_bit_exact(L, H, hd, dtype, seed):
    m = kv()
    keys, _ = synth.outlier_prompt_keys(L, H, hd, seed)
    ref, out = _run(m, keys, dtype)
    assert _margin_ok(ref, 128)
    _check(ref, out, H, 128)


def test_full_size_long_prompt():
    """Long-prompt path: L = 65536 post-RoPE keys, 8 heads x 128, 5% outlier blocks."""
    m = kv()
    keys, mask = synth.outlier_prompt_keys(65536, 8, 128, 4)
    ref, out = _run(m, keys, torch.bfloat16)
    assert _margin_ok(ref, 128)
    _check(ref, out, 8, 128)


def test_edge_cases():
    m = kv()
    k39, _ = synth.outlier_prompt_keys(39, 2, 16, 5)       # all suffix
    ref, out = _run(m, k39, torch.float32)
    _check(ref, out, 2, 128)
    assert out["counts"][0] == 39
    k403, _ = synth.outlier_prompt_keys(403, 2, 16, 6)     # fewer candidates than the budget
    ref, out = _run(m, k403, torch.float32)
    _check(ref, out, 2, 128)
    zeros = np.zeros((8 * 300, 2, 16))                      # all scores tie at 0: lowest indices
    ref, out = _run(m, zeros, torch.float32, per_head=10)
    _check(ref, out, 2, 10)
    assert list(out["head_blocks"][0][:10]) == list(range(10))
    ref, out = _run(m, k403, torch.float32, per_head=0, radius=0)
    _check(ref, out, 2, 0)


@pytest.mark.parametrize("L,dtype,seed", [(4096 + 5, torch.bfloat16, 7), (2000, torch.float32, 8)])
def test_block_scores_match_oracle(L, dtype, seed):
    """The float64 block scores themselves (left at the start of the workspace), not only the
    blocks they select, against the oracle's scores to 1e-12 relative."""
    m = kv()
    H, hd = 8, 128
    keys, _ = synth.outlier_prompt_keys(L, H, hd, seed)
    keys[:8, 3, :] = 0.0                                   # a zero block scores 0
    kt = torch.as_tensor(keys, dtype=dtype, device="cuda").contiguous()
    seen = kt.to(torch.float64).cpu().numpy()
    ref = osel.select_prompt_blocks(seen, 8, 128, 4, 32)
    ws = torch.zeros(m.select_workspace_size(L, H, 8), dtype=torch.uint8, device="cuda")
    m.select_prompt_blocks(kt, 8, 128, 4, 32, ws=ws)
    torch.cuda.synchronize()
    n_cand = ref["n_cand"]
    got = ws[:8 * H * n_cand].view(torch.float64).view(H, n_cand).cpu().numpy()
    assert ref["scores"][3, 0] == 0.0 and got[3, 0] == 0.0
    np.testing.assert_allclose(got, ref["scores"], rtol=1e-12, atol=1e-15)
