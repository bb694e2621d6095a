"""GPU diagnostics (Section 5.1 eq. 12; the orthogonality Section 4.4 restores) against the
float64 oracle."""

import numpy as np
import pytest
import torch

from gpu_util import kv, set_state, stored
from oracle import accounting, reorth as oreo

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("storage", [torch.float32, torch.bfloat16])
def test_diagnostics_match_oracle(storage):
    m = kv()
    d, r, n_cap = 512, 128, 3000
    g = np.random.Generator(np.random.PCG64(9))
    hists, ref = [], []
    for n, k, drift in ((3000, 128, 3e-3), (1700, 96, 3e-2), (0, 0, 0.0)):
        h = m.LowRankHistory(d, r, n_cap, storage=storage)
        if k:
            U = stored(np.linalg.qr(g.standard_normal((n, k)))[0] +
                       drift * g.standard_normal((n, k)) / np.sqrt(n), storage)
            B = stored(np.linalg.qr(g.standard_normal((d, k)))[0] +
                       drift * g.standard_normal((d, k)) / np.sqrt(d), storage)
            set_state(h, U, np.geomspace(10, 1, k), B, np.arange(n))
            ref.append((oreo.orthogonality_error(U), oreo.orthogonality_error(B), n, k))
        else:
            ref.append((0.0, 0.0, 0, 0))
        hists.append(h)
    n_exact = [640, 128, 33]
    ou, ob, pb = m.diagnostics(hists, n_exact=n_exact, exact_bytes=2)
    ou, ob, pb = ou.cpu().numpy(), ob.cpu().numpy(), pb.cpu().numpy()
    sf = 4 if storage == torch.float32 else 2
    for i, (eu, eb, n, k) in enumerate(ref):
        assert abs(ou[i] - eu) <= 1e-3 * eu + 1e-5
        assert abs(ob[i] - eb) <= 1e-3 * eb + 1e-5
        assert pb[i] == accounting.persistent_bytes(n, k, d, n_exact[i], sf, 2)
