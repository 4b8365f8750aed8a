"""Calibration stability across independent calibration draws (the pages report
calibration as a one-time step whose result carries over to new data).

For the Llama-, Qwen-14B- and Qwen-1.5B-shaped heads, four independent
2048-token draws of the same head model give the same d_eff and QJL count, top
eigenvalues within a few percent of each other, bit allocations that differ in
at most a handful of coordinates, and the same signal subspace (keys: the top
d_eff eigenvectors; values: the planted block of equal spikes). These hold
because N = 2048 is large against d = 128 and the planted spectra have wide
gaps; the bounds leave about a factor of two over the measured spread.
"""

import numpy as np
import pytest

from oracle import calibration as ocal
from synthetic import CONFIGS, make_workload

DRAWS = 4


def _draws(name, side):
    cfg = CONFIGS[name]
    bits = cfg["bits_k"] if side == "k" else cfg["bits_v"]
    out = []
    for ds in range(DRAWS):
        w = make_workload(name, 0, batch=1, tokens=2048, data_stream=ds, with_calibration=False)
        x = (w.k if side == "k" else w.v)[0, 0].double().numpy()
        out.append(ocal.calibrate(x, avg_bits=bits, is_key=side == "k", stream=0))
    return cfg, out


def _projector_spread(cals, k):
    proj = [c.V[:, :k] @ c.V[:, :k].T for c in cals]
    return max(np.linalg.norm(p - proj[0], 2) for p in proj[1:])


@pytest.mark.parametrize("name", ["llama8b", "qwen14b", "qwen1_5b_long"])
@pytest.mark.parametrize("side", ["k", "v"])
def test_calibration_is_stable_across_draws(name, side):
    cfg, cals = _draws(name, side)
    assert len({c.d_eff for c in cals}) == 1
    assert len({c.m for c in cals}) == 1
    lam = np.array([c.lam[:4] for c in cals])
    assert np.all(lam.std(axis=0) / lam.mean(axis=0) < 0.1)
    bits = np.array([c.bits for c in cals])
    assert max(int(np.sum(b != bits[0])) for b in bits) <= 8
    assert all(int(b.sum()) == int(bits[0].sum()) for b in bits)
    k = cals[0].d_eff if side == "k" else cfg["v_spikes"]
    assert _projector_spread(cals, k) < 0.2
