"""The calibration-stability study (README: "Calibration stability (CV=3.9%)")
run through sq_calibrate / sq_compress_kv / sq_decompress_kv on the GPU,
against the same study done by the oracle on the same calibration draws and
evaluation vectors."""

import math

import numpy as np
import pytest
import torch

from oracle import calibration as ocal
from oracle import codec as ocodec
from synthetic.workloads import CONFIGS, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from compressed_attention_head_b200.stability import calibration_stability  # noqa: E402


def _oracle_study(name, n_draws, n_eval, heads):
    cfg = dict(CONFIGS[name])
    g = cfg["n_q"] // cfg["n_kv"]
    cfg.update(n_kv=heads, n_q=heads * g)
    ev = make_workload(cfg, 0, device="cuda", batch=1, tokens=n_eval, with_calibration=False)
    out = {"keys": [], "values": []}
    for draw in range(n_draws):
        cal = make_workload(cfg, 0, device="cuda", batch=1, tokens=1, calib_draw=draw + 1)
        for side, xc, xe, b, is_key in (("keys", cal.k_cal, ev.k, cfg["bits_k"], True),
                                         ("values", cal.v_cal, ev.v, cfg["bits_v"], False)):
            cos = []
            for h in range(heads):
                c = ocal.calibrate(xc[h].double().cpu().numpy(), avg_bits=b, is_key=is_key, stream=h)
                x = xe[0, h].double().cpu().numpy()
                o = ocodec.compress(x, c)
                xh = ocodec.decompress(o["words"], o["norm"], o["rnorm"], c, apply_qjl=is_key)
                cos.append(np.sum(x * xh, 1) / (np.linalg.norm(x, axis=1) * np.linalg.norm(xh, axis=1)))
            out[side].append(float(np.mean(np.concatenate(cos))))
    res = {}
    for side, vals in out.items():
        mean = float(np.mean(vals))
        res[side] = {"per_draw": vals, "mean": mean, "cv": float(np.std(vals)) / mean}
    return res


@pytest.mark.parametrize("name", ["llama8b", "qwen1_5b_long"])
def test_calibration_stability_matches_the_oracle(name):
    gpu = calibration_stability(name, n_draws=5, n_eval=2048, heads=2)
    ref = _oracle_study(name, 5, 2048, 2)
    for side in ("keys", "values"):
        g, r = gpu[side], ref[side]
        assert np.max(np.abs(np.array(g["per_draw"]) - np.array(r["per_draw"]))) < 1e-3, (side, g, r)
        assert abs(g["cv"] - r["cv"]) <= 0.3 * max(g["cv"], r["cv"]) + 2e-4, (side, g["cv"], r["cv"])
        # compression quality is high and stable across draws on these spectra
        assert g["mean"] > 0.9 and g["cv"] < 0.05
