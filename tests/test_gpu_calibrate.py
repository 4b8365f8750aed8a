"""GPU calibration (second moment, Jacobi, finalize) against the oracle.

Individual eigenvectors of a (near-)degenerate noise subspace are not unique,
so the GPU calibration is checked by invariants rather than element by
element: orthonormality and eigen-residual of its own basis, eigenvalues
and d_eff against the oracle's, the signal subspace (projector) when the
spectral gap is large, the bit budget and the greedy optimality of the
allocation for its own eigenvalues, and the QJL matrix from the shared
counter-based generator.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import calibrate_oracle, read_records
from oracle import calibration as ocal
from oracle import codebook as ocb
from oracle import rng as orng
from synthetic import make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from compressed_attention_head_b200 import sq  # noqa: E402


def _gpu_calibrate(x_cal, avg_bits, is_key, qjl=True, seed=42, max_sweeps=30):
    nh, n, d = x_cal.shape
    p = sq.calib_params(d, nh, avg_bits, is_key, qjl=qjl, seed=seed, max_sweeps=max_sweeps)
    recs = sq.alloc_records(nh, d)
    ws = torch.empty(sq.sq_calibrate_workspace(p, n), dtype=torch.uint8, device="cuda")
    status = torch.full((nh,), -1, dtype=torch.int32, device="cuda")
    x = x_cal.contiguous().cuda()
    sq.sq_calibrate(p, x, n, n * d, d, recs, ws, status)
    torch.cuda.synchronize()
    return read_records(recs, nh, d), status.cpu().tolist()


@pytest.mark.parametrize("name", ["tiny", "llama8b", "gemma9b_sweep"])
def test_calibration_invariants(name):
    w = make_workload(name, batch=1, tokens=16)
    cfg = w.cfg
    nh = 2
    for kind, xcal, bits, is_key in (("k", w.k_cal[:nh], cfg["bits_k"], True), ("v", w.v_cal[:nh], cfg["bits_v"], False)):
        gpu, status = _gpu_calibrate(xcal, bits, is_key)
        assert status == [0] * nh
        ref = calibrate_oracle(xcal, bits, is_key)
        for hi, (g, r) in enumerate(zip(gpu, ref)):
            d = g.d
            lmax = r.lam[0]
            assert np.max(np.abs(g.V.T @ g.V - np.eye(d))) < 1e-9
            c = ocal.second_moment(xcal[hi].double().numpy())
            res = np.linalg.norm(c @ g.V - g.V * g.lam, axis=0)
            assert np.max(res) < 1e-9 * lmax
            assert np.max(np.abs(g.lam - r.lam)) < 1e-9 * lmax
            assert g.d_eff == r.d_eff and g.m == r.m
            assert abs(g.trace - r.trace) < 1e-10 * r.trace
            if np.isfinite(r.kappa) and r.kappa > 10:
                pg = g.V[:, :r.d_eff] @ g.V[:, :r.d_eff].T
                pr = r.V[:, :r.d_eff] @ r.V[:, :r.d_eff].T
                assert np.max(np.abs(pg - pr)) < 1e-6
            # sign convention
            for i in range(d):
                j = int(np.argmax(np.abs(g.V[:, i])))
                assert g.V[j, i] > 0
            # budget and greedy optimality for the GPU's own eigenvalues
            assert g.bits.sum() + g.m == g.total_bits
            assert np.all(np.diff(g.bits) <= 0) or np.any(np.diff(g.lam) == 0)
            dist = ocb.distortion_table()
            gain_next = np.where(g.bits < 8, g.lam * (dist[np.minimum(g.bits, 7)] - dist[np.minimum(g.bits + 1, 8)]), -np.inf)
            gain_last = np.where(g.bits > 0, g.lam * (dist[np.maximum(g.bits - 1, 0)] - dist[g.bits]), np.inf)
            assert np.max(gain_next) <= np.min(gain_last) * (1 + 1e-12) + 1e-300
            assert np.array_equal(g.offsets, ocal.bit_offsets(g.bits))
            # QJL matrix from the shared counter-based definition
            if g.m:
                s_ref = orng.qjl_matrix(42, g.stream, g.m)
                assert np.max(np.abs(g.S - s_ref)) < 1e-12 * max(1.0, np.max(np.abs(s_ref)))
            assert np.allclose(g.sigma, ocal.scales(g.lam, True), rtol=1e-12, atol=1e-300)


def test_exact_spectra_deff():
    """Calibration vectors with an exactly known second moment (identity, rank 4)."""
    d = 32
    eye = torch.eye(d).repeat(4, 1) * 2.0          # 128 rows: C = 16 I / 128, a flat spectrum
    gpu, st = _gpu_calibrate(eye[None].float(), 3.0, False)
    assert st == [0] and gpu[0].d_eff == d
    r4 = torch.zeros(8, d)
    for i in range(4):
        r4[2 * i, i] = 1.0
        r4[2 * i + 1, i] = -1.0
    gpu, st = _gpu_calibrate(r4[None], 3.0, True)
    assert gpu[0].d_eff == 4 and gpu[0].m == 4


def test_not_converged_status():
    w = make_workload("llama8b", batch=1, tokens=16)
    _, status = _gpu_calibrate(w.k_cal[:1], 3.0, True, max_sweeps=1)
    assert status == [sq.SQ_ERR_NOT_CONVERGED]


def test_import_rejects_malformed_record():
    w = make_workload("tiny", batch=1, tokens=16)
    ref = calibrate_oracle(w.k_cal[:2], 3.0, True)
    from oracle import record as orec
    size = sq.sq_calib_bytes(32)
    host = np.zeros(2 * size, dtype=np.uint8)
    for i, c in enumerate(ref):
        raw = np.frombuffer(orec.write(c), dtype=np.uint8)
        host[i * size:i * size + raw.size] = raw
    host[size + 24] ^= 1            # second record: code_bits no longer matches the bits
    dev = torch.from_numpy(host).cuda()
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    sq.sq_calib_import(dev, 2, 32, status)
    torch.cuda.synchronize()
    assert status.cpu().tolist() == [0, sq.SQ_ERR_RECORD]
