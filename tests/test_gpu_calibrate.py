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

from gpu_helpers import calibrate_oracle, compare_compressed, read_records, records_to_device
from oracle import calibration as ocal
from oracle import codebook as ocb
from oracle import rng as orng
from synthetic import make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from compressed_attention_head_b200 import sq  # noqa: E402


def _gpu_calibrate(x_cal, avg_bits, is_key, qjl=True, seed=42, max_sweeps=30, rotation=0, cumvar=0.0):
    nh, n, d = x_cal.shape
    p = sq.calib_params(d, nh, avg_bits, is_key, qjl=qjl, seed=seed, max_sweeps=max_sweeps, rotation=rotation,
                        cumvar=cumvar)
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


@pytest.mark.parametrize("name", ["llama8b", "gemma9b_sweep"])
def test_random_rotation_matches_the_oracle(name):
    """The random-rotation variant (the A/B baseline): the basis is a
    deterministic function of the seed and head, so the GPU's basis,
    variances, widths and d_eff equal the oracle's (to float64 rounding of a
    Gram-Schmidt against a Householder QR); the spectral basis beats it on the
    expected distortion of the same budget."""
    w = make_workload(name, batch=1, tokens=16)
    cfg = w.cfg
    nh = 2
    for xcal, bits, is_key in ((w.k_cal[:nh], cfg["bits_k"], True), (w.v_cal[:nh], cfg["bits_v"], False)):
        gpu, status = _gpu_calibrate(xcal, bits, is_key, seed=11, rotation=1)
        assert status == [0] * nh
        for h, g in enumerate(gpu):
            r = ocal.calibrate(xcal[h].double().numpy(), avg_bits=bits, is_key=is_key, seed=11, stream=h,
                               rotation="random")
            assert g.flags == r.flags and g.flags & ocal.FLAG_RANDOM_ROTATION
            assert np.max(np.abs(g.V - r.V)) < 1e-10
            assert np.max(np.abs(g.lam - r.lam)) < 1e-10 * r.lam[0]
            assert g.d_eff == r.d_eff and g.m == r.m
            assert np.array_equal(g.bits, r.bits)
            spec = ocal.calibrate(xcal[h].double().numpy(), avg_bits=bits, is_key=is_key, stream=h)
            dist = ocb.distortion_table()
            assert np.sum(spec.sigma ** 2 * dist[spec.bits]) < np.sum(r.sigma ** 2 * dist[r.bits])


def test_random_rotation_records_compress_like_the_oracle():
    """Compression with random-rotation records (imported from the oracle)."""
    w = make_workload("llama8b", batch=1, tokens=200)
    cals = [ocal.calibrate(w.k_cal[h].double().numpy(), avg_bits=3.0, is_key=True, seed=5, stream=h,
                           rotation="random") for h in range(2)]
    recs = records_to_device(cals)
    kc = sq.alloc_cache(1, 2, 200, cals[0].words, True)
    x = w.k[:, :2].contiguous()
    sq.sq_compress_kv(recs, None, x.cuda(), None, 1, 2, 128, 200, None, kc, None)
    torch.cuda.synchronize()
    words = kc.words_u32()
    for h in range(2):
        compare_compressed(words[0, h, :200], kc.norm[0, h, :200].cpu().numpy(), kc.rnorm[0, h, :200].cpu().numpy(),
                           x[0, h].double().numpy(), cals[h])


@pytest.mark.parametrize("name", ["llama8b", "qwen1_5b_long"])
def test_cumulative_variance_d_eff(name):
    """d_eff by cumulative variance (0.9 of the trace): the GPU's d_eff is the
    oracle's rule applied to the GPU's eigenvalues and equals the oracle's."""
    w = make_workload(name, batch=1, tokens=16)
    for xcal, bits, is_key in ((w.k_cal[:2], 3.0, True), (w.v_cal[:2], 3.0, False)):
        gpu, status = _gpu_calibrate(xcal, bits, is_key, cumvar=0.9)
        assert status == [0, 0]
        for h, g in enumerate(gpu):
            r = ocal.calibrate(xcal[h].double().numpy(), avg_bits=bits, is_key=is_key, stream=h, cumvar=0.9)
            assert g.d_eff == ocal.effective_dim(g.lam, cumvar=0.9) == r.d_eff
            assert g.flags & ocal.FLAG_CUMVAR and g.m == (r.m if is_key else 0)
