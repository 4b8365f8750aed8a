"""Pins of the oracle's codec: bit layout, quantization, QJL, reconstruction."""

import math

import numpy as np
import pytest

from oracle import calibration as cal
from oracle import codebook as cb
from oracle import codec, record, rng


def _head(bits, m=0, d=None, sigma=None, V=None, S=None, normalize=True, is_key=None):
    bits = np.asarray(bits, dtype=np.int64)
    d = d or len(bits)
    total = int(bits.sum()) + m
    return cal.HeadCalib(
        d=d, d_eff=max(m, 1), m=m, total_bits=total, code_bits=int(bits.sum()),
        words=(total + 31) // 32,
        flags=(cal.FLAG_IS_KEY if (is_key or m) else 0) | (cal.FLAG_QJL if m else 0)
        | (cal.FLAG_NORMALIZE if normalize else 0),
        sweeps=0, stream=0, max_bits=8, seed=0, trace=1.0, kappa=1.0, avg_bits=total / d,
        lam=np.ones(d), sigma=np.ones(d) if sigma is None else np.asarray(sigma, float),
        V=np.eye(d) if V is None else V, S=np.zeros((m, m)) if S is None else S,
        bits=bits, offsets=cal.bit_offsets(bits))


def test_pack_hand_built_examples(golden):
    for line in golden("pack_example.txt"):
        b_s, c_s, q_s, w_s = [p.strip() for p in line.split("|")]
        bits = [int(x) for x in b_s.split()]
        codes = np.array([[int(x) for x in c_s.split()]])
        qb = np.array([[int(x) for x in q_s.split()]]) if q_s else np.zeros((1, 0), np.int64)
        head = _head(bits, m=qb.shape[1])
        words = codec.pack(codes, qb, head)
        want = [int(x, 16) for x in w_s.split()]
        assert words[0].tolist() == want
        c2, q2 = codec.unpack(words, head)
        assert np.array_equal(c2, codes) and np.array_equal(q2, qb)


def test_pack_round_trip_random():
    r = np.random.default_rng(5)
    bits = np.sort(r.integers(0, 9, size=64))[::-1]
    head = _head(bits, m=7)
    codes = np.stack([r.integers(0, 2 ** b, size=200) if b else np.zeros(200, int) for b in bits], axis=1)
    qb = r.integers(0, 2, size=(200, 7))
    w = codec.pack(codes, qb, head)
    assert w.shape == (200, head.words) and w.dtype == np.uint32
    c2, q2 = codec.unpack(w, head)
    assert np.array_equal(c2, codes) and np.array_equal(q2, qb)
    # padding past B bits is zero
    used = head.total_bits
    if used % 32:
        assert np.all(w[:, -1] >> np.uint32(used % 32) == 0)


def test_record_round_trip():
    x = np.random.default_rng(0).standard_normal((300, 32)) * np.linspace(5, 0.5, 32)
    c = cal.calibrate(x, avg_bits=2.5, is_key=True, seed=9, stream=3)
    raw = record.write(c)
    assert len(raw) == record.canonical_bytes(32)
    c2 = record.read(raw + b"\0" * 100)
    for f in ("d", "d_eff", "m", "total_bits", "code_bits", "words", "flags", "stream", "seed"):
        assert getattr(c2, f) == getattr(c, f)
    for f in ("lam", "sigma", "V", "S", "bits", "offsets"):
        assert np.array_equal(getattr(c2, f), getattr(c, f))


def test_identity_basis_reduces_to_scalar_quantizer():
    """V = I, sigma = 1, unnormalized: each coordinate is quantized on its own."""
    r = np.random.default_rng(1)
    bits = np.array([3, 3, 2, 1, 8, 0])
    head = _head(bits, normalize=False)
    x = r.standard_normal((1000, 6))
    out = codec.compress(x, head)
    for i, b in enumerate(bits):
        if b:
            assert np.array_equal(out["codes"][:, i], cb.quantize(x[:, i], b))
    xh = codec.decompress(out["words"], out["norm"], out["rnorm"], head)
    for i, b in enumerate(bits):
        assert np.array_equal(xh[:, i], cb.dequantize(out["codes"][:, i], b))


def test_zero_vector():
    x = np.random.default_rng(2).standard_normal((64, 32))
    c = cal.calibrate(x, avg_bits=3.0, is_key=True, seed=1)
    out = codec.compress(np.zeros((1, 32)), c)
    assert out["norm"][0] == 0.0
    xh = codec.decompress(out["words"], out["norm"], out["rnorm"], c)
    assert np.all(xh == 0.0)


def test_eight_bits_everywhere_is_nearly_lossless():
    r = np.random.default_rng(3)
    x = r.standard_normal((500, 32)) * np.linspace(3, 1, 32)
    c = cal.calibrate(x, avg_bits=8.0, is_key=False)
    assert np.all(c.bits == 8)
    out = codec.compress(x, c)
    xh = codec.decompress(out["words"], out["norm"], out["rnorm"], c)
    rel = np.linalg.norm(xh - x, axis=1) / np.linalg.norm(x, axis=1)
    assert np.max(rel) < 0.03 and np.mean(rel) < 0.01


def test_distortion_matches_water_filling_objective():
    """E||u - u_hat||^2 ~ sum_i sigma_i^2 D(b_i) on data drawn from the calibrated spectrum."""
    r = np.random.default_rng(4)
    d = 32
    q, _ = np.linalg.qr(r.standard_normal((d, d)))
    lam = np.concatenate([np.full(4, 40.0), np.linspace(2, 0.5, d - 4)])
    xc = (r.standard_normal((200_000, d)) * np.sqrt(lam)) @ q.T
    c = cal.calibrate(xc, avg_bits=3.0, is_key=False, normalize=False)
    x = (r.standard_normal((50_000, d)) * np.sqrt(lam)) @ q.T
    out = codec.compress(x, c)
    xh = codec.decompress(out["words"], out["norm"], out["rnorm"], c)
    mse = np.mean(np.sum((x - xh) ** 2, axis=1))
    pred = np.sum(c.sigma ** 2 * cb.distortion_table()[c.bits])
    assert abs(mse - pred) / pred < 0.03


def test_quantization_decisions_at_thresholds():
    bits = np.array([3, 2])
    head = _head(bits, normalize=False)
    _, t3, _ = cb.lloyd_max(3)
    _, t2, _ = cb.lloyd_max(2)
    x = np.array([[t3[4], t2[2]], [np.nextafter(t3[4], 9), np.nextafter(t2[2], 9)]])
    out = codec.compress(x, head)
    assert out["codes"].tolist() == [[4, 2], [5, 3]]
    ex, _, _ = codec.exemptions(out, head)
    assert ex.all()


def test_qjl_estimator_unbiased_brute_force():
    """Mean over many independent S of the QJL inner-product estimate equals <q, r>.

    Gaussian closed form: E[<s, q> sign<s, r>] = sqrt(2/pi) <q, r> / ||r||, so
    sqrt(pi/2) / m * ||r|| * sum_j (S q)_j sign((S r)_j) is unbiased.
    """
    m = 3
    qv = np.array([0.7, -1.2, 0.4])
    rv = np.array([0.05, 0.02, -0.03])
    n = 20000
    est = np.empty(n)
    for s in range(n):
        S = rng.qjl_matrix(1000 + s, 0, m)
        head = _head([0, 0, 0], m=m, S=S, normalize=False, sigma=np.ones(3))
        # y equal to the residual itself (codes are absent, c_hat = 0)
        rho, qb, _ = codec.qjl_signs(rv[None, :], np.zeros((1, 3)), head)
        sgn = 2.0 * qb[0] - 1.0
        est[s] = codec.QJL_SCALE / m * rho[0] * np.dot(S @ qv, sgn)
    truth = float(qv @ rv)
    se = est.std() / math.sqrt(n)
    assert abs(est.mean() - truth) < 5 * se
    # variance bound of the m-projection estimator: <= (pi/2)/m * ||r||^2 ||q||^2
    assert est.var() <= (math.pi / 2) / m * (rv @ rv) * (qv @ qv) * 1.05


def test_qjl_residual_lives_on_signal_dims():
    x = np.random.default_rng(6).standard_normal((400, 32)) * np.concatenate([np.full(4, 10.0), np.ones(28)])
    c = cal.calibrate(x, avg_bits=3.0, is_key=True, seed=3)
    out = codec.compress(x[:50], c)
    # rho is the norm of the signal-dim residual in the normalized rotated domain
    norm, y = codec.rotate(x[:50], c)
    c_hat = codec.levels(out["codes"], c)
    r = y[:, :c.m] - c.sigma[:c.m] * c_hat[:, :c.m]
    assert np.allclose(out["rho64"], np.linalg.norm(r, axis=1), rtol=1e-12)
    # the QJL term adds only along the first m eigenvectors
    a = codec.decompress(out["words"], out["norm"], out["rnorm"], c, apply_qjl=True)
    b = codec.decompress(out["words"], out["norm"], out["rnorm"], c, apply_qjl=False)
    diff_rot = (a - b) @ c.V
    assert np.max(np.abs(diff_rot[:, c.m:])) < 1e-10 * np.max(np.abs(diff_rot))
