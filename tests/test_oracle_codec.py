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


def _place(proj_target, S, r_other, j_free, iters=60):
    """A residual r with (S r)_j equal to proj_target(rho) for the free coordinate
    j_free, the other coordinate fixed: a small fixed-point iteration, since the
    band itself scales with rho = ||r||."""
    r = np.zeros(2)
    r[1 - j_free] = r_other
    for _ in range(iters):
        rho = float(np.linalg.norm(r))
        target = proj_target(rho)
        # solve row j of S r = target for r[j_free] (the row that carries it)
        row = 0 if j_free == 0 else 1
        r[j_free] = (target - S[row, 1 - j_free] * r[1 - j_free]) / S[row, j_free]
    return r


def test_qjl_bit_exemption_band():
    """A QJL bit is exempt exactly when |(S r)_j| <= 1e-5 * ||row j of S|| * rho,
    and every bit and rho of a token whose signal-dim code is exempt are exempt.

    S = [[3, 0], [4, 1]] has row norms 3 and sqrt(17) but column norms 5 and 1,
    so a rule built on column norms decides cases 2 and 3 the other way; rho is
    far from 1 in every case, so a rule without rho fails cases 1 and 3; the
    exempt bit is 0 in cases 1 and 4 and bit 1 in case 3, so swapped indices fail.
    """
    S = np.array([[3.0, 0.0], [4.0, 1.0]])
    head = _head([0, 0, 3], m=2, S=S, normalize=False)
    band = lambda j, rho: 1e-5 * np.linalg.norm(S[j]) * rho       # noqa: E731
    # (r, expected q_ex): bit 0 is driven by r0 alone (row 0 of S), bit 1 by 4 r0 + r1
    cases = [
        (_place(lambda rho: 0.5 * band(0, rho), S, -7.0, 0), [True, False]),     # 1: bit 0 at half the band
        (_place(lambda rho: 1.5 * band(0, rho), S, -7.0, 0), [False, False]),    # 2: 1.5 bands (column rule: inside)
        (None, [False, True]),                                                     # 3: bit 1 at 0.9 of its band
        (_place(lambda rho: 0.99 * band(0, rho), S, 5.0, 0), [True, False]),     # 4: just inside
        (_place(lambda rho: 1.01 * band(0, rho), S, 5.0, 0), [False, False]),    # 5: just outside
    ]
    # case 3: r0 = 2 fixed, r1 chosen so that (S r)_1 = 4 r0 + r1 = 0.9 band(1, rho)
    r = np.array([2.0, -8.0])
    for _ in range(60):
        rho = float(np.linalg.norm(r))
        r[1] = 0.9 * band(1, rho) - 4.0 * r[0]
    cases[2] = (r, [False, True])
    x = np.array([[c[0][0], c[0][1], 0.1] for c in cases])
    out = codec.compress(x, head)
    code_ex, q_ex, rho_ex = codec.exemptions(out, head)
    assert not code_ex.any() and not rho_ex.any()
    assert q_ex.tolist() == [c[1] for c in cases]
    # the projections sit where the cases put them (relative to the row band)
    ratios = np.abs(out["proj"]) / (1e-5 * np.linalg.norm(S, axis=1)[None, :] * out["rho64"][:, None])
    assert np.allclose([ratios[0, 0], ratios[1, 0], ratios[2, 1], ratios[3, 0], ratios[4, 0]],
                       [0.5, 1.5, 0.9, 0.99, 1.01], rtol=1e-6)
    assert np.all(out["rho64"] > 4.9)


def test_qjl_bits_of_a_token_with_an_exempt_signal_code():
    """A signal-dim code on a threshold makes rho and all m QJL bits of that token
    exempt, whatever the projections; a token without one has none exempt."""
    S = np.array([[1.0, 2.0], [-3.0, 0.5]])
    head = _head([2, 0, 1], m=2, S=S, normalize=False)
    _, t2, _ = cb.lloyd_max(2)
    x = np.array([[t2[2], 0.7, 0.3],        # coordinate 0 exactly on its threshold
                  [0.2, 0.7, 0.3]])          # nothing near a threshold or a zero projection
    out = codec.compress(x, head)
    code_ex, q_ex, rho_ex = codec.exemptions(out, head)
    assert code_ex.tolist() == [[True, False, False], [False, False, False]]
    assert rho_ex.tolist() == [True, False]
    assert q_ex.tolist() == [[True, True], [False, False]]
    assert np.min(np.abs(out["proj"][0])) > 1e-2     # exempt through the code, not through the band
