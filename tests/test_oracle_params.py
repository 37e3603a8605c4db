"""Pins of the oracle's parameter generation: RNG, Haar and Hadamard rotations,
QJL sign matrix, Gaussian Lloyd-Max codebooks.

Each check compares the oracle with something other than itself: a published
test vector, a closed form, a textbook table, a library routine (numpy QR,
scipy Hadamard, scipy quadrature) or a distributional property.
"""
import math
import os

import numpy as np
import pytest
from scipy import integrate, linalg, stats

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


# ----------------------------------------------------------------- RNG
def test_splitmix64_published_outputs(orc):
    want = [int(r, 16) for r in _golden_rows("splitmix64_seed0.txt")]
    got = [int(v) for v in orc.splitmix64(0, 0, 3)]
    assert got == want


def test_stream_tags_are_offset_states(orc):
    # stream (seed, tag) starts at state seed + tag * 2^48: stream (5, 1) equals
    # stream (5 + 2^48, 0)
    a = orc.splitmix64(5, 1, 8)
    b = orc.splitmix64(5 + (1 << 48), 0, 8)
    assert np.array_equal(a, b)


def test_uniform_open_interval_and_moments(orc):
    u = orc.uniform(3, 0, 200000)
    assert u.min() > 0.0 and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 4 * math.sqrt(1 / 12 / u.size)
    # top 53 bits of the word, centred in their cell
    w = orc.splitmix64(3, 0, 4)
    assert np.allclose(u[:4], ((w >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53, rtol=0, atol=0)


def test_box_muller_is_standard_normal(orc):
    z = orc.gaussian(11, 0, 400000)
    assert abs(z.mean()) < 4 / math.sqrt(z.size)
    assert abs(z.var() - 1.0) < 4 * math.sqrt(2 / z.size)
    # KS against the normal law, and even/odd outputs uncorrelated
    assert stats.kstest(z[:100000], "norm").pvalue > 1e-3
    assert abs(np.corrcoef(z[0::2], z[1::2])[0, 1]) < 4 / math.sqrt(z.size / 2)


def test_box_muller_pair_formula(orc):
    # first pair from the first two uniforms: sqrt(-2 ln u1) (cos, sin)(2 pi u2)
    u = orc.uniform(2, 0, 2)
    z = orc.gaussian(2, 0, 2)
    r = math.sqrt(-2 * math.log(u[0]))
    assert z[0] == pytest.approx(r * math.cos(2 * math.pi * u[1]), abs=1e-15)
    assert z[1] == pytest.approx(r * math.sin(2 * math.pi * u[1]), abs=1e-15)


def test_signs_top_bit(orc):
    s = orc.signs(9, 1, 4096)
    w = orc.splitmix64(9, 1, 4096)
    assert np.array_equal(s, np.where((w >> np.uint64(63)) == 1, -1, 1).astype(np.int8))
    assert abs(s.mean()) < 4 / math.sqrt(s.size)


# ----------------------------------------------------------------- Haar
@pytest.mark.parametrize("d", [8, 32, 128])
def test_haar_is_the_positive_diagonal_qr_factor(orc, d):
    seed = 17
    R = orc.haar(d, seed)
    G = orc.gaussian(seed, 0, d * d).reshape(d, d)
    assert np.abs(R.T @ R - np.eye(d)).max() < 1e-12
    T = R.T @ G   # the triangular factor of G = R T
    assert np.abs(np.tril(T, -1)).max() < 1e-10
    assert (np.diag(T) > 0).all()
    # numpy's QR with its sign fixed to a positive diagonal gives the same matrix
    Q, Rq = np.linalg.qr(G)
    Q = Q * np.sign(np.diag(Rq))
    assert np.abs(Q - R).max() < 1e-10


def test_haar_distribution_trace_moments(orc):
    # Haar on O(d): E[tr Q] = 0 and E[(tr Q)^2] = 1 (Diaconis-Shahshahani);
    # plain Householder QR without the sign fix does not have these moments.
    d, n = 6, 4000
    tr = np.array([np.trace(orc.haar(d, s)) for s in range(n)])
    assert abs(tr.mean()) < 4 * 1.0 / math.sqrt(n)
    assert abs((tr ** 2).mean() - 1.0) < 0.12


# ----------------------------------------------------------------- Hadamard
@pytest.mark.parametrize("d", [8, 64, 128])
def test_fwht_equals_sylvester_matrix(orc, d):
    H = linalg.hadamard(d)  # Sylvester order
    x = np.random.default_rng(d).standard_normal(d)
    assert np.abs(orc.fwht(x) - H @ x).max() < 1e-12
    assert np.array_equal(H @ H, d * np.eye(d))


def test_hadamard_rotation_matrix(orc):
    d = 128
    o = orc.Oracle(d, 4, 5, rot=orc.ROT_HADAMARD)
    D = o.hadamard_signs
    assert np.array_equal(D, orc.signs(5, 2, d))
    R = o.R
    want = np.diag(D.astype(np.float64)) @ linalg.hadamard(d) / math.sqrt(d)   # R = D H / sqrt(d)
    assert np.abs(R - want).max() < 1e-15
    x = np.random.default_rng(0).standard_normal(d)
    assert np.abs(R.T @ x - orc.fwht(D * x) / math.sqrt(d)).max() < 1e-12   # y = H D x / sqrt(d)
    assert np.abs(R.T @ R - np.eye(d)).max() < 1e-14


def test_qjl_matrix_from_stream(orc):
    o = orc.Oracle(128, 4, 21)
    assert np.array_equal(o.S, orc.signs(21, 1, 128 * 128).reshape(128, 128))
    assert set(np.unique(o.S)) == {-1, 1}


# ----------------------------------------------------------------- Lloyd-Max
def test_one_bit_closed_form(orc):
    c, t = orc.lloyd_max(1)
    s = math.sqrt(2 / math.pi)
    assert c[0] == pytest.approx(-s, abs=1e-15) and c[1] == pytest.approx(s, abs=1e-15)
    assert t[0] == 0.0


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_conditions_by_quadrature(orc, bits):
    c, t = orc.lloyd_max(bits)
    L = 1 << bits
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    for j in range(L):
        m0 = integrate.quad(stats.norm.pdf, edges[j], edges[j + 1], epsabs=1e-13, epsrel=1e-12)[0]
        m1 = integrate.quad(lambda x: x * stats.norm.pdf(x), edges[j], edges[j + 1], epsabs=1e-13, epsrel=1e-12)[0]
        assert c[j] == pytest.approx(m1 / m0, abs=1e-11)           # centroid = conditional mean
    assert np.abs(t - 0.5 * (c[:-1] + c[1:])).max() < 1e-15        # boundary = midpoint
    assert np.abs(c + c[::-1]).max() < 1e-13                       # symmetric
    assert abs(t[(L - 1) // 2]) < 1e-13                            # 0 is a boundary
    assert np.all(np.diff(c) > 0)


def _distortion(c, t):
    edges = np.concatenate([[-np.inf], t, [np.inf]])
    return sum(integrate.quad(lambda x, cj=c[j]: (x - cj) ** 2 * stats.norm.pdf(x), edges[j], edges[j + 1],
                              epsabs=1e-15, epsrel=1e-13)[0] for j in range(len(c)))


def test_textbook_table(orc):
    for row in _golden_rows("gaussian_lloyd_max.txt"):
        bits, lev, thr, mse = [p.strip() for p in row.split("|")]
        bits = int(bits)
        lev = np.array([float(v) for v in lev.split()])
        thr = np.array([float(v) for v in thr.split()])
        c, t = orc.lloyd_max(bits)
        L = 1 << bits
        assert np.abs(c[L // 2:] - lev).max() < 2e-4
        assert np.abs(t[(L - 1) // 2:] - thr).max() < 2e-4
        D = _distortion(c, t)
        assert D == pytest.approx(float(mse), rel=1e-3)
        # the page's bound (sqrt(3) pi / 2) / 4^b on the per-coordinate distortion
        assert D <= math.sqrt(3) * math.pi / 2 / 4 ** bits


def test_codebooks_of_a_context(orc):
    o = orc.Oracle(128, 4, 0, key_mode=orc.KEY_PROD)
    assert o.code_bits(orc.KIND_VALUE) == 4 and o.code_bits(orc.KIND_KEY) == 3
    cv, tv = o.codebook(orc.KIND_VALUE)
    ck, tk = o.codebook(orc.KIND_KEY)
    assert np.array_equal(cv, orc.lloyd_max(4)[0]) and np.array_equal(ck, orc.lloyd_max(3)[0])
    o2 = orc.Oracle(128, 4, 0, key_mode=orc.KEY_MSE)
    assert o2.code_bits(orc.KIND_KEY) == 4
