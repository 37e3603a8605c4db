"""Pins of the layout and codebook variants ([TQ-RS] "TurboQuant : compresser le
KV-cache…", "Étape 2" / "Couche 2": the exact spherical-Beta Lloyd-Max codebook;
"Couche 3": packed indices -- here 3-bit codes as a dense bit string).

The exact-d codebook quantizes v = sqrt(d) u_1 of a unit vector u uniform on the
sphere, whose law is (u_1 + 1)/2 ~ Beta((d-1)/2, (d-1)/2).  Pinned by the 1-bit
closed form, Lloyd's two conditions recomputed here with scipy's Beta law and
quadrature, the large-d limit (the Gaussian codebook), and optimality on exact
sphere samples; the dense packing by round trips, its bit order and the chunk
sizes.
"""
import math

import numpy as np
import pytest
from scipy import integrate, special, stats

D = 128


def test_one_bit_closed_form(orc):
    # E|v| = sqrt(d) E|u_1| = sqrt(d) Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    c, t = orc.lloyd_max_beta(D, 1)
    want = math.sqrt(D) * math.exp(special.gammaln(D / 2) - special.gammaln((D + 1) / 2)) / math.sqrt(math.pi)
    assert abs(c[1] - want) < 1e-12 and abs(c[0] + want) < 1e-12 and abs(t[0]) < 1e-15


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_lloyd_conditions_of_the_beta_law(orc, bits):
    c, t = orc.lloyd_max_beta(D, bits)
    L = 1 << bits
    a = (D - 1) / 2
    law = stats.beta(a, a, loc=-math.sqrt(D), scale=2 * math.sqrt(D))   # the law of v = sqrt(d) u_1
    edges = np.concatenate([[-math.sqrt(D)], t, [math.sqrt(D)]])
    for j in range(L):
        lo, hi = edges[j], edges[j + 1]
        mass = law.cdf(hi) - law.cdf(lo) if hi <= 0 else law.sf(lo) - law.sf(hi)
        mom = integrate.quad(lambda v: v * law.pdf(v), lo, hi, epsabs=1e-14, epsrel=1e-13, limit=200)[0]
        assert abs(mom / mass - c[j]) < 1e-9, (j, mom / mass, c[j])          # centroid = conditional mean
    assert np.allclose(t, 0.5 * (c[1:] + c[:-1]), atol=1e-15, rtol=0)       # boundary = midpoint
    assert np.allclose(c, -c[::-1], atol=1e-13)                             # symmetric law, symmetric codebook


def test_large_d_limit_is_the_gaussian_codebook(orc):
    for bits in (2, 3):
        cb, _ = orc.lloyd_max_beta(1 << 16, bits)
        cg, _ = orc.lloyd_max(bits)
        assert np.abs(cb - cg).max() < 1e-4
    # and at d = 128 the two differ by O(1/d), not more
    cb, _ = orc.lloyd_max_beta(D, 4)
    cg, _ = orc.lloyd_max(4)
    assert 1e-4 < np.abs(cb - cg).max() < 0.1


def test_beta_codebook_is_better_on_exact_sphere_coordinates(orc):
    rng = np.random.default_rng(0)
    u = rng.standard_normal((40000, D))
    v = math.sqrt(D) * (u / np.linalg.norm(u, axis=1, keepdims=True)).ravel()
    for bits in (2, 3):
        cb, tb = orc.lloyd_max_beta(D, bits)
        cg, tg = orc.lloyd_max(bits)
        mse_b = np.mean((v - cb[np.searchsorted(tb, v, side="left")]) ** 2)
        mse_g = np.mean((v - cg[np.searchsorted(tg, v, side="left")]) ** 2)
        assert mse_b < mse_g


def test_dense3_round_trip_and_bit_order(orc):
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 8, 4096)
    assert np.array_equal(orc.unpack(orc.pack(codes, 3), codes.size, 3), codes)
    allc = np.tile(np.arange(8), 16)               # every code at every offset modulo 8
    assert np.array_equal(orc.unpack(orc.pack(allc, 3), allc.size, 3), allc)
    # code i in bits [3i, 3i+3), least significant bit first
    # 1 -> bits 0..2, 2 -> bits 3..5, 7 -> bits 6..8 (straddling bytes 0 and 1), 5 -> bits 21..23
    assert list(orc.pack([1, 2, 7, 0, 0, 0, 0, 5], 3)) == [0xD1, 0x01, 0xA0]


def test_dense3_chunk_sizes(orc):
    o4 = orc.Oracle(D, 4, 0, dense3=True)          # keys: 3-bit codes + signs + norm + gamma
    assert o4.chunk_bytes(orc.KIND_KEY) == 16 * (48 + 16 + 4 + 4)
    assert o4.chunk_bytes(orc.KIND_VALUE) == 16 * (64 + 4)   # 4-bit values keep nibbles
    o3 = orc.Oracle(D, 3, 0, key_mode=orc.KEY_MSE, dense3=True)
    assert o3.chunk_bytes(orc.KIND_VALUE) == 16 * (48 + 4) and o3.chunk_bytes(orc.KIND_KEY) == 16 * (48 + 4)
    o2 = orc.Oracle(D, 2, 0, dense3=True)          # no 3-bit codes: unchanged
    assert o2.chunk_bytes(orc.KIND_KEY) == 16 * (16 + 16 + 8) and o2.chunk_bytes(orc.KIND_VALUE) == 16 * (32 + 4)


@pytest.mark.parametrize("beta,dense3", [(True, False), (False, True), (True, True)])
def test_variants_compress_and_decode(orc, beta, dense3):
    """The variants run the same method: the MSE bound holds, the dense layout holds
    the same codes as the nibble layout, and decode equals brute-force attention."""
    o = orc.Oracle(D, 4, 12, beta=beta, dense3=dense3)
    onib = orc.Oracle(D, 4, 12, beta=beta)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((2000, D))
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    r = o.compress_vectors(orc.KIND_VALUE, x)
    xh = o.decompress_vectors(orc.KIND_VALUE, r["codes"], None, r["norm"])
    assert np.mean(np.sum((x - xh) ** 2, 1)) <= math.sqrt(3) * math.pi / 2 / 4 ** 4
    T, Hkv, G = 45, 2, 3
    kx = (rng.standard_normal((T, Hkv, D)) * 2).astype(np.float16)
    vx = rng.standard_normal((T, Hkv, D)).astype(np.float16)
    slots = np.arange(T, dtype=np.int32)
    nb = (T + 15) // 16
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    o.compress_paged(0, kx, slots, kc)
    o.compress_paged(1, vx, slots, vc)
    kn, vn = onib.new_cache(0, nb, Hkv), onib.new_cache(1, nb, Hkv)
    onib.compress_paged(0, kx, slots, kn)
    onib.compress_paged(1, vx, slots, vn)
    for kind, a, b in ((0, kc, kn), (1, vc, vn)):
        ra, rb = o.read_paged(kind, a, slots, Hkv), onib.read_paged(kind, b, slots, Hkv)
        assert np.array_equal(ra["codes"], rb["codes"]) and np.array_equal(ra["norm"], rb["norm"])
    q = rng.standard_normal((1, G * Hkv, D)) / math.sqrt(D)
    bt = np.arange(nb, dtype=np.int32)[None]
    out = o.decode(q, kc, vc, bt, np.array([T], np.int32), Hkv)
    kt = o.decompress_paged(0, kc, slots, Hkv)
    vt = o.decompress_paged(1, vc, slots, Hkv)
    for h in range(G * Hkv):
        p = special.softmax(kt[:, h // G] @ q[0, h] / math.sqrt(D))
        assert np.abs(out[0, h] - p @ vt[:, h // G]).max() < 1e-12
