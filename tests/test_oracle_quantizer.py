"""Pins of the oracle's compress / decompress / QJL / packing / decode.

What fixes each check: the MSE bound and the 4-bit cosine floor printed on the
FlashQuant page ("TurboQuant" and "使用方式" sections), the unbiasedness and
O(1/d) variance claimed for the QJL estimator (its "QJL校正" section), the
nibble / 2-bit packing and the 68-byte vector of the page's tables, the
orthogonality invariant of the rotation, and brute-force fp64 attention on tiny
inputs written here with numpy / scipy.
"""
import math

import numpy as np
import pytest
from scipy import special

D = 128


def _unit_vectors(n, d, seed):
    x = np.random.default_rng(seed).standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


# ----------------------------------------------------------------- packing
@pytest.mark.parametrize("w", [1, 2, 4])
def test_pack_roundtrip_random_and_exhaustive(orc, w):
    rng = np.random.default_rng(w)
    codes = rng.integers(0, 1 << w, 4096)
    assert np.array_equal(orc.unpack(orc.pack(codes, w), codes.size, w), codes)
    # every byte value decodes and re-encodes to itself
    allbytes = np.arange(256, dtype=np.uint8)
    per = 8 // w
    assert np.array_equal(orc.pack(orc.unpack(allbytes, 256 * per, w), w), allbytes)


def test_pack_bit_order_convention(orc):
    # nibble: byte i = c[2i] | c[2i+1] << 4
    assert list(orc.pack([0x1, 0xF, 0x7, 0x2] + [0] * 12, 4)[:2]) == [0xF1, 0x27]
    # crumb: byte i = sum_k c[4i+k] << 2k
    assert orc.pack([1, 2, 3, 0] + [0] * 12, 2)[0] == 1 | 2 << 2 | 3 << 4
    # bit: byte i = sum_k b[8i+k] << k
    assert orc.pack([1, 0, 0, 0, 0, 0, 0, 1], 1)[0] == 0x81


def test_chunk_sizes_match_the_pages_byte_counts(orc):
    o4 = orc.Oracle(D, 4, 0)
    # values: 64 B of nibbles + 4 B fp32 norm = 68 B per vector, x 16 tokens
    assert o4.chunk_bytes(orc.KIND_VALUE) == 16 * 68
    # keys (3-bit code in nibbles + 16 B signs + norm + gamma) = 88 B per vector
    assert o4.chunk_bytes(orc.KIND_KEY) == 16 * 88
    o2 = orc.Oracle(D, 2, 0)
    assert o2.chunk_bytes(orc.KIND_VALUE) == 16 * 36 and o2.chunk_bytes(orc.KIND_KEY) == 16 * 40
    o3 = orc.Oracle(D, 3, 0)
    assert o3.chunk_bytes(orc.KIND_VALUE) == 16 * 68 and o3.chunk_bytes(orc.KIND_KEY) == 16 * 56
    om = orc.Oracle(D, 4, 0, key_mode=orc.KEY_MSE)
    assert om.chunk_bytes(orc.KIND_KEY) == 16 * 68


# ----------------------------------------------------------------- quantizer
@pytest.mark.parametrize("rot", [0, 1])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_mse_bound_on_unit_vectors(orc, bits, rot):
    # mean over 1e4 seeded random unit vectors of ||x - x_hat||^2 <= (sqrt(3) pi/2)/4^b
    o = orc.Oracle(D, bits, 1, rot=rot, key_mode=orc.KEY_MSE)
    x = _unit_vectors(10000, D, 100 + bits)
    out = o.compress_vectors(orc.KIND_VALUE, x)
    xh = o.decompress_vectors(orc.KIND_VALUE, out["codes"], None, out["norm"])
    mse = np.mean(np.sum((x - xh) ** 2, axis=1))
    assert mse <= math.sqrt(3) * math.pi / 2 / 4 ** bits
    # and close to the Gaussian Lloyd-Max distortion of the codebook
    Dg = {1: 0.363380, 2: 0.117482, 3: 0.034548, 4: 0.009501}[bits]
    assert abs(mse - Dg) / Dg < 0.05


def test_cosine_at_four_bits(orc):
    o = orc.Oracle(D, 4, 2)
    x = np.random.default_rng(5).standard_normal((4000, D)) * np.exp(0.5 * np.random.default_rng(6).standard_normal(D))
    out = o.compress_vectors(orc.KIND_VALUE, x)
    xh = o.decompress_vectors(orc.KIND_VALUE, out["codes"], None, out["norm"])
    cos = np.sum(x * xh, 1) / np.linalg.norm(x, axis=1) / np.linalg.norm(xh, axis=1)
    assert cos.mean() >= 0.95 and cos.min() > 0.95


def test_rotation_direction_is_R_transpose(orc):
    # x = +/- (column j of R)  =>  y = R^T x = +/- e_j: coordinate j takes the
    # top / bottom cell, every other coordinate sits at 0 (cell L/2-1 or L/2).
    o = orc.Oracle(D, 4, 3)
    R = o.R
    x = np.stack([R[:, 7], -R[:, 90]])
    c = o.compress_vectors(orc.KIND_VALUE, x)["codes"]
    assert c[0, 7] == 15 and c[1, 90] == 0
    others = np.delete(c[0], 7)
    assert set(np.unique(others)) <= {7, 8}


def test_zero_vector(orc):
    o = orc.Oracle(D, 4, 3)
    for kind, L in ((orc.KIND_VALUE, 16), (orc.KIND_KEY, 8)):
        out = o.compress_vectors(kind, np.zeros((1, D)))
        assert np.all(out["codes"] == L // 2 - 1) and out["norm"][0] == 0.0
        if kind == orc.KIND_KEY:
            assert np.all(out["signs"] == 1) and out["gamma"][0] == 0.0


def test_scale_invariance_of_codes(orc):
    # codes depend only on the direction x/||x|| (step 1 of the page)
    o = orc.Oracle(D, 4, 4)
    x = np.random.default_rng(0).standard_normal((64, D))
    a = o.compress_vectors(orc.KIND_VALUE, x)
    b = o.compress_vectors(orc.KIND_VALUE, 8.0 * x)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.allclose(b["norm"], 8 * a["norm"], rtol=1e-15)


def test_gamma_equals_rotated_domain_residual(orc):
    # ||x - x_hat|| (original domain) = n * ||u - c[idx]/sqrt(d)|| (rotated domain)
    o = orc.Oracle(D, 4, 6)
    x = np.random.default_rng(1).standard_normal((256, D))
    out = o.compress_vectors(orc.KIND_KEY, x, diagnostics=True)
    ck, _ = o.codebook(orc.KIND_KEY)
    u = out["v"] / math.sqrt(D)
    g = out["norm"] * np.linalg.norm(u - ck[out["codes"]] / math.sqrt(D), axis=1)
    assert np.abs(g - out["gamma"]).max() < 1e-12 * out["norm"].max()


def test_bucketize_matches_boundaries(orc):
    o = orc.Oracle(D, 4, 7)
    x = np.random.default_rng(2).standard_normal((512, D))
    out = o.compress_vectors(orc.KIND_VALUE, x, diagnostics=True)
    c, t = o.codebook(orc.KIND_VALUE)
    assert np.array_equal(out["codes"], np.searchsorted(t, out["v"], side="left"))


# ----------------------------------------------------------------- QJL
def _estimates(orc, q, k, seeds, bits=4, rot=0, d=D):
    est, mse_only = [], []
    for s in seeds:
        o = orc.Oracle(d, bits, s, rot=rot)
        out = o.compress_vectors(orc.KIND_KEY, k[None])
        kt = o.decompress_vectors(orc.KIND_KEY, out["codes"], out["signs"], out["norm"], out["gamma"])[0]
        est.append(q @ kt)
        # MSE-only reconstruction (the QJL term dropped)
        kh = o.decompress_vectors(orc.KIND_KEY, out["codes"], out["signs"], out["norm"], np.zeros(1))[0]
        mse_only.append(q @ kh)
    return np.array(est), np.array(mse_only)


@pytest.mark.slow
def test_qjl_estimator_unbiased_over_1000_seeds(orc):
    rng = np.random.default_rng(123)
    q = rng.standard_normal(D)
    k = 10.0 * q / np.linalg.norm(q) + rng.standard_normal(D)   # large <q,k>: gives the check power
    truth = q @ k
    est, mse_only = _estimates(orc, q, k, range(1000))
    e = est - truth
    assert abs(e.mean()) <= 3 * e.std(ddof=1) / math.sqrt(e.size)
    # power: the MSE-only inner product is shrunk and fails the same test
    e2 = mse_only - truth
    assert abs(e2.mean()) > 3 * e2.std(ddof=1) / math.sqrt(e2.size)


def test_qjl_decompress_matches_estimator(orc):
    # <q, k_tilde> = <q, k_hat> + gamma sqrt(pi/2)/d <S q, 2 sigma - 1>
    o = orc.Oracle(D, 4, 8)
    rng = np.random.default_rng(4)
    k = rng.standard_normal((32, D))
    q = rng.standard_normal(D)
    out = o.compress_vectors(orc.KIND_KEY, k)
    kt = o.decompress_vectors(orc.KIND_KEY, out["codes"], out["signs"], out["norm"], out["gamma"])
    kh = o.decompress_vectors(orc.KIND_KEY, out["codes"], out["signs"], out["norm"], np.zeros(32))
    sq = o.S.astype(np.float64) @ q
    est = kh @ q + out["gamma"] * math.sqrt(math.pi / 2) / D * ((2 * out["signs"] - 1) @ sq)
    assert np.abs(kt @ q - est).max() < 1e-12 * np.abs(est).max()


def test_qjl_signs_are_signs_of_the_residual_sketch(orc):
    o = orc.Oracle(D, 4, 9)
    k = np.random.default_rng(5).standard_normal((64, D))
    out = o.compress_vectors(orc.KIND_KEY, k, diagnostics=True)
    kh = o.decompress_vectors(orc.KIND_KEY, out["codes"], out["signs"], out["norm"], np.zeros(64))
    sk = (k - kh) @ o.S.T.astype(np.float64)
    assert np.array_equal(out["signs"], (sk >= 0).astype(np.int32))
    assert np.allclose(out["sk"] * out["norm"][:, None], sk, atol=1e-12)
    assert np.allclose(out["gamma"], np.linalg.norm(k - kh, axis=1), rtol=1e-13)


@pytest.mark.slow
def test_qjl_variance_scales_as_one_over_d(orc):
    # var(e) * d roughly constant for d in {32, 64, 128, 256}, with q, k of unit norm
    vals = []
    for d in (32, 64, 128, 256):
        rng = np.random.default_rng(d)
        q = rng.standard_normal(d)
        q /= np.linalg.norm(q)
        k = rng.standard_normal(d)
        k /= np.linalg.norm(k)
        est, _ = _estimates(orc, q, k, range(200), bits=2, rot=1, d=d)
        vals.append(np.var(est - q @ k) * d)
    assert max(vals) / min(vals) < 2.0


# ----------------------------------------------------------------- paged cache + decode
def _paged_case(orc, o, T, H, seed, shuffle=True):
    rng = np.random.default_rng(seed)
    x = {kind: rng.standard_normal((T, H, D)).astype(np.float16) for kind in (0, 1)}
    nb = (T + 15) // 16 + 3
    blocks = rng.permutation(nb)[: (T + 15) // 16] if shuffle else np.arange((T + 15) // 16)
    slots = (blocks[np.arange(T) // 16] * 16 + np.arange(T) % 16).astype(np.int32)
    caches = {}
    for kind in (0, 1):
        caches[kind] = o.new_cache(kind, nb, H)
        assert o.compress_paged(kind, x[kind], slots, caches[kind]) == 0
    return x, slots, blocks, caches


def test_paged_store_matches_vector_compress(orc):
    o = orc.Oracle(D, 4, 10)
    T, H = 37, 2
    x, slots, blocks, caches = _paged_case(orc, o, T, H, 0)
    for kind in (0, 1):
        got = o.read_paged(kind, caches[kind], slots, H)
        want = o.compress_vectors(kind, x[kind].reshape(-1, D))
        assert np.array_equal(got["codes"].reshape(-1, D), want["codes"])
        assert np.array_equal(got["norm"].reshape(-1), want["norm"].astype(np.float32).astype(np.float64))
        if kind == 0:
            assert np.array_equal(got["signs"].reshape(-1, D), want["signs"])
            assert np.array_equal(got["gamma"].reshape(-1), want["gamma"].astype(np.float32).astype(np.float64))


def test_paged_skips_out_of_range_slots(orc):
    o = orc.Oracle(D, 4, 10)
    cache = o.new_cache(1, 2, 1)
    x = np.ones((3, 1, D))
    assert o.compress_paged(1, x, np.array([0, 40, -1], np.int32), cache) == 1
    assert cache[1].sum() == 0 and cache[0].sum() != 0


@pytest.mark.parametrize("rot,bits,km", [(0, 4, 0), (1, 2, 0), (0, 3, 1)])
def test_decode_forms_agree_and_match_bruteforce(orc, rot, bits, km):
    o = orc.Oracle(D, bits, 12, rot=rot, key_mode=km)
    Hkv, G, B = 2, 3, 2
    T = 45
    rng = np.random.default_rng(7)
    kx = rng.standard_normal((T * B, Hkv, D)).astype(np.float16) * 2
    vx = rng.standard_normal((T * B, Hkv, D)).astype(np.float16)
    nbps = (T + 15) // 16
    nb = B * nbps + 2
    perm = rng.permutation(nb)
    bt = perm[: B * nbps].reshape(B, nbps).astype(np.int32)
    seq = np.array([T, 17], np.int32)
    slots = np.concatenate([bt[b][np.arange(T) // 16] * 16 + np.arange(T) % 16 for b in range(B)]).astype(np.int32)
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    o.compress_paged(0, kx, slots, kc)
    o.compress_paged(1, vx, slots, vc)
    q = rng.standard_normal((B, G * Hkv, D)) / math.sqrt(D)
    o0 = o.decode(q, kc, vc, bt, seq, Hkv, form=0)
    o1 = o.decode(q, kc, vc, bt, seq, Hkv, form=1)
    assert np.abs(o0 - o1).max() < 1e-12
    # brute force: softmax attention over the decompressed keys / values
    kt = o.decompress_paged(0, kc, slots, Hkv).reshape(B, T, Hkv, D)
    vt = o.decompress_paged(1, vc, slots, Hkv).reshape(B, T, Hkv, D)
    for b in range(B):
        for h in range(G * Hkv):
            g = h // G
            n = seq[b]
            s = kt[b, :n, g] @ q[b, h] / math.sqrt(D)
            p = special.softmax(s)
            want = p @ vt[b, :n, g]
            assert np.abs(o1[b, h] - want).max() < 1e-12


def test_decode_empty_sequence_and_bad_block(orc):
    o = orc.Oracle(D, 4, 13)
    kc, vc = o.new_cache(0, 2, 1), o.new_cache(1, 2, 1)
    q = np.ones((1, 1, D))
    out = o.decode(q, kc, vc, np.zeros((1, 1), np.int32), np.zeros(1, np.int32), 1)
    assert np.all(out == 0)
    with pytest.raises(ValueError):
        o.decode(q, kc, vc, np.array([[5]], np.int32), np.array([3], np.int32), 1)


def test_tie_goes_to_the_lower_cell(orc):
    # d = 64: the Hadamard rotation has entries exactly +-1/8, so x = D H e_j
    # rotates exactly to 8 e_j and every other coordinate lands exactly on the
    # boundary 0, which (ties going low) is not counted: cell L/2 - 1.
    from scipy import linalg
    d = 64
    o = orc.Oracle(d, 4, 14, rot=orc.ROT_HADAMARD)
    Dg = o.hadamard_signs.astype(np.float64)
    x = (Dg[:, None] * linalg.hadamard(d))[:, 5]
    out = o.compress_vectors(orc.KIND_VALUE, x[None], diagnostics=True)
    assert out["v"][0, 5] == 8.0 and np.all(np.delete(out["v"][0], 5) == 0.0)
    assert out["codes"][0, 5] == 15 and np.all(np.delete(out["codes"][0], 5) == 7)
