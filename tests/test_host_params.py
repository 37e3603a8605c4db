"""libtq's host-side parameter generation (its own Gram-Schmidt QR, Lloyd-Max
solver and random streams) against the independent oracle."""
import numpy as np
import pytest


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_02_b200 import build
    build.build()
    from kv_cache_vector_02_b200 import tq as mod
    return mod


@pytest.mark.parametrize("rot", [0, 1])
@pytest.mark.parametrize("bits,km", [(4, 0), (3, 0), (2, 0), (4, 1)])
@pytest.mark.parametrize("seed", [0, 12345])
def test_params_match_oracle(tq, orc, rot, bits, km, seed):
    ctx = tq.tq_init_host(128, bits, seed, rot, km)
    p = tq.tq_export_params(ctx)
    o = orc.Oracle(128, bits, seed, rot=rot, key_mode=km)
    assert np.abs(p["R"] - o.R).max() < 1e-12
    assert np.array_equal(p["S"], o.S)
    if rot == 1:
        assert np.array_equal(p["hsigns"], o.hadamard_signs)
    cv, tv = o.codebook(orc.KIND_VALUE)
    ck, tk = o.codebook(orc.KIND_KEY)
    assert np.abs(p["cv"] - cv).max() < 1e-13 and np.abs(p["tv"] - tv).max() < 1e-13
    assert np.abs(p["ck"] - ck).max() < 1e-13 and np.abs(p["tk"] - tk).max() < 1e-13
    assert tq.tq_code_bits(ctx, tq.KIND_KEY) == o.code_bits(orc.KIND_KEY)
    assert tq.tq_chunk_bytes(ctx, tq.KIND_KEY) == o.chunk_bytes(orc.KIND_KEY)
    assert tq.tq_chunk_bytes(ctx, tq.KIND_VALUE) == o.chunk_bytes(orc.KIND_VALUE)


def test_fp32_rotation_is_orthogonal(tq):
    # the single-precision copy used by the kernels: ||R^T R - I||_max < 1e-5
    p = tq.tq_export_params(tq.tq_init_host(128, 4, 0))
    R32 = p["R"].astype(np.float32).astype(np.float64)
    assert np.abs(R32.T @ R32 - np.eye(128)).max() < 1e-5


@pytest.mark.parametrize("bits,km", [(4, 0), (3, 1), (2, 0)])
def test_sphere_codebook_matches_oracle(tq, orc, bits, km):
    """libtq's exact-d codebook (angle form: reduction formula of the sine power)
    against the oracle's (incomplete beta continued fraction)."""
    ctx = tq.tq_init_ex(128, bits, 0, 0, km, tq.FLAG_SPHERE_CODEBOOK | tq.FLAG_HOST_ONLY)
    p = tq.tq_export_params(ctx)
    o = orc.Oracle(128, bits, 0, key_mode=km, beta=True)
    cv, tv = o.codebook(orc.KIND_VALUE)
    ck, tk = o.codebook(orc.KIND_KEY)
    assert np.abs(p["cv"] - cv).max() < 1e-11 and np.abs(p["tv"] - tv).max() < 1e-11
    assert np.abs(p["ck"] - ck).max() < 1e-11 and np.abs(p["tk"] - tk).max() < 1e-11
    g = tq.tq_export_params(tq.tq_init_host(128, bits, 0, 0, km))
    assert np.abs(p["cv"] - g["cv"]).max() > 1e-4   # really another codebook


def test_unknown_init_flag_is_refused(tq):
    import ctypes
    h = ctypes.c_void_p()
    assert tq._lib.tq_init_ex(128, 4, 0, 0, 0, 0x100, ctypes.byref(h)) == tq.TQ_ERR_UNSUPPORTED
