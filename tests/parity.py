"""Acceptance rules of the CUDA path against the oracle, and GPU run helpers.

Tolerances (from the statement of the problem; readings noted):
  * codes and signs are bit-exact, except coordinates whose oracle value lies
    within WINDOW * ||x|| of the boundary it crossed, and at most
    MAX_MISMATCH_RATE of all coordinates may differ that way.
      - code j: the coordinate is y_j = (R^T x)_j, its boundary t_k ||x|| / sqrt(d)
        (in the oracle's diagnostic units v = sqrt(d) y / ||x|| the window is
        WINDOW * sqrt(d));
      - sign j: the coordinate is (S r)_j and its boundary 0, so the window is
        |(S r)_j| < WINDOW * ||x|| (the oracle reports sk = (S r)_j / ||x||).
  * norms and gammas within NORM_RTOL relative.  A vector that carries an
    allowed code mismatch has a (slightly) different residual, so its signs are
    not compared and its gamma only within EXCLUDED_GAMMA_RTOL (a boundary
    coordinate sits half a cell from both levels, so |r| barely moves); such
    vectors are counted and may be at most the allowed mismatches.
  * decode output within DECODE_ATOL max-abs of the oracle on the same cache.

Every comparison appends its counts to STATS; the test session prints them at
the end (see conftest.py).
"""
from __future__ import annotations

import math

import numpy as np

WINDOW = 1e-6
MAX_MISMATCH_RATE = 1e-5
NORM_RTOL = 1e-6
EXCLUDED_GAMMA_RTOL = 1e-5
DECODE_ATOL = 2e-3
D = 128

STATS: list = []   # (label, dict) of every compress / decode comparison in the session


def record(label: str, stats: dict):
    STATS.append((label, dict(stats)))


def compare_compress(o, kind, x, got, label=""):
    """x: [N, 128] fp16 inputs; got: dict from oracle.read_paged of the GPU bytes,
    flattened to [N, ...].  Returns stats; raises AssertionError on a violation."""
    ref = o.compress_vectors(kind, np.asarray(x, np.float64), diagnostics=True)
    code_win = WINDOW * math.sqrt(D)
    N = ref["codes"].shape[0]
    cg = got["codes"].reshape(N, D)
    cr = ref["codes"]
    _, t = o.codebook(kind)
    mis = cg != cr
    bad_code = 0
    vec_with_code_mis = np.zeros(N, bool)
    if mis.any():
        ii, jj = np.nonzero(mis)
        for i, j in zip(ii, jj):
            a, b = int(cg[i, j]), int(cr[i, j])
            v = ref["v"][i, j]
            ok = abs(a - b) == 1 and abs(v - t[min(a, b)]) < code_win
            if not ok:
                bad_code += 1
            vec_with_code_mis[i] = True
    n_mis = int(mis.sum())
    stats = {"vectors": N, "coords": N * D, "code_mismatch": n_mis, "code_bad": bad_code,
             "excluded_vectors": int(vec_with_code_mis.sum())}
    # norms (stored fp32): relative 1e-6 against the exact norm
    ng = got["norm"].reshape(N)
    nr = ref["norm"]
    nz = nr > 0
    rel = np.zeros(N)
    rel[nz] = np.abs(ng[nz] - nr[nz]) / nr[nz]
    stats["norm_max_rel"] = float(rel.max()) if N else 0.0
    assert np.all(ng[~nz] == 0.0), label + ": zero vector with a non-zero norm"
    sign_mis = 0
    sign_bad = 0
    if o.is_prod(kind):
        keep = ~vec_with_code_mis
        sg = got["signs"].reshape(N, D)[keep]
        sr = ref["signs"][keep]
        sk = ref["sk"][keep]
        smis = sg != sr
        sign_mis = int(smis.sum())
        sign_bad = int((smis & (np.abs(sk) >= WINDOW)).sum())
        gg_all = got["gamma"].reshape(N)
        gr_all = ref["gamma"]
        gg, gr = gg_all[keep], gr_all[keep]
        gz = gr > 0
        grel = np.zeros(gr.shape)
        grel[gz] = np.abs(gg[gz] - gr[gz]) / gr[gz]
        assert np.all(gg[~gz] == 0.0), label + ": zero residual with a non-zero gamma"
        stats["gamma_max_rel"] = float(grel.max()) if grel.size else 0.0
        ex = vec_with_code_mis & (gr_all > 0)
        erel = np.abs(gg_all[ex] - gr_all[ex]) / gr_all[ex] if ex.any() else np.zeros(0)
        stats["excluded_gamma_max_rel"] = float(erel.max()) if erel.size else 0.0
    stats.update(sign_mismatch=sign_mis, sign_bad=sign_bad)
    coords = N * D
    record(label, stats)
    assert bad_code == 0, "%s: %d code mismatches outside the window (%s)" % (label, bad_code, stats)
    assert sign_bad == 0, "%s: %d sign mismatches outside the window (%s)" % (label, sign_bad, stats)
    allowed = MAX_MISMATCH_RATE * coords * (2 if o.is_prod(kind) else 1)
    assert n_mis + sign_mis <= allowed, "%s: too many boundary mismatches (%s)" % (label, stats)
    assert stats["excluded_vectors"] <= allowed, "%s: too many vectors with a code mismatch (%s)" % (label, stats)
    assert stats["norm_max_rel"] <= NORM_RTOL, "%s: norm (%s)" % (label, stats)
    if o.is_prod(kind):
        assert stats["gamma_max_rel"] <= NORM_RTOL, "%s: gamma (%s)" % (label, stats)
        assert stats["excluded_gamma_max_rel"] <= EXCLUDED_GAMMA_RTOL, "%s: gamma of excluded (%s)" % (label, stats)
    return stats


def check_decode(got, want, label="", atol=DECODE_ATOL):
    """Max-abs check of a decode output against the oracle; records the error."""
    err = float(np.abs(np.asarray(got, np.float64) - want).max()) if np.size(want) else 0.0
    record(label, {"decode_max_abs": err, "outputs": int(np.size(want))})
    assert err <= atol, "%s: decode max-abs %.3e > %.1e" % (label, err, atol)
    return err


def zero_gamma(o, kcache):
    """Copy of a prod key cache with every gamma zeroed: the oracle run on it is the
    estimator without its QJL term (a decode that dropped the term would match it)."""
    k0 = np.array(kcache, copy=True)
    k0[..., -16 * 4:] = 0   # gamma f32[16] is the last field of a prod key chunk
    return k0


# ----------------------------------------------------------------- GPU helpers
def torch_cuda():
    import torch
    return torch


def gpu_ctx(bits=4, seed=0, rot=0, km=0):
    from kv_cache_vector_02_b200 import tq
    return tq.tq_init(128, bits, seed, rot, km)


def gpu_compress(ctx, k, v, slots, num_blocks, Hkv):
    """k, v: torch fp16 tensors (any device; moved to cuda).  Returns device caches."""
    import torch
    from kv_cache_vector_02_b200 import tq
    dev = torch.device("cuda")
    kc = torch.zeros((num_blocks, Hkv, tq.tq_chunk_bytes(ctx, tq.KIND_KEY)), dtype=torch.uint8, device=dev)
    vc = torch.zeros((num_blocks, Hkv, tq.tq_chunk_bytes(ctx, tq.KIND_VALUE)), dtype=torch.uint8, device=dev)
    sl = torch.as_tensor(np.asarray(slots, np.int32), device=dev)
    tq.tq_compress(ctx, None if k is None else k.to(dev).contiguous(), None if v is None else v.to(dev).contiguous(),
                   sl, kc, vc)
    torch.cuda.synchronize()
    return kc, vc
