"""Pins of the oracle's causal prefill attention over the compressed cache (the
prefill attention kernel of [FQ-TQ] "FlashQuant：生产级KV缓存压缩方案…", section
"架构设计": queries of many positions against the compressed keys, decompressed on
the fly).

Reading: query i of a chunk at positions q_start .. q_start + Tq - 1 attends causally
to the sequence's tokens 0 .. q_start + i, whose keys and values are already in the
cache, with the same score estimator as the decode.  Pinned against brute-force
attention over the decompressed keys (the estimator's k~) and values, written here
with numpy, and against the one-token and full-length special cases.
"""
import math

import numpy as np
import pytest
from scipy import special

D = 128


def _cache(orc, o, T, Hkv, rng):
    nb = (T + 15) // 16 + 2
    bt = rng.permutation(nb)[: (T + 15) // 16].astype(np.int32)
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    t = np.arange(T)
    slots = (bt[t // 16] * 16 + t % 16).astype(np.int32)
    o.compress_paged(0, (rng.standard_normal((T, Hkv, D)) * 2).astype(np.float16), slots, kc)
    o.compress_paged(1, rng.standard_normal((T, Hkv, D)).astype(np.float16), slots, vc)
    return kc, vc, bt, slots


@pytest.mark.parametrize("q_start,Tq,Hkv,G,km", [(0, 21, 1, 3, 0), (37, 30, 2, 2, 0), (100, 9, 2, 4, 1)])
def test_prefill_is_causal_attention_over_decompressed_tokens(orc, q_start, Tq, Hkv, G, km):
    rng = np.random.default_rng(q_start + Tq)
    o = orc.Oracle(D, 4, 5, key_mode=km)
    T = q_start + Tq
    kc, vc, bt, slots = _cache(orc, o, T, Hkv, rng)
    q = rng.standard_normal((Tq, G * Hkv, D)) / math.sqrt(D)
    got = o.prefill(q, kc, vc, bt, q_start, Hkv)
    kt = o.decompress_paged(0, kc, slots, Hkv)   # k~ (the estimator's key) or k_hat (MSE keys)
    vt = o.decompress_paged(1, vc, slots, Hkv)
    for i in range(Tq):
        n = q_start + i + 1
        for h in range(G * Hkv):
            p = special.softmax(kt[:n, h // G] @ q[i, h] / math.sqrt(D))
            assert np.abs(got[i, h] - p @ vt[:n, h // G]).max() < 1e-12


def test_prefill_special_cases(orc):
    rng = np.random.default_rng(3)
    o = orc.Oracle(D, 4, 6)
    kc, vc, bt, slots = _cache(orc, o, 40, 1, rng)
    vt = o.decompress_paged(1, vc, slots, 1)
    q = rng.standard_normal((40, 2, D)) / math.sqrt(D)
    # the first query sees one token: its value
    first = o.prefill(q[:1], kc, vc, bt, 0, 1)
    assert np.abs(first[0] - vt[0, 0]).max() < 1e-12
    # the last query of a chunk is the decode of the whole sequence
    last = o.prefill(q[30:], kc, vc, bt, 30, 1)[-1]
    dec = o.decode(q[39:], kc, vc, bt[None], np.array([40], np.int32), 1)[0]
    assert np.abs(last - dec).max() < 1e-13
