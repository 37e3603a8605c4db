"""Pins of the oracle's residual window ([TQ-RS] "TurboQuant : compresser le
KV-cache…", "Couche 5 — Fenêtre résiduelle" and "Couche 7", residual_window=128;
the KIVI page's fp16 residual of the most recent tokens): the last tokens of a
sequence stay in fp16 and join the same softmax as the compressed tokens.

Pinned against brute-force fp64 softmax attention written here with numpy over
the concatenation [decompressed tokens | window tokens], against the plain decode
when the window is empty, and against textbook attention when every token is in
the window.
"""
import math

import numpy as np
import pytest
from scipy import special

D = 128


def _case(orc, bits, km, rot, seed, B=2, Hkv=2, G=3, T=45, W=20):
    o = orc.Oracle(D, bits, 12, rot=rot, key_mode=km)
    rng = np.random.default_rng(seed)
    kx = (rng.standard_normal((T * B, Hkv, D)) * 2).astype(np.float16)
    vx = rng.standard_normal((T * B, Hkv, D)).astype(np.float16)
    nbps = (T + 15) // 16
    nb = B * nbps + 2
    bt = rng.permutation(nb)[: B * nbps].reshape(B, nbps).astype(np.int32)
    slots = np.concatenate([bt[b][np.arange(T) // 16] * 16 + np.arange(T) % 16 for b in range(B)]).astype(np.int32)
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    o.compress_paged(0, kx, slots, kc)
    o.compress_paged(1, vx, slots, vc)
    tk = (rng.standard_normal((B, W, Hkv, D)) * 2).astype(np.float16)
    tv = rng.standard_normal((B, W, Hkv, D)).astype(np.float16)
    q = rng.standard_normal((B, G * Hkv, D)) * 3 / math.sqrt(D)
    return o, kc, vc, bt, slots, tk, tv, q


@pytest.mark.parametrize("rot,bits,km", [(0, 4, 0), (1, 2, 0), (0, 3, 1)])
def test_window_matches_bruteforce(orc, rot, bits, km):
    B, Hkv, G, T, W = 2, 2, 3, 45, 20
    o, kc, vc, bt, slots, tk, tv, q = _case(orc, bits, km, rot, 3, B, Hkv, G, T, W)
    seq = np.array([T, 17], np.int32)
    tl = np.array([W, 5], np.int32)
    o0 = o.decode(q, kc, vc, bt, seq, Hkv, form=0, tail_k=tk, tail_v=tv, tail_lens=tl)
    o1 = o.decode(q, kc, vc, bt, seq, Hkv, form=1, tail_k=tk, tail_v=tv, tail_lens=tl)
    assert np.abs(o0 - o1).max() < 1e-12
    kt = o.decompress_paged(0, kc, slots, Hkv).reshape(B, T, Hkv, D)
    vt = o.decompress_paged(1, vc, slots, Hkv).reshape(B, T, Hkv, D)
    for b in range(B):
        for h in range(G * Hkv):
            g = h // G
            keys = np.concatenate([kt[b, :seq[b], g], tk[b, :tl[b], g].astype(np.float64)])
            vals = np.concatenate([vt[b, :seq[b], g], tv[b, :tl[b], g].astype(np.float64)])
            p = special.softmax(keys @ q[b, h] / math.sqrt(D))
            assert np.abs(o1[b, h] - p @ vals).max() < 1e-12


def test_empty_window_is_the_plain_decode(orc):
    o, kc, vc, bt, slots, tk, tv, q = _case(orc, 4, 0, 0, 4)
    seq = np.array([45, 30], np.int32)
    plain = o.decode(q, kc, vc, bt, seq, 2)
    win = o.decode(q, kc, vc, bt, seq, 2, tail_k=tk, tail_v=tv, tail_lens=np.zeros(2, np.int32))
    assert np.array_equal(plain, win)


def test_window_only_is_textbook_attention(orc):
    """No compressed token: exact softmax attention over the fp16 window."""
    B, Hkv, G, W = 2, 2, 3, 20
    o, kc, vc, bt, slots, tk, tv, q = _case(orc, 4, 0, 0, 5, B, Hkv, G, 45, W)
    tl = np.array([W, 1], np.int32)
    out = o.decode(q, kc, vc, bt, np.zeros(B, np.int32), Hkv, tail_k=tk, tail_v=tv, tail_lens=tl)
    for b in range(B):
        for h in range(G * Hkv):
            k = tk[b, :tl[b], h // G].astype(np.float64)
            v = tv[b, :tl[b], h // G].astype(np.float64)
            s = k @ q[b, h] / math.sqrt(D)
            e = np.exp(s - s.max())
            assert np.abs(out[b, h] - (e / e.sum()) @ v).max() < 1e-12
    # one window token: the output is that token's value exactly
    assert np.abs(out[1, :G] - tv[1, 0, 0].astype(np.float64)).max() < 1e-15


def test_window_length_out_of_range_is_refused(orc):
    o, kc, vc, bt, slots, tk, tv, q = _case(orc, 4, 0, 0, 6)
    with pytest.raises(ValueError):
        o.decode(q, kc, vc, bt, np.array([45, 30], np.int32), 2, tail_k=tk, tail_v=tv,
                 tail_lens=np.array([21, 0], np.int32))
