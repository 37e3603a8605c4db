"""The allocation-free decode entry point must give the same attention output as
the workspace entry point.

Some callers cannot allocate device memory when they decode: a serving runtime
that hands nearly all of HBM to its own KV-cache allocator at start-up (a fresh
cudaMalloc would fail or fragment it), or a caller that must not risk the
device-wide synchronisation that cudaMalloc / cudaFree can cause inside its
decode loop.  tq_decode_attention_noalloc serves them from a fixed per-device
array inside libtq instead of a caller workspace.

Kept in its own file, collected last, so a failure here leaves every other test
already run.  Works alone in a fresh process and after the rest of the suite.
"""
import math

import numpy as np
import pytest

from parity import DECODE_ATOL, check_decode, gpu_ctx

pytestmark = pytest.mark.gpu


def _case(orc, seed, B, Hkv, G, T, seq):
    rng = np.random.default_rng(seed)
    o = orc.Oracle(128, 4, 5)
    nbps = (T + 15) // 16
    nb = B * nbps + 5
    bt = rng.permutation(nb)[: B * nbps].reshape(B, nbps).astype(np.int32)
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    pool = min(nb, 64)   # distinct pages: the rest repeat them (the oracle cost stays small)
    tk = pool * 16
    sl = np.arange(tk, dtype=np.int32)
    o.compress_paged(0, (rng.standard_normal((tk, Hkv, 128)) * 2).astype(np.float16), sl, kc)
    o.compress_paged(1, rng.standard_normal((tk, Hkv, 128)).astype(np.float16), sl, vc)
    kc[pool:] = kc[rng.integers(0, pool, nb - pool)]
    vc[pool:] = vc[rng.integers(0, pool, nb - pool)]
    qs = [(rng.standard_normal((B, G * Hkv, 128)) * 2 / math.sqrt(128)).astype(np.float16) for _ in range(2)]
    return o, kc, vc, bt, np.asarray(seq, np.int32), qs


def _both_entry_points(orc, o, kc, vc, bt, seq, qs, T, Hkv, label):
    import torch
    from kv_cache_vector_02_b200 import tq
    dev = torch.device("cuda")
    ctx = gpu_ctx(4, 5, 0, 0)
    kc_d, vc_d = torch.as_tensor(kc, device=dev), torch.as_tensor(vc, device=dev)
    bt_d, sl_d = torch.as_tensor(bt, device=dev), torch.as_tensor(seq, device=dev)
    need = tq.tq_decode_workspace_bytes(ctx, bt.shape[0], qs[0].shape[1], Hkv, T)
    assert need <= tq.NOALLOC_SCRATCH_BYTES
    # the workspace arm starts from NaN bytes: nothing in a workspace has to start at zero
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=dev)
    for i, q in enumerate(qs):  # two calls in a row (the scratch keeps the previous call's contents)
        q_d = torch.as_tensor(q, device=dev)
        ref = torch.empty((q.shape[0], q.shape[1], 128), dtype=torch.float32, device=dev)
        got = torch.empty_like(ref)
        tq.tq_decode_attention(ctx, q_d, kc_d, vc_d, bt_d, sl_d, T, ref, ws, Hkv=Hkv)
        tq.tq_decode_attention_noalloc(ctx, q_d, kc_d, vc_d, bt_d, sl_d, T, got, Hkv=Hkv)
        torch.cuda.synchronize()
        assert tq.tq_get_device_error(ctx) == 0
        g, r = got.cpu().numpy(), ref.cpu().numpy()
        assert np.abs(g - r).max() <= DECODE_ATOL
        want = o.decode(q.astype(np.float64), kc, vc, bt, seq, Hkv)
        check_decode(g, want, "%s call %d (scratch %d of %d bytes)" % (label, i, need, tq.NOALLOC_SCRATCH_BYTES))
    return need


def test_noalloc_decode_matches_workspace_decode(orc):
    T = 700
    o, kc, vc, bt, seq, qs = _case(orc, 11, 3, 4, 4, T, [T, 333, 1])
    _both_entry_points(orc, o, kc, vc, bt, seq, qs, T, 4, "noalloc small")


def test_noalloc_request_just_under_the_limit(orc):
    """A plan whose scratch ends within a few KB of the array's end (an off-by-one
    in the plan's rounding against the fixed size would show here)."""
    from kv_cache_vector_02_b200 import tq
    ctx = gpu_ctx(4, 5, 0, 0)
    Hkv, G, T = 1, 16, 32
    lim = tq.NOALLOC_SCRATCH_BYTES
    # largest batch whose workspace fits, and how much a few more sequences add
    B = 1
    while tq.tq_decode_workspace_bytes(ctx, B * 2, G * Hkv, Hkv, T) <= lim:
        B *= 2
    lo, hi = B, B * 2
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if tq.tq_decode_workspace_bytes(ctx, mid, G * Hkv, Hkv, T) <= lim:
            lo = mid
        else:
            hi = mid
    B = lo
    need = tq.tq_decode_workspace_bytes(ctx, B, G * Hkv, Hkv, T)
    step = tq.tq_decode_workspace_bytes(ctx, B + 1, G * Hkv, Hkv, T) - need
    assert lim - need < max(step, 1) + 512, (need, step)
    rng = np.random.default_rng(3)
    seq = rng.integers(0, T + 1, B)
    seq[0] = T
    o, kc, vc, bt, seq, qs = _case(orc, 12, B, Hkv, G, T, seq)
    got_need = _both_entry_points(orc, o, kc, vc, bt, seq, qs, T, Hkv, "noalloc near limit B=%d" % B)
    assert got_need == need


def test_noalloc_refuses_more_than_its_scratch():
    import torch
    from kv_cache_vector_02_b200 import tq
    ctx = gpu_ctx()
    B, Hq, Hkv, L = 256, 64, 8, 131072
    assert tq.tq_decode_workspace_bytes(ctx, B, Hq, Hkv, L) > tq.NOALLOC_SCRATCH_BYTES
    dev = torch.device("cuda")
    q = torch.zeros((B, Hq, 128), dtype=torch.float16, device=dev)
    kc = torch.zeros((1, Hkv, 1408), dtype=torch.uint8, device=dev)
    vc = torch.zeros((1, Hkv, 1088), dtype=torch.uint8, device=dev)
    bt = torch.zeros((B, 1), dtype=torch.int32, device=dev)
    sl = torch.zeros(B, dtype=torch.int32, device=dev)
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device=dev)
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention_noalloc(ctx, q, kc, vc, bt, sl, L, out, Hkv=Hkv)
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    # the refusal happens exactly above the array's size
    Hkv, G, T = 1, 16, 32
    B = 1
    while tq.tq_decode_workspace_bytes(ctx, B, G * Hkv, Hkv, T) <= tq.NOALLOC_SCRATCH_BYTES:
        B += max(1, B // 8)
    q = torch.zeros((B, G * Hkv, 128), dtype=torch.float16, device=dev)
    kc = torch.zeros((1, Hkv, 1408), dtype=torch.uint8, device=dev)
    vc = torch.zeros((1, Hkv, 1088), dtype=torch.uint8, device=dev)
    bt = torch.zeros((B, 2), dtype=torch.int32, device=dev)
    sl = torch.zeros(B, dtype=torch.int32, device=dev)
    out = torch.empty((B, G * Hkv, 128), dtype=torch.float32, device=dev)
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention_noalloc(ctx, q, kc, vc, bt, sl, T, out, Hkv=Hkv)
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
