"""The allocation-free decode entry point (for callers that cannot allocate device
memory at the call site, e.g. a runtime that owns all of HBM through its own
allocator) must give the same attention output as the workspace entry point.

Kept in its own file, collected last, so a failure here leaves every other test
already run.  Works alone in a fresh process and after the rest of the suite.
"""
import math

import numpy as np
import pytest

from parity import DECODE_ATOL, gpu_ctx

pytestmark = pytest.mark.gpu


def _case(orc, seed):
    rng = np.random.default_rng(seed)
    o = orc.Oracle(128, 4, 5)
    B, Hkv, G, T = 3, 4, 4, 700
    nbps = (T + 15) // 16
    nb = B * nbps + 5
    bt = rng.permutation(nb)[: B * nbps].reshape(B, nbps).astype(np.int32)
    seq = np.array([T, 333, 1], np.int32)
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    for b in range(B):
        t = np.arange(T)
        sl = (bt[b][t // 16] * 16 + t % 16).astype(np.int32)
        o.compress_paged(0, (rng.standard_normal((T, Hkv, 128)) * 2).astype(np.float16), sl, kc)
        o.compress_paged(1, rng.standard_normal((T, Hkv, 128)).astype(np.float16), sl, vc)
    qs = [(rng.standard_normal((B, G * Hkv, 128)) / math.sqrt(128)).astype(np.float16) for _ in range(2)]
    return o, kc, vc, bt, seq, qs, T, Hkv


def test_noalloc_decode_matches_workspace_decode(orc):
    import torch
    from kv_cache_vector_02_b200 import tq
    o, kc, vc, bt, seq, qs, T, Hkv = _case(orc, 11)
    dev = torch.device("cuda")
    ctx = gpu_ctx(4, 5, 0, 0)
    kc_d, vc_d = torch.as_tensor(kc, device=dev), torch.as_tensor(vc, device=dev)
    bt_d, sl_d = torch.as_tensor(bt, device=dev), torch.as_tensor(seq, device=dev)
    need = tq.tq_decode_workspace_bytes(ctx, bt.shape[0], qs[0].shape[1], Hkv, T)
    assert need <= tq.NOALLOC_SCRATCH_BYTES
    ws = torch.zeros(need, dtype=torch.uint8, device=dev)
    for q in qs:  # two calls in a row (the scratch keeps the previous call's contents)
        q_d = torch.as_tensor(q, device=dev)
        ref = torch.empty((q.shape[0], q.shape[1], 128), dtype=torch.float32, device=dev)
        got = torch.empty_like(ref)
        tq.tq_decode_attention(ctx, q_d, kc_d, vc_d, bt_d, sl_d, T, ref, ws, Hkv=Hkv)
        tq.tq_decode_attention_noalloc(ctx, q_d, kc_d, vc_d, bt_d, sl_d, T, got, Hkv=Hkv)
        torch.cuda.synchronize()
        assert tq.tq_get_device_error(ctx) == 0
        assert np.abs(got.cpu().numpy() - ref.cpu().numpy()).max() <= DECODE_ATOL
        want = o.decode(q.astype(np.float64), kc, vc, bt, seq, Hkv)
        assert np.abs(got.cpu().numpy() - want).max() <= DECODE_ATOL


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
