"""Failure detection on the GPU: a bounded wait that runs out.

tq_debug_stall makes the next launches withhold what their waits expect (the
compress kernels skip their input copies; the decode kernel's CTAs do not publish
the partial results another CTA merges), so those waits (on a flag nothing will
set) give up after their bounded limit.  The kernel must then report TQ_DEVERR_TIMEOUT through the device error
word, release what it holds and return; the context must stay usable and the
next ordinary call must again match the oracle exactly.  Nothing here faults,
traps or hangs a GPU.
"""
import time

import numpy as np
import pytest

from parity import check_decode, compare_compress, gpu_compress, gpu_ctx

pytestmark = pytest.mark.gpu


def _inputs(T=300, H=2, seed=4):
    import torch
    rng = np.random.default_rng(seed)
    k = torch.as_tensor((rng.standard_normal((T, H, 128)) * 2).astype(np.float16))
    v = torch.as_tensor(rng.standard_normal((T, H, 128)).astype(np.float16))
    nb = (T + 15) // 16
    slots = np.arange(T, dtype=np.int32)
    return k, v, slots, nb


@pytest.mark.parametrize("rot,bits,km", [(0, 4, 0), (1, 2, 1)])
def test_compress_wait_runs_out_then_context_recovers(orc, rot, bits, km):
    import torch
    from kv_cache_vector_02_b200 import tq
    ctx = gpu_ctx(bits, 3, rot, km)
    k, v, slots, nb = _inputs()
    tq.tq_debug_stall(ctx, 1)          # the key launch of the next call loads nothing
    t0 = time.time()
    gpu_compress(ctx, k, v, slots, nb, 2)
    dt = time.time() - t0
    err = tq.tq_get_device_error(ctx)
    assert err & tq.DEVERR_TIMEOUT, err
    assert dt >= 1.0, dt               # the key kernel waited out its limit ...
    assert dt < 60.0, dt               # ... and then returned
    # same context, ordinary call: exact again
    kc, vc = gpu_compress(ctx, k, v, slots, nb, 2)
    assert tq.tq_get_device_error(ctx) == 0
    o = orc.Oracle(128, bits, 3, rot=rot, key_mode=km)
    for kind, x, c in ((0, k, kc), (1, v, vc)):
        got = o.read_paged(kind, c.cpu().numpy(), slots, 2)
        xs = x.numpy().reshape(-1, 128)
        got = {kk: (vv.reshape(xs.shape[0], -1) if vv is not None and vv.ndim == 3 else
                    (vv.reshape(-1) if vv is not None else None)) for kk, vv in got.items()}
        compare_compress(o, kind, xs, got, "after timeout rot%d b%d km%d kind %d" % (rot, bits, km, kind))
    torch.cuda.synchronize()


def test_decode_wait_runs_out_then_context_recovers(orc):
    import torch
    from kv_cache_vector_02_b200 import tq
    o = orc.Oracle(128, 4, 3)
    rng = np.random.default_rng(9)
    B, T, Hkv, G = 2, 300, 2, 4
    nbps = (T + 15) // 16
    nb = B * nbps
    bt = rng.permutation(nb).reshape(B, nbps).astype(np.int32)
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    for b in range(B):
        t = np.arange(T)
        sl = (bt[b][t // 16] * 16 + t % 16).astype(np.int32)
        o.compress_paged(0, (rng.standard_normal((T, Hkv, 128)) * 2).astype(np.float16), sl, kc)
        o.compress_paged(1, rng.standard_normal((T, Hkv, 128)).astype(np.float16), sl, vc)
    q = (rng.standard_normal((B, G * Hkv, 128)) / 11).astype(np.float16)
    seq = np.array([T, 211], np.int32)
    ctx = gpu_ctx(4, 3, 0, 0)
    dev = torch.device("cuda")
    args = (torch.as_tensor(q, device=dev), torch.as_tensor(kc, device=dev), torch.as_tensor(vc, device=dev),
            torch.as_tensor(bt, device=dev), torch.as_tensor(seq, device=dev), T)
    ws = torch.full((tq.tq_decode_workspace_bytes(ctx, B, G * Hkv, Hkv, T),), 0xFF, dtype=torch.uint8, device=dev)
    out = torch.empty((B, G * Hkv, 128), dtype=torch.float32, device=dev)
    tq.tq_debug_stall(ctx, 1)          # the next decode publishes no partial result (unit 1 spans 2 CTAs)
    t0 = time.time()
    tq.tq_decode_attention(ctx, *args, out, ws, Hkv=Hkv)
    torch.cuda.synchronize()
    dt = time.time() - t0
    err = tq.tq_get_device_error(ctx)
    assert err & tq.DEVERR_TIMEOUT, err
    assert 1.0 <= dt < 60.0, dt
    tq.tq_decode_attention(ctx, *args, out, ws, Hkv=Hkv)
    torch.cuda.synchronize()
    assert tq.tq_get_device_error(ctx) == 0
    want = o.decode(q.astype(np.float64), kc, vc, bt, seq, Hkv)
    check_decode(out.cpu().numpy(), want, "decode after timeout")
