"""GPU parity with the exact-d (spherical Beta) Lloyd-Max codebooks
(tq_init_ex with TQ_FLAG_SPHERE_CODEBOOK; [TQ-RS] "Étape 2" / "Couche 2"): the
same kernels run with the other codebook and bucketize tables, against the
oracle built with the same codebook."""
import math

import numpy as np
import pytest

from parity import check_decode, compare_compress

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rot,bits,km", [(0, 4, 0), (1, 3, 1), (0, 2, 0)])
def test_sphere_codebook_compress_and_decode(orc, rot, bits, km):
    import torch
    from kv_cache_vector_02_b200 import tq, workloads as W
    ctx = tq.tq_init_ex(128, bits, 7, rot, km, tq.FLAG_SPHERE_CODEBOOK)
    o = orc.Oracle(128, bits, 7, rot=rot, key_mode=km, beta=True)
    w = W.WORKLOADS["llama8b"].with_(T=1024, decode_steps=0, rotation=rot, bits=bits, key_mode=km)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    k, v = W.gen_kv(w, 0), W.gen_kv(w, 1)
    dev = torch.device("cuda")
    kc = torch.zeros((w.num_blocks, w.Hkv, tq.tq_chunk_bytes(ctx, tq.KIND_KEY)), dtype=torch.uint8, device=dev)
    vc = torch.zeros((w.num_blocks, w.Hkv, tq.tq_chunk_bytes(ctx, tq.KIND_VALUE)), dtype=torch.uint8, device=dev)
    tq.tq_compress(ctx, k.to(dev), v.to(dev), torch.as_tensor(slots, device=dev), kc, vc)
    torch.cuda.synchronize()
    assert tq.tq_get_device_error(ctx) == 0
    for kind, x, c in ((0, k, kc), (1, v, vc)):
        got = o.read_paged(kind, c.cpu().numpy(), slots, w.Hkv)
        xs = x.numpy().reshape(-1, 128)
        got = {kk: (vv.reshape(xs.shape[0], -1) if vv is not None and vv.ndim == 3 else
                    (vv.reshape(-1) if vv is not None else None)) for kk, vv in got.items()}
        compare_compress(o, kind, xs, got, "sphere codebook rot%d b%d km%d kind %d" % (rot, bits, km, kind))
    q = (W.gen_q(w).numpy().astype(np.float32) * 3).astype(np.float16)
    seq = np.full(w.B, w.T, np.int32)
    out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_decode_workspace_bytes(ctx, w.B, w.Hq, w.Hkv, w.T), dtype=torch.uint8, device=dev)
    tq.tq_decode_attention(ctx, torch.as_tensor(q, device=dev), kc, vc, torch.as_tensor(bt, device=dev),
                           torch.as_tensor(seq, device=dev), w.T, out, ws)
    torch.cuda.synchronize()
    assert tq.tq_get_device_error(ctx) == 0
    want = o.decode(q.astype(np.float64), kc.cpu().numpy(), vc.cpu().numpy(), bt, seq, w.Hkv)
    check_decode(out.cpu().numpy(), want, "sphere codebook decode rot%d b%d km%d" % (rot, bits, km))
