"""Repeated runs on the same inputs give the same bytes: a guard against races
between the kernels' producer / consumer stages (a stage refilled while a
consumer still reads it changes the output from run to run)."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rot", [0, 1])
def test_compress_and_decode_are_deterministic(rot):
    import torch
    from kv_cache_vector_02_b200 import tq, workloads as W
    w = W.WORKLOADS["batched"].with_(rotation=rot)
    dev = torch.device("cuda")
    ctx = tq.tq_init(128, w.bits, w.param_seed, w.rotation, w.key_mode)
    bt_np = W.block_table(w)
    slots = torch.as_tensor(W.prefill_slots(w, bt_np), device=dev)
    k, v = W.gen_kv(w, 0, device=dev), W.gen_kv(w, 1, device=dev)
    shape = lambda kind: (w.num_blocks, w.Hkv, tq.tq_chunk_bytes(ctx, kind))  # noqa: E731
    kc0 = torch.zeros(shape(tq.KIND_KEY), dtype=torch.uint8, device=dev)
    vc0 = torch.zeros(shape(tq.KIND_VALUE), dtype=torch.uint8, device=dev)
    tq.tq_compress(ctx, k, v, slots, kc0, vc0)
    bt = torch.as_tensor(bt_np, device=dev)
    seq = torch.full((w.B,), w.T, dtype=torch.int32, device=dev)
    q = W.gen_q(w, 0, device=dev)
    ws = torch.zeros(tq.tq_decode_workspace_bytes(ctx, w.B, w.Hq, w.Hkv, w.T), dtype=torch.uint8, device=dev)
    out0 = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=dev)
    tq.tq_decode_attention(ctx, q, kc0, vc0, bt, seq, w.T, out0, ws)
    kc, vc, out = torch.empty_like(kc0), torch.empty_like(vc0), torch.empty_like(out0)
    for _ in range(8):
        kc.zero_()
        vc.zero_()
        tq.tq_compress(ctx, k, v, slots, kc, vc)
        tq.tq_decode_attention(ctx, q, kc, vc, bt, seq, w.T, out, ws)
        torch.cuda.synchronize()
        assert torch.equal(kc, kc0), "key pages differ between runs"
        assert torch.equal(vc, vc0), "value pages differ between runs"
        assert torch.equal(out, out0), "decode output differs between runs"
    assert tq.tq_get_device_error(ctx) == 0
