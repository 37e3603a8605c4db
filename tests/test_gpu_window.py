"""GPU parity of the fp16 residual window (tq_decode_attention_window) against the
oracle: the last tokens of each sequence stay uncompressed and join the same
softmax as the compressed pages ([TQ-RS] "Couche 5 — Fenêtre résiduelle",
"Couche 7" residual_window=128)."""
import numpy as np
import pytest

from parity import check_decode, gpu_compress, gpu_ctx, record

pytestmark = pytest.mark.gpu

WIN = 128


def _window(w, seed, device="cpu"):
    """fp16 window tokens of the workload's law: [B, WIN, Hkv, 128]."""
    from kv_cache_vector_02_b200 import workloads as W
    ww = w.with_(T=WIN, layers=1, decode_steps=0, data_seed=seed)
    k = W.gen_kv(ww, 0, device=device).reshape(w.B, WIN, w.Hkv, 128)
    v = W.gen_kv(ww, 1, device=device).reshape(w.B, WIN, w.Hkv, 128)
    return k.contiguous(), v.contiguous()


def _run(ctx, q, kc, vc, bt, seq, maxlen, tk, tv, tl, Hkv):
    import torch
    from kv_cache_vector_02_b200 import tq
    dev = torch.device("cuda")
    q = torch.as_tensor(q).to(dev)
    B, Hq = q.shape[0], q.shape[1]
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device=dev)
    ws = torch.full((tq.tq_decode_workspace_bytes(ctx, B, Hq, Hkv, maxlen),), 0xFF, dtype=torch.uint8, device=dev)
    tq.tq_decode_attention_window(ctx, q, torch.as_tensor(kc).to(dev), torch.as_tensor(vc).to(dev),
                                  torch.as_tensor(np.asarray(bt, np.int32)).to(dev),
                                  torch.as_tensor(np.asarray(seq, np.int32)).to(dev), maxlen,
                                  tk.to(dev), tv.to(dev), torch.as_tensor(np.asarray(tl, np.int32)).to(dev),
                                  out, ws, Hkv=Hkv)
    torch.cuda.synchronize()
    return out.cpu().numpy(), tq.tq_get_device_error(ctx)


@pytest.mark.parametrize("qmul", [1, 4])
def test_llama8b_window(orc, qmul):
    """One 4096-token sequence compressed by libtq plus a 128-token fp16 window."""
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS["llama8b"].with_(decode_steps=0)
    o = orc.Oracle(128, w.bits, w.param_seed)
    ctx = gpu_ctx(w.bits, w.param_seed, 0, 0)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    kc, vc = gpu_compress(ctx, W.gen_kv(w, 0), W.gen_kv(w, 1), slots, w.num_blocks, w.Hkv)
    tk, tv = _window(w, 77)
    q = (W.gen_q(w).numpy().astype(np.float32) * qmul).astype(np.float16)
    seq, tl = [w.T], [WIN]
    got, err = _run(ctx, q, kc, vc, bt, seq, w.T, tk, tv, tl, w.Hkv)
    assert err == 0
    want = o.decode(q.astype(np.float64), kc.cpu().numpy(), vc.cpu().numpy(), bt, np.array(seq, np.int32), w.Hkv,
                    tail_k=tk.numpy(), tail_v=tv.numpy(), tail_lens=np.array(tl, np.int32))
    check_decode(got, want, "window llama8b 4096+128 q x%d" % qmul)
    # the window matters: without it the oracle is far from the GPU output
    plain = o.decode(q.astype(np.float64), kc.cpu().numpy(), vc.cpu().numpy(), bt, np.array(seq, np.int32), w.Hkv)
    gap = float(np.abs(got - plain).max())
    record("window llama8b q x%d [no-window gap]" % qmul, {"decode_max_abs": gap, "outputs": int(plain.size)})
    assert gap >= 10 * float(np.abs(got - want).max())


def test_batched_window_ragged(orc):
    """32 x 4096 compressed tokens (libtq) with windows of uneven lengths, three
    sequences recomputed by the oracle (q scaled x4: logits spread over several units)."""
    import torch
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS["batched"]
    o = orc.Oracle(128, w.bits, w.param_seed)
    ctx = gpu_ctx(w.bits, w.param_seed, 0, 0)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    kc, vc = gpu_compress(ctx, W.gen_kv(w, 0, device="cuda"), W.gen_kv(w, 1, device="cuda"), slots,
                          w.num_blocks, w.Hkv)
    tk, tv = _window(w, 78)
    rng = np.random.default_rng(5)
    tl = rng.integers(0, WIN + 1, w.B).astype(np.int32)
    tl[0], tl[13] = WIN, 0
    q = (W.gen_q(w).numpy().astype(np.float32) * 4).astype(np.float16)
    seq = np.full(w.B, w.T, np.int32)
    seq[31] = 1000
    got, err = _run(ctx, q, kc, vc, bt, seq, w.T, tk, tv, tl, w.Hkv)
    assert err == 0
    sel = np.array([0, 13, 31])
    want = o.decode(q[sel].astype(np.float64), kc.cpu().numpy(), vc.cpu().numpy(), bt[sel], seq[sel], w.Hkv,
                    tail_k=tk.numpy()[sel], tail_v=tv.numpy()[sel], tail_lens=tl[sel])
    check_decode(got[sel], want, "window batched ragged (3 seqs) q x4")
    del kc, vc
    torch.cuda.empty_cache()


def test_window_only_and_empty_window(orc):
    """seq_lens = 0: exact fp16 attention over the window alone; tail_lens = 0: the
    plain decode."""
    o = orc.Oracle(128, 4, 9)
    rng = np.random.default_rng(2)
    B, Hkv, G, T = 3, 2, 4, 100
    nbps = (T + 15) // 16
    nb = B * nbps
    bt = rng.permutation(nb).reshape(B, nbps).astype(np.int32)
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    for b in range(B):
        t = np.arange(T)
        sl = (bt[b][t // 16] * 16 + t % 16).astype(np.int32)
        o.compress_paged(0, (rng.standard_normal((T, Hkv, 128)) * 2).astype(np.float16), sl, kc)
        o.compress_paged(1, rng.standard_normal((T, Hkv, 128)).astype(np.float16), sl, vc)
    import torch
    tk = torch.as_tensor((rng.standard_normal((B, 40, Hkv, 128)) * 2).astype(np.float16))
    tv = torch.as_tensor(rng.standard_normal((B, 40, Hkv, 128)).astype(np.float16))
    q = (rng.standard_normal((B, G * Hkv, 128)) * 3 / np.sqrt(128)).astype(np.float16)
    ctx = gpu_ctx(4, 9, 0, 0)
    cases = [("window only", [0, 0, 0], [40, 1, 17]), ("empty window", [T, 55, 1], [0, 0, 0]),
             ("both", [T, 0, 33], [40, 7, 0])]
    for label, seq, tl in cases:
        got, err = _run(ctx, q, kc, vc, bt, seq, T, tk, tv, tl, Hkv)
        assert err == 0
        want = o.decode(q.astype(np.float64), kc, vc, bt, np.array(seq, np.int32), Hkv, tail_k=tk.numpy(),
                        tail_v=tv.numpy(), tail_lens=np.array(tl, np.int32))
        check_decode(got, want, "window %s" % label)


def test_window_bad_length_is_flagged(orc):
    from kv_cache_vector_02_b200 import tq
    import torch
    o = orc.Oracle(128, 4, 9)
    kc, vc = o.new_cache(0, 2, 1), o.new_cache(1, 2, 1)
    tk = torch.zeros((1, 8, 1, 128), dtype=torch.float16)
    tv = torch.zeros((1, 8, 1, 128), dtype=torch.float16)
    q = np.zeros((1, 2, 128), np.float16)
    ctx = gpu_ctx(4, 9, 0, 0)
    got, err = _run(ctx, q, kc, vc, np.zeros((1, 2), np.int32), [0], 32, tk, tv, [9], 1)
    assert err == tq.DEVERR_SEQLEN
    assert np.all(got == 0)
