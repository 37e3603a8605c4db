"""GPU parity of the causal prefill attention (tq_prefill_attention) against the
oracle ([FQ-TQ] "FlashQuant：生产级KV缓存压缩方案…", section "架构设计": the fused
prefill attention kernel; estimator of "注意力计算的特殊挑战与QJL校正").

The bar follows the decode's: 2e-3 max-abs plus, because the first queries of a
chunk attend to a handful of tokens, 2^-10 of the largest attended |v_hat| (the value
levels and the softmax weights enter the MMA in fp16)."""
import math

import numpy as np
import pytest

from parity import DECODE_ATOL, gpu_compress, gpu_ctx, record

pytestmark = pytest.mark.gpu


def _run(ctx, q, kc, vc, bt, q_start, Hkv, out_fp32=True):
    import torch
    from kv_cache_vector_02_b200 import tq
    dev = torch.device("cuda")
    q = torch.as_tensor(q).to(dev)
    out = torch.full((q.shape[0], q.shape[1], 128), float("nan"), dtype=torch.float32 if out_fp32 else torch.float16,
                     device=dev)
    tq.tq_prefill_attention(ctx, q, torch.as_tensor(kc).to(dev), torch.as_tensor(vc).to(dev),
                            torch.as_tensor(np.asarray(bt, np.int32)).to(dev), q_start, out, Hkv=Hkv)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), tq.tq_get_device_error(ctx)


def _check(o, got, want, vc, bt, q_start, Hkv, G, label, rows=None):
    """Per (query, head): |got - want| <= 2e-3 + 2^-10 max|v_hat| over the attended tokens."""
    Tq = want.shape[0]
    rows = np.arange(Tq) if rows is None else rows
    T = q_start + int(rows.max()) + 1
    t = np.arange(T)
    slots = (np.asarray(bt)[t // 16] * 16 + t % 16).astype(np.int32)
    vmax = np.maximum.accumulate(np.abs(o.decompress_paged(1, vc, slots, Hkv)).max(axis=2), axis=0)  # [T, Hkv]
    bound = DECODE_ATOL + 2.0 ** -10 * np.repeat(vmax[q_start + rows], G, axis=1)
    err = np.abs(got - want).max(axis=2)
    record(label, {"decode_max_abs": float(err.max()), "outputs": int(want.size),
                   "max_err_over_bound": float((err / bound).max())})
    assert np.all(err <= bound), (label, float(err.max()), float((err / bound).max()))


def _oracle_cache(orc, o, T, Hkv, rng, law_scale=2.0):
    nbt = (T + 15) // 16
    nb = nbt + 3
    bt = rng.permutation(nb)[:nbt].astype(np.int32)
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    t = np.arange(T)
    sl = (bt[t // 16] * 16 + t % 16).astype(np.int32)
    o.compress_paged(0, (rng.standard_normal((T, Hkv, 128)) * law_scale).astype(np.float16), sl, kc)
    o.compress_paged(1, rng.standard_normal((T, Hkv, 128)).astype(np.float16), sl, vc)
    return kc, vc, bt


@pytest.mark.parametrize("q_start,Tq,Hkv,G,bits,rot,km", [
    (0, 37, 1, 3, 4, 0, 0),      # TQ4 prod, Haar; a ragged query block
    (50, 70, 2, 4, 4, 1, 0),     # Hadamard; chunk starting mid-page, two query blocks
    (16, 20, 2, 2, 2, 0, 0),     # TQ2: 1-bit key codes + signs, 2-bit values
    (3, 64, 1, 8, 3, 0, 1),      # MSE keys (3-bit), 3-bit values
    (100, 130, 2, 1, 4, 1, 1),   # MSE keys (4-bit), one query head per kv head
    (40, 45, 2, 4, 3, 0, 0),     # bits 3 prod: 2-bit key codes + signs, 3-bit values
    (0, 33, 1, 2, 2, 1, 1),      # MSE keys (2-bit), 2-bit values
])
def test_prefill_on_oracle_cache(orc, q_start, Tq, Hkv, G, bits, rot, km):
    rng = np.random.default_rng(q_start * 7 + Tq)
    o = orc.Oracle(128, bits, 21, rot=rot, key_mode=km)
    kc, vc, bt = _oracle_cache(orc, o, q_start + Tq, Hkv, rng)
    q = (rng.standard_normal((Tq, G * Hkv, 128)) / math.sqrt(128)).astype(np.float16)
    ctx = gpu_ctx(bits, 21, rot, km)
    got, err = _run(ctx, q, kc, vc, bt, q_start, Hkv)
    assert err == 0
    want = o.prefill(q.astype(np.float64), kc, vc, bt, q_start, Hkv)
    _check(o, got, want, vc, bt, q_start, Hkv, G, "prefill q%d+%d Hkv%d G%d b%d rot%d km%d" % (
        q_start, Tq, Hkv, G, bits, rot, km))


def test_prefill_llama8b_chunk_sampled(orc):
    """The last 512 tokens of a 4096-token llama8b sequence as one prefill chunk over a
    cache written by libtq; every 17th query (all 32 heads) recomputed by the oracle;
    fp16 output."""
    import torch
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS["llama8b"].with_(decode_steps=0)
    o = orc.Oracle(128, w.bits, w.param_seed)
    ctx = gpu_ctx(w.bits, w.param_seed, 0, 0)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    kc, vc = gpu_compress(ctx, W.gen_kv(w, 0), W.gen_kv(w, 1), slots, w.num_blocks, w.Hkv)
    q_start, Tq = w.T - 512, 512
    rng = np.random.default_rng(8)
    q = (rng.standard_normal((Tq, w.Hq, 128)) * 2 / math.sqrt(128)).astype(np.float16)
    got, err = _run(ctx, q, kc, vc, bt[0], q_start, w.Hkv, out_fp32=False)
    assert err == 0
    rows = np.arange(0, Tq, 17)
    kcn, vcn = kc.cpu().numpy(), vc.cpu().numpy()
    want = o.decode(q[rows].astype(np.float64), kcn, vcn, np.tile(bt[0], (rows.size, 1)),
                    (q_start + rows + 1).astype(np.int32), w.Hkv)
    _check(o, got[rows], want, vcn, bt[0], q_start, w.Hkv, w.Hq // w.Hkv, "prefill llama8b 3584+512 (fp16 out)",
           rows=rows)
    del kc, vc
    torch.cuda.empty_cache()


def test_prefill_last_query_equals_decode(orc):
    """Query i of the chunk and a decode of the sequence cut at position q_start + i
    see the same tokens: the two kernels agree to the decode bar."""
    import torch
    from kv_cache_vector_02_b200 import tq
    o = orc.Oracle(128, 4, 22)
    rng = np.random.default_rng(9)
    q_start, Tq, Hkv, G = 200, 33, 2, 4
    kc, vc, bt = _oracle_cache(orc, o, q_start + Tq, Hkv, rng)
    q = (rng.standard_normal((Tq, G * Hkv, 128)) / math.sqrt(128)).astype(np.float16)
    ctx = gpu_ctx(4, 22, 0, 0)
    got, err = _run(ctx, q, kc, vc, bt, q_start, Hkv)
    assert err == 0
    dev = torch.device("cuda")
    lens = (q_start + 1 + np.arange(Tq)).astype(np.int32)
    out = torch.empty((Tq, G * Hkv, 128), dtype=torch.float32, device=dev)
    ws = torch.empty(tq.tq_decode_workspace_bytes(ctx, Tq, G * Hkv, Hkv, q_start + Tq), dtype=torch.uint8, device=dev)
    tq.tq_decode_attention(ctx, torch.as_tensor(q).to(dev), torch.as_tensor(kc).to(dev), torch.as_tensor(vc).to(dev),
                           torch.as_tensor(np.tile(bt, (Tq, 1))).to(dev), torch.as_tensor(lens).to(dev), q_start + Tq,
                           out, ws, Hkv=Hkv)
    torch.cuda.synchronize()
    assert tq.tq_get_device_error(ctx) == 0
    gap = float(np.abs(out.cpu().numpy() - got).max())
    record("prefill vs decode (same prefixes)", {"decode_max_abs": gap, "outputs": int(got.size)})
    assert gap <= 2 * DECODE_ATOL


def test_prefill_bad_block_and_empty_chunk(orc):
    import torch
    from kv_cache_vector_02_b200 import tq
    o = orc.Oracle(128, 4, 23)
    rng = np.random.default_rng(10)
    kc, vc, bt = _oracle_cache(orc, o, 40, 1, rng)
    ctx = gpu_ctx(4, 23, 0, 0)
    q = (rng.standard_normal((8, 2, 128)) / math.sqrt(128)).astype(np.float16)
    bad = bt.copy()
    bad[1] = 10 ** 6
    got, err = _run(ctx, q, kc, vc, bad, 32, 1)
    assert err & tq.DEVERR_BLOCK
    assert np.all(np.isfinite(got))
    # an empty chunk launches nothing and leaves the output alone
    dev = torch.device("cuda")
    out = torch.full((0, 2, 128), 1.0, device=dev)
    tq.tq_prefill_attention(ctx, torch.zeros((0, 2, 128), dtype=torch.float16, device=dev),
                            torch.as_tensor(kc).to(dev), torch.as_tensor(vc).to(dev),
                            torch.as_tensor(bt).to(dev), 0, out, Hkv=1)
    torch.cuda.synchronize()
    assert tq.tq_get_device_error(ctx) == 0
    # more query heads than grid rows: refused on the host
    qh = torch.zeros((1, 65536, 128), dtype=torch.float16, device=dev)
    with pytest.raises(tq.TQError) as e:
        tq.tq_prefill_attention(ctx, qh, torch.as_tensor(kc).to(dev), torch.as_tensor(vc).to(dev),
                                torch.as_tensor(bt).to(dev), 0, torch.zeros_like(qh), Hkv=1)
    assert e.value.status == tq.TQ_ERR_INVALID_ARG


def test_prefill_ignores_rows_past_the_chunk(orc):
    """The last page's rows past the chunk hold 0xFF bytes (NaN norms): no query reads them."""
    o = orc.Oracle(128, 4, 24)
    rng = np.random.default_rng(11)
    q_start, Tq, Hkv, G = 20, 25, 1, 4   # tokens 0 .. 44: the last page has 13 unused rows
    T = q_start + Tq
    nbt = (T + 15) // 16
    bt = rng.permutation(nbt + 1)[:nbt].astype(np.int32)
    kc = np.full_like(o.new_cache(0, nbt + 1, Hkv), 0xFF)
    vc = np.full_like(o.new_cache(1, nbt + 1, Hkv), 0xFF)
    t = np.arange(T)
    sl = (bt[t // 16] * 16 + t % 16).astype(np.int32)
    o.compress_paged(0, (rng.standard_normal((T, Hkv, 128)) * 2).astype(np.float16), sl, kc)
    o.compress_paged(1, rng.standard_normal((T, Hkv, 128)).astype(np.float16), sl, vc)
    q = (rng.standard_normal((Tq, G * Hkv, 128)) / math.sqrt(128)).astype(np.float16)
    ctx = gpu_ctx(4, 24, 0, 0)
    got, err = _run(ctx, q, kc, vc, bt, q_start, Hkv)
    assert err == 0 and np.all(np.isfinite(got))
    want = o.prefill(q.astype(np.float64), kc, vc, bt, q_start, Hkv)
    _check(o, got, want, vc, bt, q_start, Hkv, G, "prefill with 0xFF past the chunk")
