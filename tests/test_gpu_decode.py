"""GPU decode attention and decompress parity against the oracle."""
import math

import numpy as np
import pytest

from parity import DECODE_ATOL, check_decode, gpu_compress, gpu_ctx, record, zero_gamma

pytestmark = pytest.mark.gpu


def _decode_gpu(ctx, q, kc, vc, bt, seq_lens, max_seq_len, Hkv, out_fp32=True, scale=0.0):
    import torch
    from kv_cache_vector_02_b200 import tq
    dev = torch.device("cuda")
    q = torch.as_tensor(q).to(dev)
    B, Hq = q.shape[0], q.shape[1]
    kc = torch.as_tensor(kc).to(dev)
    vc = torch.as_tensor(vc).to(dev)
    bt = torch.as_tensor(np.asarray(bt, np.int32)).to(dev)
    sl = torch.as_tensor(np.asarray(seq_lens, np.int32)).to(dev)
    out = torch.empty((B, Hq, 128), dtype=torch.float32 if out_fp32 else torch.float16, device=dev)
    ws = torch.zeros(tq.tq_decode_workspace_bytes(ctx, B, Hq, Hkv, max_seq_len), dtype=torch.uint8, device=dev)
    tq.tq_decode_attention(ctx, q, kc, vc, bt, sl, max_seq_len, out, ws, scale=scale, Hkv=Hkv)
    torch.cuda.synchronize()
    err = tq.tq_get_device_error(ctx)
    return out.float().cpu().numpy(), err


def _pool_cache(orc, o, w, nb_pool, seed):
    """Oracle-compressed chunks of the workload's law: [nb_pool, Hkv, chunk] per kind."""
    from kv_cache_vector_02_b200 import workloads as W
    wp = w.with_(B=1, T=nb_pool * 16, layers=1, decode_steps=0, data_seed=seed)
    caches = []
    slots = np.arange(nb_pool * 16, dtype=np.int32)
    for kind in (0, 1):
        x = W.gen_kv(wp, kind).numpy()
        c = o.new_cache(kind, nb_pool, w.Hkv)
        o.compress_paged(kind, x, slots, c)
        caches.append(c)
    return caches


@pytest.mark.parametrize("rot,bits,km", [(0, 4, 0), (1, 4, 0), (0, 2, 0), (1, 3, 1)])
def test_tiny_decode_on_oracle_cache(orc, rot, bits, km):
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS["tiny"].with_(rotation=rot, bits=bits, key_mode=km)
    o = orc.Oracle(128, bits, w.param_seed, rot=rot, key_mode=km)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    kc, vc = o.new_cache(0, w.num_blocks, 1), o.new_cache(1, w.num_blocks, 1)
    o.compress_paged(0, W.gen_kv(w, 0).numpy(), slots, kc)
    o.compress_paged(1, W.gen_kv(w, 1).numpy(), slots, vc)
    q = W.gen_q(w).numpy()
    seq = np.array([w.T], np.int32)
    want = o.decode(q.astype(np.float64), kc, vc, bt, seq, w.Hkv)
    ctx = gpu_ctx(bits, w.param_seed, rot, km)
    got, err = _decode_gpu(ctx, q, kc, vc, bt, seq, w.T, w.Hkv)
    assert err == 0
    check_decode(got, want, "decode tiny rot%d b%d km%d" % (rot, bits, km))


@pytest.mark.parametrize("B,T,Hkv,G,maxlen", [(3, 45, 2, 3, 64), (2, 1, 1, 16, 16), (4, 300, 2, 4, 300),
                                               (1, 700, 1, 8, 4096)])
def test_ragged_decode_on_oracle_cache(orc, B, T, Hkv, G, maxlen):
    o = orc.Oracle(128, 4, 9)
    rng = np.random.default_rng(B * 1000 + T)
    nbps = (maxlen + 15) // 16
    nb = B * nbps + 3
    bt = rng.permutation(nb)[: B * nbps].reshape(B, nbps).astype(np.int32)
    seq = rng.integers(max(T // 2, 0), T + 1, size=B).astype(np.int32)
    seq[0] = T
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    for b in range(B):
        t = np.arange(T)
        sl = (bt[b][t // 16] * 16 + t % 16).astype(np.int32)
        o.compress_paged(0, (rng.standard_normal((T, Hkv, 128)) * 2).astype(np.float16), sl, kc)
        o.compress_paged(1, rng.standard_normal((T, Hkv, 128)).astype(np.float16), sl, vc)
    q = (rng.standard_normal((B, G * Hkv, 128)) / math.sqrt(128)).astype(np.float16)
    want = o.decode(q.astype(np.float64), kc, vc, bt, seq, Hkv)
    ctx = gpu_ctx(4, 9, 0, 0)
    got, err = _decode_gpu(ctx, q, kc, vc, bt, seq, maxlen, Hkv)
    assert err == 0
    check_decode(got, want, "decode ragged B%d T%d Hkv%d G%d" % (B, T, Hkv, G))


def test_llama8b_compress_append_decode_end_to_end(orc):
    """Compress the 4096-token context, then 64 steps: append one token (compress)
    and decode over seq_len + 1 tokens; GPU path end to end vs oracle end to end."""
    import torch
    from kv_cache_vector_02_b200 import tq, workloads as W
    w = W.WORKLOADS["llama8b"]
    o = orc.Oracle(128, w.bits, w.param_seed)
    ctx = gpu_ctx(w.bits, w.param_seed, 0, 0)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    k, v = W.gen_kv(w, 0), W.gen_kv(w, 1)
    kc_g, vc_g = gpu_compress(ctx, k, v, slots, w.num_blocks, w.Hkv)
    kc_o, vc_o = o.new_cache(0, w.num_blocks, w.Hkv), o.new_cache(1, w.num_blocks, w.Hkv)
    o.compress_paged(0, k.numpy(), slots, kc_o)
    o.compress_paged(1, v.numpy(), slots, vc_o)
    dev = torch.device("cuda")
    bt_d = torch.as_tensor(bt, device=dev)
    ws = torch.zeros(tq.tq_decode_workspace_bytes(ctx, w.B, w.Hq, w.Hkv, w.max_seq_len), dtype=torch.uint8,
                     device=dev)
    worst = 0.0
    for step in range(w.decode_steps):
        ks, vs = W.gen_step_kv(w, 0, step), W.gen_step_kv(w, 1, step)
        ss = W.step_slots(w, bt, step)
        tq.tq_compress(ctx, ks.to(dev), vs.to(dev), torch.as_tensor(ss, device=dev), kc_g, vc_g)
        o.compress_paged(0, ks.numpy(), ss, kc_o)
        o.compress_paged(1, vs.numpy(), ss, vc_o)
        q = W.gen_q(w, step)
        seq = np.full(w.B, w.T + step + 1, np.int32)
        out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=dev)
        tq.tq_decode_attention(ctx, q.to(dev), kc_g, vc_g, bt_d, torch.as_tensor(seq, device=dev), w.max_seq_len,
                               out, ws)
        if step % 16 == 15 or step == 0:
            want = o.decode(q.numpy().astype(np.float64), kc_o, vc_o, bt, seq, w.Hkv)
            worst = max(worst, float(np.abs(out.cpu().numpy() - want).max()))
    assert tq.tq_get_device_error(ctx) == 0
    record("decode llama8b 64 appended steps (worst)", {"decode_max_abs": worst, "outputs": w.B * w.Hq * 128 * 5})
    assert worst <= DECODE_ATOL, worst


@pytest.mark.parametrize("name,bits,rot,nseq", [("batched", 4, 0, 3), ("long70b", 4, 0, 1), ("long70b", 2, 1, 1)])
def test_full_size_decode(orc, name, bits, rot, nseq):
    """Full-size decode on a cache tiled from oracle-compressed pages; the oracle
    recomputes `nseq` sequences (all their query heads)."""
    import torch
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS[name].with_(bits=bits, rotation=rot)
    o = orc.Oracle(128, bits, w.param_seed, rot=rot)
    pool = _pool_cache(orc, o, w, 512, seed=41)
    rng = np.random.default_rng(43)
    pick = rng.integers(0, 512, size=w.num_blocks)
    kc, vc = pool[0][pick], pool[1][pick]
    bt = W.block_table(w)
    seq = np.full(w.B, w.T, np.int32)
    q = W.gen_q(w).numpy()
    ctx = gpu_ctx(bits, w.param_seed, rot, 0)
    got, err = _decode_gpu(ctx, q, kc, vc, bt, seq, w.T, w.Hkv)
    assert err == 0
    sel = rng.choice(w.B, size=nseq, replace=False)
    want = o.decode(q[sel].astype(np.float64), kc, vc, bt[sel], seq[sel], w.Hkv)
    check_decode(got[sel], want, "decode %s b%d rot%d (%d seqs)" % (name, bits, rot, nseq))
    torch.cuda.empty_cache()


def test_fp16_output_matches_fp32_output(orc):
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS["tiny"]
    o = orc.Oracle(128, 4, 0)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    kc, vc = o.new_cache(0, w.num_blocks, 1), o.new_cache(1, w.num_blocks, 1)
    o.compress_paged(0, W.gen_kv(w, 0).numpy(), slots, kc)
    o.compress_paged(1, W.gen_kv(w, 1).numpy(), slots, vc)
    q = W.gen_q(w).numpy()
    ctx = gpu_ctx(4, 0, 0, 0)
    a, _ = _decode_gpu(ctx, q, kc, vc, bt, [w.T], w.T, 1, out_fp32=True)
    b, _ = _decode_gpu(ctx, q, kc, vc, bt, [w.T], w.T, 1, out_fp32=False)
    assert np.abs(a - b).max() <= np.abs(a).max() * 2 ** -10


@pytest.mark.parametrize("rot,bits,km", [(0, 4, 0), (1, 2, 0), (0, 3, 1)])
def test_decompress_matches_oracle(orc, rot, bits, km):
    import torch
    from kv_cache_vector_02_b200 import tq
    o = orc.Oracle(128, bits, 4, rot=rot, key_mode=km)
    rng = np.random.default_rng(8)
    T, H = 77, 3
    nb = 8
    perm = rng.permutation(nb)
    slots = (perm[np.arange(T) // 16] * 16 + np.arange(T) % 16).astype(np.int32)
    ctx = gpu_ctx(bits, 4, rot, km)
    dev = torch.device("cuda")
    for kind in (0, 1):
        x = (rng.standard_normal((T, H, 128)) * 2).astype(np.float16)
        c = o.new_cache(kind, nb, H)
        o.compress_paged(kind, x, slots, c)
        want = o.decompress_paged(kind, c, slots, H)
        out = torch.empty((T, H, 128), dtype=torch.float32, device=dev)
        tq.tq_decompress(ctx, kind, torch.as_tensor(c, device=dev), torch.as_tensor(slots, device=dev), out)
        got = out.cpu().numpy()
        scale = np.linalg.norm(x.astype(np.float64), axis=-1, keepdims=True)
        assert np.abs(got - want).max() <= 1e-5 * scale.max()


# Every instantiation of the decode kernel: (key code mode, value code mode, QJL or not)
# x (one or two tiles of 8 query heads).  bits 4 / 3 / 2 with prod keys (3-, 2-, 1-bit
# key codes + signs) and with MSE keys (4-, 3-, 2-bit key codes).
DECODE_MODES = [(0, 4, 0), (1, 3, 0), (1, 2, 0), (0, 4, 1), (1, 3, 1), (0, 2, 1)]


@pytest.mark.parametrize("rot,bits,km", DECODE_MODES)
@pytest.mark.parametrize("G", [4, 16])
def test_every_decode_mode(orc, rot, bits, km, G):
    o = orc.Oracle(128, bits, 21, rot=rot, key_mode=km)
    rng = np.random.default_rng(100 * bits + 10 * km + G)
    B, T, Hkv, maxlen = 3, 211, 2, 224
    nbps = (maxlen + 15) // 16
    nb = B * nbps + 2
    bt = rng.permutation(nb)[: B * nbps].reshape(B, nbps).astype(np.int32)
    seq = np.array([T, 17, 160], np.int32)
    kc, vc = o.new_cache(0, nb, Hkv), o.new_cache(1, nb, Hkv)
    for b in range(B):
        t = np.arange(T)
        sl = (bt[b][t // 16] * 16 + t % 16).astype(np.int32)
        o.compress_paged(0, (rng.standard_normal((T, Hkv, 128)) * 2).astype(np.float16), sl, kc)
        o.compress_paged(1, rng.standard_normal((T, Hkv, 128)).astype(np.float16), sl, vc)
    q = (rng.standard_normal((B, G * Hkv, 128)) * 3 / math.sqrt(128)).astype(np.float16)
    want = o.decode(q.astype(np.float64), kc, vc, bt, seq, Hkv)
    ctx = gpu_ctx(bits, 21, rot, km)
    got, err = _decode_gpu(ctx, q, kc, vc, bt, seq, maxlen, Hkv)
    assert err == 0
    check_decode(got, want, "decode mode rot%d b%d km%d G%d" % (rot, bits, km, G))


def _logit_spread(q, k, scale=1 / math.sqrt(128)):
    """Spread (max - min over tokens, smallest over heads) of the exact logits
    q.k * scale: how far the softmax is from uniform."""
    lg = np.einsum("hd,td->ht", q.astype(np.float64), k.astype(np.float64)) * scale
    return float((lg.max(1) - lg.min(1)).min())


def _power_check(o, got, want, kc, vc, bt, seq, Hkv, q, label):
    """The GPU output is within the bar of the oracle, and at least 10x its own error
    away from the oracle without the QJL term (gamma zeroed): a decode that dropped
    or mangled that term could not pass."""
    err = check_decode(got, want, label)
    want0 = o.decode(q.astype(np.float64), zero_gamma(o, kc), vc, bt, seq, Hkv)
    gap = float(np.abs(np.asarray(got, np.float64) - want0).max())
    record(label + " [no-QJL gap]", {"decode_max_abs": gap, "outputs": int(want0.size),
                                     "ratio": gap / max(err, 1e-30)})
    assert gap >= 10 * err, "%s: no-QJL oracle only %.2e away, GPU error %.2e" % (label, gap, err)


@pytest.mark.parametrize("rot", [0, 1])
def test_peaked_tiny_decode_power(orc, rot):
    """Tiny workload with q scaled x8 (logits spread over several units)."""
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS["tiny"].with_(rotation=rot)
    o = orc.Oracle(128, w.bits, w.param_seed, rot=rot)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    k, v = W.gen_kv(w, 0).numpy(), W.gen_kv(w, 1).numpy()
    kc, vc = o.new_cache(0, w.num_blocks, 1), o.new_cache(1, w.num_blocks, 1)
    o.compress_paged(0, k, slots, kc)
    o.compress_paged(1, v, slots, vc)
    q = (W.gen_q(w).numpy().astype(np.float32) * 8).astype(np.float16)
    spread = _logit_spread(q[0], k[:, 0])
    assert spread >= 3.0, spread
    seq = np.array([w.T], np.int32)
    want = o.decode(q.astype(np.float64), kc, vc, bt, seq, 1)
    ctx = gpu_ctx(w.bits, w.param_seed, rot, 0)
    got, err = _decode_gpu(ctx, q, kc, vc, bt, seq, w.T, 1)
    assert err == 0
    _power_check(o, got, want, kc, vc, bt, seq, 1, q, "decode tiny peaked x8 rot%d (spread %.1f)" % (rot, spread))


def test_peaked_batched_decode_power(orc):
    """Batched workload (32 x 4096 tokens, 8 kv / 32 q heads) with q scaled x4, on a
    cache that libtq compressed from the workload's own K and V; the oracle decodes
    three sequences of it."""
    import torch
    from kv_cache_vector_02_b200 import tq, workloads as W
    w = W.WORKLOADS["batched"]
    o = orc.Oracle(128, w.bits, w.param_seed)
    ctx = gpu_ctx(w.bits, w.param_seed, 0, 0)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    k = W.gen_kv(w, 0, device="cuda")
    v = W.gen_kv(w, 1, device="cuda")
    kc, vc = gpu_compress(ctx, k, v, slots, w.num_blocks, w.Hkv)
    q = (W.gen_q(w).numpy().astype(np.float32) * 4).astype(np.float16)
    seq = np.full(w.B, w.T, np.int32)
    got, err = _decode_gpu(ctx, q, kc, vc, bt, seq, w.T, w.Hkv)
    assert err == 0
    sel = np.array([0, 13, 31])
    k0 = k[: w.T, 0].float().cpu().numpy()   # sequence 0, kv head 0
    spread = _logit_spread(q[0, :4], k0)
    assert spread >= 3.0, spread
    kc_h, vc_h = kc.cpu().numpy(), vc.cpu().numpy()
    want = o.decode(q[sel].astype(np.float64), kc_h, vc_h, bt[sel], seq[sel], w.Hkv)
    _power_check(o, got[sel], want, kc_h, vc_h, bt[sel], seq[sel], w.Hkv, q[sel],
                 "decode batched peaked x4 (3 seqs, spread %.1f)" % spread)
    del k, v, kc, vc
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,Hkv,G,window", [(4000, 2, 3, False), (600, 1, 5, True)])
def test_many_short_sequences(orc, B, Hkv, G, window):
    """Thousands of short sequences (0 to 48 tokens): more sequences than the
    shared-memory prefix sums hold (B = 4000), dozens of units and pieces per CTA,
    units split across CTAs, several 16-row batches per CTA in the merge (G = 3, 5),
    empty sequences; the second case adds an fp16 residual window to every unit."""
    import torch
    from kv_cache_vector_02_b200 import tq, workloads as W
    maxlen = 48
    w = W.WORKLOADS["llama8b"].with_(Hkv=Hkv, Hq=G * Hkv)
    o = orc.Oracle(128, 4, w.param_seed)
    pool = _pool_cache(orc, o, w, 64, seed=51)
    rng = np.random.default_rng(B + G)
    nbps = maxlen // 16
    nb = B * nbps
    pick = rng.integers(0, 64, size=nb)
    kc, vc = pool[0][pick], pool[1][pick]
    bt = rng.permutation(nb).reshape(B, nbps).astype(np.int32)
    seq = rng.integers(0, maxlen + 1, size=B).astype(np.int32)
    seq[:3] = 0
    seq[-2:] = 0
    seq[B // 2] = maxlen
    q = (rng.standard_normal((B, G * Hkv, 128)) * 2 / math.sqrt(128)).astype(np.float16)
    ctx = gpu_ctx(4, w.param_seed, 0, 0)
    if not window:
        got, err = _decode_gpu(ctx, q, kc, vc, bt, seq, maxlen, Hkv)
        assert err == 0
        want = o.decode(q.astype(np.float64), kc, vc, bt, seq, Hkv)
    else:
        cap = 20
        tk = (rng.standard_normal((B, cap, Hkv, 128)) * 2).astype(np.float16)
        tv = rng.standard_normal((B, cap, Hkv, 128)).astype(np.float16)
        tl = rng.integers(0, cap + 1, size=B).astype(np.int32)
        dev = torch.device("cuda")
        out = torch.empty((B, G * Hkv, 128), dtype=torch.float32, device=dev)
        ws = torch.full((tq.tq_decode_workspace_bytes(ctx, B, G * Hkv, Hkv, maxlen),), 0xFF, dtype=torch.uint8, device=dev)
        args = [torch.as_tensor(x).to(dev) for x in (q, kc, vc, bt, seq)]
        tq.tq_decode_attention_window(ctx, *args, maxlen, torch.as_tensor(tk).to(dev), torch.as_tensor(tv).to(dev),
                                      torch.as_tensor(tl).to(dev), out, ws, Hkv=Hkv)
        torch.cuda.synchronize()
        err = tq.tq_get_device_error(ctx)
        assert err == 0
        got = out.cpu().numpy()
        want = o.decode(q.astype(np.float64), kc, vc, bt, seq, Hkv, tail_k=tk, tail_v=tv, tail_lens=tl)
    if not window:
        assert np.all(got[seq == 0] == 0)
    # The bar scales with the attended values: the value centroids and P enter the
    # MMA in fp16, so an output made of one or a few tokens carries about 2^-11 of
    # their magnitude per rounding (these sequences have 1 to 48 tokens, and the
    # llama8b law's outlier channels reach |v| ~ 30).
    t = [np.arange(L) for L in seq]
    slots = np.concatenate([bt[b][tt // 16] * 16 + tt % 16 for b, tt in enumerate(t)]).astype(np.int32)
    vals = np.abs(o.decompress_paged(1, vc, slots, Hkv)).max(axis=2)            # [tokens, Hkv]
    vmax = np.zeros((B, Hkv))
    starts = np.concatenate([[0], np.cumsum(seq)])[:-1]
    has = seq > 0
    vmax[has] = np.maximum.reduceat(vals, starts[has], axis=0)
    if window:
        for b in range(B):
            if tl[b] > 0:
                vmax[b] = np.maximum(vmax[b], np.abs(tv[b, :tl[b]].astype(np.float64)).max(axis=(0, 2)))
    bound = DECODE_ATOL + 2.0 ** -10 * np.repeat(vmax, G, axis=1)                # [B, Hq]
    err = np.abs(got - want).max(axis=2)
    label = "decode %d short seqs Hkv%d G%d%s" % (B, Hkv, G, " + window" if window else "")
    record(label, {"decode_max_abs": float(err.max()), "outputs": int(want.size),
                   "max_err_over_bound": float((err / bound).max())})
    assert np.all(err <= bound), (label, float(err.max()), float((err / bound).max()))


def test_partial_pages_ignore_unused_rows(orc):
    """The unused rows of each sequence's last page hold 0xFF bytes (NaN norms, maximal
    codes): the decode reads only the sequence's tokens."""
    o = orc.Oracle(128, 4, 31)
    rng = np.random.default_rng(31)
    B, Hkv, G, maxlen = 5, 2, 4, 100
    nbps = (maxlen + 15) // 16
    nb = B * nbps
    bt = rng.permutation(nb).reshape(B, nbps).astype(np.int32)
    seq = np.array([100, 1, 37, 64, 85], np.int32)
    kc = np.full_like(o.new_cache(0, nb, Hkv), 0xFF)
    vc = np.full_like(o.new_cache(1, nb, Hkv), 0xFF)
    for b in range(B):
        t = np.arange(seq[b])
        sl = (bt[b][t // 16] * 16 + t % 16).astype(np.int32)
        o.compress_paged(0, (rng.standard_normal((seq[b], Hkv, 128)) * 2).astype(np.float16), sl, kc)
        o.compress_paged(1, rng.standard_normal((seq[b], Hkv, 128)).astype(np.float16), sl, vc)
    q = (rng.standard_normal((B, G * Hkv, 128)) / math.sqrt(128)).astype(np.float16)
    ctx = gpu_ctx(4, 31, 0, 0)
    got, err = _decode_gpu(ctx, q, kc, vc, bt, seq, maxlen, Hkv)
    assert err == 0
    assert np.all(np.isfinite(got))
    want = o.decode(q.astype(np.float64), kc, vc, bt, seq, Hkv)
    check_decode(got, want, "decode with 0xFF in unused page rows")
