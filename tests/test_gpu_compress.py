"""GPU compress parity against the oracle (element by element on small cases,
sampled vectors on the full-size workloads)."""
import numpy as np
import pytest

from parity import compare_compress, gpu_compress, gpu_ctx

pytestmark = pytest.mark.gpu

# (rot, bits, key_mode): every (rotation, code width) pair of the compress kernels, both key modes
SETTINGS = [(0, 4, 0), (1, 4, 0), (0, 2, 0), (1, 3, 0), (0, 3, 0), (0, 3, 1), (1, 2, 1)]


def _read(orc_obj, kind, cache, slots, H):
    return orc_obj.read_paged(kind, cache.cpu().numpy(), slots, H)


def _check_all(orc, o, ctx, k, v, slots, num_blocks, H, label):
    kc, vc = gpu_compress(ctx, k, v, slots, num_blocks, H)
    out = {}
    for kind, x, c in ((0, k, kc), (1, v, vc)):
        got = _read(o, kind, c, slots, H)
        xs = x.cpu().numpy().reshape(-1, 128)
        out[kind] = compare_compress(o, kind, xs, {kk: (vv.reshape(xs.shape[0], -1) if vv is not None and vv.ndim == 3
                                                         else (vv.reshape(-1) if vv is not None else None))
                                                    for kk, vv in got.items()}, label="%s kind %d" % (label, kind))
    return out


@pytest.mark.parametrize("rot,bits,km", SETTINGS)
def test_tiny_workload_full(orc, rot, bits, km):
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS["tiny"].with_(rotation=rot, bits=bits, key_mode=km)
    k, v = W.gen_kv(w, 0), W.gen_kv(w, 1)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    o = orc.Oracle(128, bits, w.param_seed, rot=rot, key_mode=km, nthreads=0)
    ctx = gpu_ctx(bits, w.param_seed, rot, km)
    _check_all(orc, o, ctx, k, v, slots, w.num_blocks, w.Hkv, "tiny rot%d b%d km%d" % (rot, bits, km))


@pytest.mark.parametrize("rot,bits,km", SETTINGS[:3])
# rows T * H: below one 128-row block, exactly one, one and a half (the odd CTA of a
# 2-CTA cluster partly filled), and several 256-row cluster tiles with a ragged tail
@pytest.mark.parametrize("T,H", [(37, 3), (16, 8), (1, 1), (25, 8), (300, 5)])
def test_ragged_shapes(orc, rot, bits, km, T, H):
    import torch
    rng = np.random.default_rng(T * 31 + H)
    k = torch.as_tensor((rng.standard_normal((T, H, 128)) * 3).astype(np.float16))
    v = torch.as_tensor(rng.standard_normal((T, H, 128)).astype(np.float16))
    nb = (T + 15) // 16 + 2
    perm = rng.permutation(nb)
    slots = (perm[np.arange(T) // 16] * 16 + np.arange(T) % 16).astype(np.int32)
    o = orc.Oracle(128, bits, 3, rot=rot, key_mode=km)
    ctx = gpu_ctx(bits, 3, rot, km)
    _check_all(orc, o, ctx, k, v, slots, nb, H, "ragged T=%d H=%d rot%d b%d km%d" % (T, H, rot, bits, km))


@pytest.mark.parametrize("rot", [0, 1])
def test_llama8b_prefill_full(orc, rot):
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS["llama8b"].with_(rotation=rot)
    k, v = W.gen_kv(w, 0), W.gen_kv(w, 1)
    bt = W.block_table(w)
    slots = W.prefill_slots(w, bt)
    o = orc.Oracle(128, 4, w.param_seed, rot=rot)
    ctx = gpu_ctx(4, w.param_seed, rot, 0)
    _check_all(orc, o, ctx, k, v, slots, w.num_blocks, w.Hkv, "llama8b rot%d" % rot)


def _sampled(orc, w, n_sample, seed):
    """Compress the whole workload on the GPU, compare a seeded sample of tokens."""
    import torch
    from kv_cache_vector_02_b200 import workloads as W
    ctx = gpu_ctx(w.bits, w.param_seed, w.rotation, w.key_mode)
    o = orc.Oracle(128, w.bits, w.param_seed, rot=w.rotation, key_mode=w.key_mode)
    if w.layers > 1:
        slots = W.flat_slots(w.tokens, perm_seed=w.data_seed)
        nb = (w.tokens + 15) // 16
    else:
        bt = W.block_table(w)
        slots = W.prefill_slots(w, bt)
        nb = w.num_blocks
    k = W.gen_kv(w, 0, device="cuda")
    v = W.gen_kv(w, 1, device="cuda")
    kc, vc = gpu_compress(ctx, k, v, slots, nb, w.Hkv)
    rng = np.random.default_rng(seed)
    tok = np.sort(rng.choice(w.tokens, size=n_sample, replace=False))
    tok_t = torch.as_tensor(tok, device="cuda")
    res = {}
    for kind, x, c in ((0, k, kc), (1, v, vc)):
        xs = x.index_select(0, tok_t).cpu().numpy().reshape(-1, 128)
        # rows of the sampled tokens only
        blocks = torch.as_tensor(slots[tok] // 16, device="cuda", dtype=torch.long)
        sub = c.index_select(0, blocks).cpu().numpy()
        sub_slots = (np.arange(n_sample) * 16 + slots[tok] % 16).astype(np.int32)
        got = o.read_paged(kind, sub, sub_slots, w.Hkv)
        got = {kk: (vv.reshape(xs.shape[0], -1) if vv is not None and vv.ndim == 3 else
                    (vv.reshape(-1) if vv is not None else None)) for kk, vv in got.items()}
        res[kind] = compare_compress(o, kind, xs, got, label="%s rot%d b%d km%d kind %d (sampled)"
                                     % (w.name, w.rotation, w.bits, w.key_mode, kind))
    del k, v, kc, vc
    torch.cuda.empty_cache()
    return res


@pytest.mark.parametrize("rot", [0, 1])
def test_batched_prefill_sampled(orc, rot):
    from kv_cache_vector_02_b200 import workloads as W
    _sampled(orc, W.WORKLOADS["batched"].with_(rotation=rot), 2048, 5)


@pytest.mark.parametrize("rot,bits", [(0, 4), (1, 4), (0, 2), (1, 2)])
def test_long70b_prefill_sampled(orc, rot, bits):
    from kv_cache_vector_02_b200 import workloads as W
    _sampled(orc, W.WORKLOADS["long70b"].with_(rotation=rot, bits=bits), 1024, 6)


@pytest.mark.parametrize("rot,bits", [(0, 4), (1, 3), (0, 3), (0, 2)])
def test_prefill80_sampled(orc, rot, bits):
    from kv_cache_vector_02_b200 import workloads as W
    _sampled(orc, W.WORKLOADS["prefill80"].with_(rotation=rot, bits=bits), 1024, 7)
