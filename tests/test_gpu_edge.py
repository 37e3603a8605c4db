"""Edge cases and error reporting of the CUDA path (no fault is provoked: every
invalid index is one the kernels' own checks turn into a skipped item and a
device error bit)."""
import numpy as np
import pytest

from parity import DECODE_ATOL, compare_compress, gpu_compress, gpu_ctx

pytestmark = pytest.mark.gpu


def _t(a, dtype=None):
    import torch
    return torch.as_tensor(np.asarray(a) if dtype is None else np.asarray(a, dtype), device="cuda")


def test_empty_compress_is_noop():
    import torch
    from kv_cache_vector_02_b200 import tq
    ctx = gpu_ctx()
    kc = torch.zeros((1, 1, 1408), dtype=torch.uint8, device="cuda")
    vc = torch.zeros((1, 1, 1088), dtype=torch.uint8, device="cuda")
    x = torch.zeros((0, 1, 128), dtype=torch.float16, device="cuda")
    tq.tq_compress(ctx, x, x, _t(np.zeros(0, np.int32)), kc, vc)
    torch.cuda.synchronize()
    assert kc.sum().item() == 0 and vc.sum().item() == 0


@pytest.mark.parametrize("rot", [0, 1])
def test_zero_vectors(orc, rot):
    import torch
    o = orc.Oracle(128, 4, 2, rot=rot)
    ctx = gpu_ctx(4, 2, rot, 0)
    x = torch.zeros((16, 2, 128), dtype=torch.float16)
    x[3, 1, 5] = 1.0   # one non-zero vector among zeros
    slots = np.arange(16, dtype=np.int32)
    kc, vc = gpu_compress(ctx, x, x, slots, 1, 2)
    for kind, c in ((0, kc), (1, vc)):
        got = o.read_paged(kind, c.cpu().numpy(), slots, 2)
        got = {k: (v.reshape(32, -1) if v is not None and v.ndim == 3 else (v.reshape(-1) if v is not None else None))
               for k, v in got.items()}
        compare_compress(o, kind, x.numpy().reshape(-1, 128), got, "zeros")


def test_negative_slots_skip_and_out_of_range_slots_flag():
    import torch
    from kv_cache_vector_02_b200 import tq
    ctx = gpu_ctx()
    rng = np.random.default_rng(0)
    x = torch.as_tensor(rng.standard_normal((4, 1, 128)).astype(np.float16))
    slots = np.array([0, -1, 1000, 3], np.int32)   # 1000 >= 2 blocks * 16
    kc, vc = gpu_compress(ctx, x, x, slots, 2, 1)
    assert tq.tq_get_device_error(ctx) == tq.DEVERR_SLOT
    assert tq.tq_get_device_error(ctx) == 0          # reading clears it
    # rows 0 and 3 of block 0 written; row 1 (negative slot) untouched; block 1 untouched
    vb = vc.cpu().numpy()
    assert vb[0, 0, 0:64].any() and vb[0, 0, 3 * 64:4 * 64].any()
    assert not vb[0, 0, 64:128].any() and not vb[1].any()


def _small_cache(orc, o, nb, H, T, seed=0):
    rng = np.random.default_rng(seed)
    slots = np.arange(T, dtype=np.int32)
    kc, vc = o.new_cache(0, nb, H), o.new_cache(1, nb, H)
    o.compress_paged(0, rng.standard_normal((T, H, 128)).astype(np.float16), slots, kc)
    o.compress_paged(1, rng.standard_normal((T, H, 128)).astype(np.float16), slots, vc)
    return kc, vc


def _decode(ctx, q, kc, vc, bt, seq, maxlen, H):
    import torch
    from kv_cache_vector_02_b200 import tq
    B, Hq = q.shape[0], q.shape[1]
    out = torch.full((B, Hq, 128), 7.0, dtype=torch.float32, device="cuda")
    ws = torch.zeros(tq.tq_decode_workspace_bytes(ctx, B, Hq, H, maxlen), dtype=torch.uint8, device="cuda")
    tq.tq_decode_attention(ctx, _t(q), _t(kc), _t(vc), _t(bt, np.int32), _t(seq, np.int32), maxlen, out, ws, Hkv=H)
    torch.cuda.synchronize()
    return out.cpu().numpy(), tq.tq_get_device_error(ctx)


def test_decode_zero_length_and_bad_lengths(orc):
    from kv_cache_vector_02_b200 import tq
    o = orc.Oracle(128, 4, 0)
    kc, vc = _small_cache(orc, o, 4, 1, 64)
    ctx = gpu_ctx()
    q = (np.random.default_rng(1).standard_normal((3, 2, 128)) / 11).astype(np.float16)
    bt = np.array([[0, 1, 2, 3]] * 3, np.int32)
    # seq 0 empty, seq 1 valid, seq 2 longer than max_seq_len (64) -> skipped, flagged, zero row
    out, err = _decode(ctx, q, kc, vc, bt, [0, 50, 65], 64, 1)
    assert err == tq.DEVERR_SEQLEN
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    want = o.decode(q[1:2].astype(np.float64), kc, vc, bt[1:2], np.array([50], np.int32), 1)
    assert np.abs(out[1] - want[0]).max() <= DECODE_ATOL


def test_decode_bad_block_id_is_skipped_and_flagged(orc):
    from kv_cache_vector_02_b200 import tq
    o = orc.Oracle(128, 4, 0)
    kc, vc = _small_cache(orc, o, 4, 1, 64)
    ctx = gpu_ctx()
    q = (np.random.default_rng(2).standard_normal((1, 1, 128)) / 11).astype(np.float16)
    out, err = _decode(ctx, q, kc, vc, np.array([[0, 99, 2, 3]], np.int32), [64], 64, 1)
    assert err == tq.DEVERR_BLOCK
    assert np.all(np.isfinite(out))


def test_invalid_arguments_are_rejected():
    import torch
    from kv_cache_vector_02_b200 import tq
    ctx = gpu_ctx()
    q = torch.zeros((1, 3, 128), dtype=torch.float16, device="cuda")
    kc = torch.zeros((1, 2, 1408), dtype=torch.uint8, device="cuda")
    vc = torch.zeros((1, 2, 1088), dtype=torch.uint8, device="cuda")
    bt = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    sl = torch.ones(1, dtype=torch.int32, device="cuda")
    out = torch.empty((1, 3, 128), dtype=torch.float32, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention(ctx, q, kc, vc, bt, sl, 16, out, ws, Hkv=2)   # 3 % 2 != 0
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    q2 = torch.zeros((1, 2, 128), dtype=torch.float16, device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_decode_attention(ctx, q2, kc, vc, bt, sl, 16, out, ws[:8], Hkv=2)  # workspace too small
    with pytest.raises(tq.TQError):
        tq.tq_init(64, 4, 0)


def test_workspace_reuse_is_stable(orc):
    import torch
    from kv_cache_vector_02_b200 import tq
    o = orc.Oracle(128, 4, 0)
    kc, vc = _small_cache(orc, o, 8, 2, 128, seed=3)
    ctx = gpu_ctx()
    q = _t((np.random.default_rng(4).standard_normal((2, 8, 128)) / 11).astype(np.float16))
    bt = _t(np.array([[0, 1, 2, 3, 4, 5, 6, 7], [7, 6, 5, 4, 3, 2, 1, 0]], np.int32))
    sl = _t(np.array([128, 100], np.int32))
    ws = torch.zeros(tq.tq_decode_workspace_bytes(ctx, 2, 8, 2, 128), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        out = torch.empty((2, 8, 128), dtype=torch.float32, device="cuda")
        tq.tq_decode_attention(ctx, q, _t(kc), _t(vc), bt, sl, 128, out, ws, Hkv=2)
        outs.append(out.cpu().numpy())
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[1], outs[2])
