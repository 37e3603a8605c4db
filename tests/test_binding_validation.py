"""The ctypes binding checks that every tensor matches the sizes it passes to the C
ABI (which sees only pointers): a short slot_mapping, a wrong dtype or a cache of
the wrong chunk size is refused on the host, before the library is called."""
import pytest

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_02_b200 import tq as m
    return m


@pytest.fixture()
def ctx(tq):
    return tq.tq_init_host(128, 4, 0, tq.ROT_HAAR, tq.KEY_PROD)


def _compress_args(tq, ctx, T=32, H=2, nb=4):
    k = torch.zeros((T, H, 128), dtype=torch.float16)
    v = torch.zeros((T, H, 128), dtype=torch.float16)
    slots = torch.arange(T, dtype=torch.int32)
    kc = torch.zeros((nb, H, tq.tq_chunk_bytes(ctx, tq.KIND_KEY)), dtype=torch.uint8)
    vc = torch.zeros((nb, H, tq.tq_chunk_bytes(ctx, tq.KIND_VALUE)), dtype=torch.uint8)
    return k, v, slots, kc, vc


@pytest.mark.parametrize("bad", ["short_slots", "slots_int64", "k_fp32", "v_shape", "kc_chunk", "vc_blocks",
                                 "k_noncontig"])
def test_compress_refuses_mismatched_tensors(tq, ctx, bad):
    k, v, slots, kc, vc = _compress_args(tq, ctx)
    if bad == "short_slots":
        slots = slots[:16]
    elif bad == "slots_int64":
        slots = slots.long()
    elif bad == "k_fp32":
        k = k.float()
    elif bad == "v_shape":
        v = v[:, :1]
    elif bad == "kc_chunk":
        kc = kc[:, :, :-16]
    elif bad == "vc_blocks":
        vc = vc[:2]
    elif bad == "k_noncontig":
        k = torch.zeros((2, 128, 32), dtype=torch.float16).permute(2, 0, 1)
    with pytest.raises(tq.TQError) as e:
        tq.tq_compress(ctx, k, v, slots, kc, vc)
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    assert "tq_compress" in str(e.value)


def test_compress_with_matching_tensors_reaches_the_library(tq, ctx):
    # shapes pass the binding; the host-only context is then refused by the library itself
    k, v, slots, kc, vc = _compress_args(tq, ctx)
    with pytest.raises(tq.TQError) as e:
        tq.tq_compress(ctx, k, v, slots, kc, vc, stream=0)
    assert e.value.status == tq.TQ_ERR_INVALID_ARG and "must be" not in str(e.value)


@pytest.mark.parametrize("bad", ["seq_lens", "block_table_rows", "out_shape", "q_dtype", "vc_chunk", "workspace"])
def test_decode_refuses_mismatched_tensors(tq, ctx, bad):
    B, Hq, Hkv, nb = 3, 8, 2, 6
    q = torch.zeros((B, Hq, 128), dtype=torch.float16)
    kc = torch.zeros((nb, Hkv, tq.tq_chunk_bytes(ctx, tq.KIND_KEY)), dtype=torch.uint8)
    vc = torch.zeros((nb, Hkv, tq.tq_chunk_bytes(ctx, tq.KIND_VALUE)), dtype=torch.uint8)
    bt = torch.zeros((B, 2), dtype=torch.int32)
    seq = torch.zeros((B,), dtype=torch.int32)
    out = torch.zeros((B, Hq, 128), dtype=torch.float32)
    ws = torch.zeros((1 << 20,), dtype=torch.uint8)
    if bad == "seq_lens":
        seq = seq[:2]
    elif bad == "block_table_rows":
        bt = bt[:1]
    elif bad == "out_shape":
        out = out[:, :4]
    elif bad == "q_dtype":
        q = q.float()
    elif bad == "vc_chunk":
        vc = vc[:, :, :64]
    elif bad == "workspace":
        ws = ws.view(torch.int32)
    with pytest.raises(tq.TQError) as e:
        tq.tq_decode_attention(ctx, q, kc, vc, bt, seq, 32, out, ws)
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    assert "must be" in str(e.value)
