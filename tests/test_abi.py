"""The C ABI library: builds, loads without a GPU, exports every declared
symbol, and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_02_b200 import build
    build.build()
    from kv_cache_vector_02_b200 import tq as mod
    return mod


def _declared():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            names += re.findall(r"^TQ_API\s+[\w\s\*]+?\b(tq_\w+)\s*\(", src, re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(tq):
    declared = _declared()
    assert len(declared) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", tq.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT\s+(tq_\w+)$", out, re.M))
    assert set(declared) <= exported, set(declared) - exported
    assert set(tq.EXPORTED) == set(declared)
    lib = ctypes.CDLL(tq.library_path())
    for n in declared:
        assert getattr(lib, n) is not None


def test_status_strings(tq):
    assert tq.tq_status_string(0) == "TQ_OK"
    assert tq.tq_status_string(5) == "TQ_ERR_DEVICE"
    assert tq.tq_status_string(99) == "TQ_ERR_UNKNOWN"


def test_host_validation_before_any_device_call(tq):
    L = tq._lib
    h = ctypes.c_void_p()
    assert L.tq_init(64, 4, 0, 0, 0, ctypes.byref(h)) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_init(128, 5, 0, 0, 0, ctypes.byref(h)) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_init(128, 1, 0, 0, 0, ctypes.byref(h)) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_init(128, 4, 0, 7, 0, ctypes.byref(h)) == tq.TQ_ERR_UNSUPPORTED
    assert L.tq_init(128, 4, 0, 0, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert L.tq_chunk_bytes(None, 0) == 0
    assert L.tq_code_bits(None, 0) == -1
    assert L.tq_destroy(None) == tq.TQ_OK


def test_host_only_context_refuses_device_work(tq):
    ctx = tq.tq_init_host(128, 4, 0)
    assert tq.tq_chunk_bytes(ctx, tq.KIND_VALUE) == 16 * 68
    assert tq.tq_chunk_bytes(ctx, tq.KIND_KEY) == 16 * 88
    L = tq._lib
    st = L.tq_compress(ctx.handle, 16, 16, 1, 1, 16, 16, 16, 1, None)
    assert st == tq.TQ_ERR_INVALID_ARG
    assert L.tq_decode_workspace_bytes(ctx.handle, 1, 1, 1, 16) == 0
    code = ctypes.c_uint32()
    assert L.tq_get_device_error(ctx.handle, None, ctypes.byref(code)) == tq.TQ_ERR_INVALID_ARG
    tq.tq_destroy(ctx)


@pytest.mark.parametrize("bits,km,ck,cv", [(4, 0, 1408, 1088), (3, 0, 896, 1088), (2, 0, 640, 576),
                                          (4, 1, 1088, 1088), (2, 1, 576, 576)])
def test_chunk_bytes(tq, bits, km, ck, cv):
    ctx = tq.tq_init_host(128, bits, 0, 0, km)
    assert tq.tq_chunk_bytes(ctx, tq.KIND_KEY) == ck and tq.tq_chunk_bytes(ctx, tq.KIND_VALUE) == cv


def test_noalloc_size_constant_matches_header(tq):
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    m = re.search(r"#define\s+TQ_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", src)
    assert m, "TQ_NOALLOC_SCRATCH_BYTES not found in tq.h"
    assert int(m.group(1)) << int(m.group(2)) == tq.NOALLOC_SCRATCH_BYTES


def test_noalloc_raw_call_refuses_bad_arguments(tq):
    """The allocation-free entry point through the raw symbol: a null or host-only
    context is refused on the host before any device is touched."""
    L = tq._lib
    f = L.tq_decode_attention_noalloc
    args = (16, 16, 16, 1, 16, 1, 16, 1, 1, 1, 16, 0.0, 16, 1, None)
    assert f(None, *args) == tq.TQ_ERR_INVALID_ARG
    ctx = tq.tq_init_host(128, 4, 0)
    assert f(ctx.handle, *args) == tq.TQ_ERR_INVALID_ARG
    tq.tq_destroy(ctx)


def test_prefill_raw_call_refuses_bad_arguments(tq):
    """tq_prefill_attention through the raw symbol: a null or host-only context, and a
    chunk that reaches past the block table, are refused on the host before any device
    is touched; an empty chunk is a no-op."""
    L = tq._lib
    f = L.tq_prefill_attention
    # (q, k_cache, v_cache, num_blocks, block_table, max_blocks, q_start, Tq, Hq, Hkv, scale, out, out_fp32, stream)
    good = (16, 16, 16, 4, 16, 4, 0, 16, 2, 1, 0.0, 16, 1, None)
    assert f(None, *good) == tq.TQ_ERR_INVALID_ARG
    ctx = tq.tq_init_host(128, 4, 0)
    assert f(ctx.handle, *good) == tq.TQ_ERR_INVALID_ARG
    tq.tq_destroy(ctx)
