"""Thin ctypes binding of libtq (include/tq.h).

Argument marshalling only: every step of the compress / decode path runs in the
CUDA kernels of libtq.so.  Functions keep the C names; tensors are torch CUDA
tensors (device pointers are taken with ``data_ptr()``), streams default to
torch's current stream.  A non-OK status raises :class:`TQError`.

The library must have been built (``python -m kv_cache_vector_02_b200.build``
or ``__graft_entry__.build()``); importing this module without it raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import numpy as np

_LIB_PATH = Path(__file__).resolve().parent / "libtq.so"

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA, TQ_ERR_OOM, TQ_ERR_DEVICE = range(6)
ROT_HAAR, ROT_HADAMARD = 0, 1
KEY_PROD, KEY_MSE = 0, 1
KIND_KEY, KIND_VALUE = 0, 1
DEVERR_SLOT, DEVERR_BLOCK, DEVERR_SEQLEN, DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8

FLAG_SPHERE_CODEBOOK, FLAG_HOST_ONLY = 0x1, 0x4

EXPORTED = ("tq_init", "tq_init_ex", "tq_init_host", "tq_destroy", "tq_chunk_bytes", "tq_code_bits", "tq_export_params", "tq_compress",
            "tq_decompress", "tq_decode_workspace_bytes", "tq_decode_attention", "tq_decode_attention_window",
            "tq_prefill_attention",
            "tq_decode_attention_noalloc",
            "tq_get_device_error", "tq_debug_stall", "tq_launch_count", "tq_status_string")


class TQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s" % (what, _lib.tq_status_string(status).decode()))


def _load():
    if not _LIB_PATH.exists():
        raise ImportError("libtq.so not built: run `python -m kv_cache_vector_02_b200.build`")
    L = ctypes.CDLL(str(_LIB_PATH))
    P, I, Z, U64, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64, ctypes.c_float
    sig = {
        "tq_init": (I, [I, I, U64, I, I, ctypes.POINTER(P)]),
        "tq_init_host": (I, [I, I, U64, I, I, ctypes.POINTER(P)]),
        "tq_init_ex": (I, [I, I, U64, I, I, I, ctypes.POINTER(P)]),
        "tq_destroy": (I, [P]),
        "tq_chunk_bytes": (Z, [P, I]),
        "tq_code_bits": (I, [P, I]),
        "tq_export_params": (I, [P, P, P, P, P, P, P, P]),
        "tq_compress": (I, [P, P, P, I, I, P, P, P, I, P]),
        "tq_decompress": (I, [P, I, P, I, P, I, I, P, I, P]),
        "tq_decode_workspace_bytes": (Z, [P, I, I, I, I]),
        "tq_decode_attention": (I, [P, P, P, P, I, P, I, P, I, I, I, I, F, P, I, P, Z, P]),
        "tq_decode_attention_window": (I, [P, P, P, P, I, P, I, P, I, I, I, I, P, P, P, I, F, P, I, P, Z, P]),
        "tq_prefill_attention": (I, [P, P, P, P, I, P, I, I, I, I, I, F, P, I, P]),
        "tq_decode_attention_noalloc": (I, [P, P, P, P, I, P, I, P, I, I, I, I, F, P, I, P]),
        "tq_get_device_error": (I, [P, P, ctypes.POINTER(ctypes.c_uint32)]),
        "tq_debug_stall": (I, [P, I]),
        "tq_launch_count": (ctypes.c_uint64, []),
        "tq_status_string": (ctypes.c_char_p, [I]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


_lib = _load()


def library_path() -> str:
    return str(_LIB_PATH)


def _check(status: int, what: str):
    if status != TQ_OK:
        raise TQError(status, what)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Context:
    """Owns one libtq context (tq_init / tq_destroy)."""

    def __init__(self, handle: int, head_dim: int, bits: int, seed: int, rotation: int, key_mode: int):
        self.handle = handle
        self.head_dim, self.bits, self.seed, self.rotation, self.key_mode = head_dim, bits, seed, rotation, key_mode
        self._chunk = {}  # chunk bytes by kind, asked of the library once

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and _lib is not None:
            _lib.tq_destroy(h)
            self.handle = None

    @property
    def _as_parameter_(self):
        return self.handle


def tq_init(head_dim: int = 128, bits: int = 4, seed: int = 0, rotation: int = ROT_HAAR,
            key_mode: int = KEY_PROD) -> Context:
    h = ctypes.c_void_p()
    _check(_lib.tq_init(head_dim, bits, seed, rotation, key_mode, ctypes.byref(h)), "tq_init")
    return Context(h.value, head_dim, bits, seed, rotation, key_mode)


def tq_init_ex(head_dim: int = 128, bits: int = 4, seed: int = 0, rotation: int = ROT_HAAR,
               key_mode: int = KEY_PROD, flags: int = 0) -> Context:
    """tq_init with TQ_FLAG_* options (see tq.h)."""
    h = ctypes.c_void_p()
    _check(_lib.tq_init_ex(head_dim, bits, seed, rotation, key_mode, flags, ctypes.byref(h)), "tq_init_ex")
    return Context(h.value, head_dim, bits, seed, rotation, key_mode)


def tq_init_host(head_dim: int = 128, bits: int = 4, seed: int = 0, rotation: int = ROT_HAAR,
                 key_mode: int = KEY_PROD) -> Context:
    """Host-only context (parameters on the host, no device touched)."""
    h = ctypes.c_void_p()
    _check(_lib.tq_init_host(head_dim, bits, seed, rotation, key_mode, ctypes.byref(h)), "tq_init_host")
    return Context(h.value, head_dim, bits, seed, rotation, key_mode)


def tq_destroy(ctx: Context):
    if ctx.handle:
        _check(_lib.tq_destroy(ctx.handle), "tq_destroy")
        ctx.handle = None


def tq_chunk_bytes(ctx: Context, kind: int) -> int:
    n = ctx._chunk.get(kind)
    if n is None:
        n = ctx._chunk[kind] = int(_lib.tq_chunk_bytes(ctx.handle, kind))
    return n


def tq_code_bits(ctx: Context, kind: int) -> int:
    return int(_lib.tq_code_bits(ctx.handle, kind))


def tq_export_params(ctx: Context) -> dict:
    d = ctx.head_dim
    bv = tq_code_bits(ctx, KIND_VALUE)
    bk = tq_code_bits(ctx, KIND_KEY)
    out = {
        "R": np.empty((d, d), np.float64), "S": np.empty((d, d), np.int8), "hsigns": np.zeros(d, np.int8),
        "cv": np.empty(1 << bv, np.float64), "tv": np.empty((1 << bv) - 1, np.float64),
        "ck": np.empty(1 << bk, np.float64), "tk": np.empty(max((1 << bk) - 1, 1), np.float64),
    }
    p = {k: v.ctypes.data_as(ctypes.c_void_p) for k, v in out.items()}
    _check(_lib.tq_export_params(ctx.handle, p["R"], p["S"], p["hsigns"], p["cv"], p["tv"], p["ck"], p["tk"]),
           "tq_export_params")
    out["tk"] = out["tk"][: (1 << bk) - 1]
    if ctx.rotation != ROT_HADAMARD:
        out["hsigns"] = None
    return out


def _expect(t, shape, dtypes, what: str, name: str):
    """The C ABI takes raw pointers plus sizes: every tensor must hold exactly what
    those sizes promise (shape, dtype, dense row-major), or the call is refused here."""
    ok = t is not None and t.dtype in dtypes and t.is_contiguous()
    if ok:
        got = t.shape
        ok = got == shape if None not in shape else (
            len(got) == len(shape) and all(w is None or g == w for g, w in zip(got, shape)))
    if not ok:
        desc = "None" if t is None else "%s %s" % (tuple(t.shape), t.dtype)
        raise TQError(TQ_ERR_INVALID_ARG, "%s: %s must be %s of %s, got %s" % (what, name, list(shape), dtypes, desc))


def tq_compress(ctx: Context, k, v, slot_mapping, k_cache, v_cache, stream=None):
    """k, v: [T, Hkv, 128] fp16 CUDA tensors (either may be None); slot_mapping [T] int32;
    caches [num_blocks, Hkv, chunk] uint8."""
    import torch
    ref = k if k is not None else v
    if ref is None:
        raise TQError(TQ_ERR_INVALID_ARG, "tq_compress: no input")
    T, Hkv = int(ref.shape[0]), int(ref.shape[1]) if ref.dim() > 1 else 0
    cache = k_cache if k_cache is not None else v_cache
    num_blocks = int(cache.shape[0]) if cache is not None else 0
    for x, c, kind, n in ((k, k_cache, KIND_KEY, "k"), (v, v_cache, KIND_VALUE, "v")):
        if x is None:
            continue
        _expect(x, (T, Hkv, ctx.head_dim), (torch.float16,), "tq_compress", n)
        _expect(c, (num_blocks, Hkv, tq_chunk_bytes(ctx, kind)), (torch.uint8,), "tq_compress", n + "_cache")
    _expect(slot_mapping, (T,), (torch.int32,), "tq_compress", "slot_mapping")
    _check(_lib.tq_compress(ctx.handle, _ptr(k), _ptr(v), T, Hkv, _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache),
                            num_blocks, _stream(stream)), "tq_compress")


def tq_decompress(ctx: Context, kind: int, cache, slot_mapping, out, stream=None):
    """out: [T, Hkv, 128] fp16 or fp32 CUDA tensor; slot_mapping [T] int32; cache [num_blocks, Hkv, chunk]."""
    import torch
    T, Hkv = int(out.shape[0]), int(out.shape[1])
    _expect(out, (T, Hkv, ctx.head_dim), (torch.float16, torch.float32), "tq_decompress", "out")
    _expect(slot_mapping, (T,), (torch.int32,), "tq_decompress", "slot_mapping")
    _expect(cache, (None, Hkv, tq_chunk_bytes(ctx, kind)), (torch.uint8,), "tq_decompress", "cache")
    _check(_lib.tq_decompress(ctx.handle, kind, _ptr(cache), int(cache.shape[0]), _ptr(slot_mapping), T, Hkv,
                              _ptr(out), 1 if out.dtype == torch.float32 else 0, _stream(stream)), "tq_decompress")


def tq_decode_workspace_bytes(ctx: Context, B: int, Hq: int, Hkv: int, max_seq_len: int) -> int:
    n = int(_lib.tq_decode_workspace_bytes(ctx.handle, B, Hq, Hkv, max_seq_len))
    if n == 0:
        raise TQError(TQ_ERR_INVALID_ARG, "tq_decode_workspace_bytes")
    return n


def tq_decode_attention(ctx: Context, q, k_cache, v_cache, block_table, seq_lens, max_seq_len: int, out,
                        workspace, scale: float = 0.0, Hkv: int | None = None, stream=None):
    """q: [B, Hq, 128] fp16; caches [num_blocks, Hkv, chunk] uint8; block_table [B, max_blocks] int32;
    seq_lens [B] int32; out [B, Hq, 128] fp16 or fp32; workspace uint8 tensor (any contents)."""
    import torch
    B, Hq = int(q.shape[0]), int(q.shape[1])
    if Hkv is None:
        Hkv = int(k_cache.shape[1])
    _check_decode_args(ctx, q, k_cache, v_cache, block_table, seq_lens, out, Hkv, "tq_decode_attention")
    _expect(workspace, (None,), (torch.uint8,), "tq_decode_attention", "workspace")
    _check(_lib.tq_decode_attention(ctx.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache), int(k_cache.shape[0]),
                                    _ptr(block_table), int(block_table.shape[1]), _ptr(seq_lens), B, Hq, Hkv,
                                    int(max_seq_len), float(scale), _ptr(out), 1 if out.dtype == torch.float32 else 0,
                                    _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                                    _stream(stream)), "tq_decode_attention")


def tq_decode_attention_window(ctx: Context, q, k_cache, v_cache, block_table, seq_lens, max_seq_len: int,
                               tail_k, tail_v, tail_lens, out, workspace, scale: float = 0.0,
                               Hkv: int | None = None, stream=None):
    """tq_decode_attention plus an fp16 residual window: tail_k, tail_v [B, W, Hkv, 128]
    fp16 (W <= 256), tail_lens [B] int32 (see tq.h)."""
    import torch
    B, Hq = int(q.shape[0]), int(q.shape[1])
    if Hkv is None:
        Hkv = int(k_cache.shape[1])
    what = "tq_decode_attention_window"
    _check_decode_args(ctx, q, k_cache, v_cache, block_table, seq_lens, out, Hkv, what)
    _expect(workspace, (None,), (torch.uint8,), what, "workspace")
    W = int(tail_k.shape[1]) if tail_k is not None and tail_k.dim() == 4 else 0
    _expect(tail_k, (B, W, Hkv, ctx.head_dim), (torch.float16,), what, "tail_k")
    _expect(tail_v, (B, W, Hkv, ctx.head_dim), (torch.float16,), what, "tail_v")
    _expect(tail_lens, (B,), (torch.int32,), what, "tail_lens")
    _check(_lib.tq_decode_attention_window(ctx.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache), int(k_cache.shape[0]),
                                           _ptr(block_table), int(block_table.shape[1]), _ptr(seq_lens), B, Hq, Hkv,
                                           int(max_seq_len), _ptr(tail_k), _ptr(tail_v), _ptr(tail_lens), W,
                                           float(scale), _ptr(out), 1 if out.dtype == torch.float32 else 0,
                                           _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                                           _stream(stream)), what)


def tq_prefill_attention(ctx: Context, q, k_cache, v_cache, block_table, q_start: int, out, scale: float = 0.0,
                         Hkv: int | None = None, stream=None):
    """Causal prefill attention of one sequence: q [Tq, Hq, 128] fp16 at positions
    q_start .. q_start + Tq - 1, block_table [max_blocks] int32, out [Tq, Hq, 128]
    fp16 or fp32 (see tq.h)."""
    import torch
    Tq, Hq = int(q.shape[0]), int(q.shape[1])
    if Hkv is None:
        Hkv = int(k_cache.shape[1])
    what = "tq_prefill_attention"
    _expect(q, (Tq, Hq, ctx.head_dim), (torch.float16,), what, "q")
    _expect(k_cache, (None, Hkv, tq_chunk_bytes(ctx, KIND_KEY)), (torch.uint8,), what, "k_cache")
    _expect(v_cache, (int(k_cache.shape[0]), Hkv, tq_chunk_bytes(ctx, KIND_VALUE)), (torch.uint8,), what, "v_cache")
    _expect(block_table, (None,), (torch.int32,), what, "block_table")
    _expect(out, (Tq, Hq, ctx.head_dim), (torch.float16, torch.float32), what, "out")
    _check(_lib.tq_prefill_attention(ctx.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache), int(k_cache.shape[0]),
                                     _ptr(block_table), int(block_table.shape[0]), int(q_start), Tq, Hq, Hkv,
                                     float(scale), _ptr(out), 1 if out.dtype == torch.float32 else 0,
                                     _stream(stream)), what)


NOALLOC_SCRATCH_BYTES = 8 << 20


def _check_decode_args(ctx, q, k_cache, v_cache, block_table, seq_lens, out, Hkv, what):
    import torch
    B, Hq = int(q.shape[0]), int(q.shape[1])
    _expect(q, (B, Hq, ctx.head_dim), (torch.float16,), what, "q")
    _expect(k_cache, (None, Hkv, tq_chunk_bytes(ctx, KIND_KEY)), (torch.uint8,), what, "k_cache")
    _expect(v_cache, (int(k_cache.shape[0]), Hkv, tq_chunk_bytes(ctx, KIND_VALUE)), (torch.uint8,), what, "v_cache")
    _expect(block_table, (B, None), (torch.int32,), what, "block_table")
    _expect(seq_lens, (B,), (torch.int32,), what, "seq_lens")
    _expect(out, (B, Hq, ctx.head_dim), (torch.float16, torch.float32), what, "out")


def tq_decode_attention_noalloc(ctx: Context, q, k_cache, v_cache, block_table, seq_lens, max_seq_len: int, out,
                                scale: float = 0.0, Hkv: int | None = None, stream=None):
    """tq_decode_attention with the library's own per-device scratch instead of a
    workspace argument, for callers that cannot allocate device memory (see tq.h).
    Calls that overlap on the GPU race on that scratch."""
    import torch
    B, Hq = int(q.shape[0]), int(q.shape[1])
    if Hkv is None:
        Hkv = int(k_cache.shape[1])
    _check_decode_args(ctx, q, k_cache, v_cache, block_table, seq_lens, out, Hkv, "tq_decode_attention_noalloc")
    _check(_lib.tq_decode_attention_noalloc(ctx.handle, _ptr(q), _ptr(k_cache), _ptr(v_cache), int(k_cache.shape[0]),
                                            _ptr(block_table), int(block_table.shape[1]), _ptr(seq_lens), B, Hq, Hkv,
                                            int(max_seq_len), float(scale), _ptr(out),
                                            1 if out.dtype == torch.float32 else 0, _stream(stream)),
           "tq_decode_attention_noalloc")


def tq_get_device_error(ctx: Context, stream=None) -> int:
    code = ctypes.c_uint32(0)
    st = _lib.tq_get_device_error(ctx.handle, _stream(stream), ctypes.byref(code))
    if st not in (TQ_OK, TQ_ERR_DEVICE):
        raise TQError(st, "tq_get_device_error")
    return int(code.value)


def tq_debug_stall(ctx: Context, launches: int):
    """Test hook: the next `launches` kernels of ctx withhold what their bounded
    waits expect (compress: its input copies; decode: the partial results another
    CTA merges), so the waits run out and TQ_DEVERR_TIMEOUT is set (see tq.h)."""
    _check(_lib.tq_debug_stall(ctx.handle, int(launches)), "tq_debug_stall")


def tq_launch_count() -> int:
    return int(_lib.tq_launch_count())


def tq_status_string(status: int) -> str:
    return _lib.tq_status_string(status).decode()
