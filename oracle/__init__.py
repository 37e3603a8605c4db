"""CPU oracle for the TurboQuant-style KV-cache compressor (TEST INFRASTRUCTURE).

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never loads it; the two share no code.

The arithmetic lives in ``tq_oracle.cpp`` (plain scalar fp64 C++, one loop per
formula, cited there by page and section).  This module compiles it with gcc,
loads it with ctypes and converts numpy arrays in and out: it adds no
arithmetic of its own apart from the exact fp16 -> fp64 widening of inputs.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "tq_oracle.cpp"
_LIB = _HERE / "liboracle.so"

ROT_HAAR, ROT_HADAMARD = 0, 1
KEY_PROD, KEY_MSE = 0, 1
KIND_KEY, KIND_VALUE = 0, 1


def build(force: bool = False) -> Path:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, -O2, OpenMP).

    With ``TQ_ORACLE_LIB`` set in the environment, that library (a copy of the
    oracle compiled elsewhere: the planted-mistake tests' mutants) is loaded
    instead and nothing is compiled."""
    override = os.environ.get("TQ_ORACLE_LIB")
    if override:
        return Path(override)
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(".so.tmp%d" % os.getpid())
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               str(_SRC), "-o", str(tmp)]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(str(build()))
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_long
_U64 = ctypes.c_uint64
_D = ctypes.c_double


def _declare(L):
    sig = {
        "orc_splitmix64": (None, [_U64, _U64, _L, _P]),
        "orc_uniform": (None, [_U64, _U64, _L, _P]),
        "orc_gaussian": (None, [_U64, _U64, _L, _P]),
        "orc_signs": (None, [_U64, _U64, _L, _P]),
        "orc_haar": (None, [_I, _U64, _P]),
        "orc_fwht": (None, [_I, _P]),
        "orc_hadamard_matrix": (None, [_I, _P, _P]),
        "orc_lloyd_max": (None, [_I, _P, _P]),
        "orc_pack": (None, [_P, _I, _I, _P]),
        "orc_unpack": (None, [_P, _I, _I, _P]),
        "orc_create": (_P, [_I, _I, _U64, _I, _I]),
        "orc_create_ex": (_P, [_I, _I, _U64, _I, _I, _I, _I]),
        "orc_lloyd_max_beta": (None, [_I, _I, _P, _P]),
        "orc_destroy": (None, [_P]),
        "orc_get_rotation": (None, [_P, _P]),
        "orc_get_S": (None, [_P, _P]),
        "orc_get_hadamard_signs": (_I, [_P, _P]),
        "orc_get_codebook": (_I, [_P, _I, _P, _P]),
        "orc_chunk_bytes": (_L, [_P, _I]),
        "orc_code_bits": (_I, [_P, _I]),
        "orc_compress_vectors": (None, [_P, _I, _P, _L, _P, _P, _P, _P, _P, _P, _I]),
        "orc_decompress_vectors": (None, [_P, _I, _P, _P, _P, _P, _L, _P, _I]),
        "orc_compress_paged": (_L, [_P, _I, _P, _I, _I, _P, _P, _I, _I]),
        "orc_read_paged": (None, [_P, _I, _P, _I, _I, _P, _P, _P, _P, _P]),
        "orc_decompress_paged": (None, [_P, _I, _P, _I, _I, _P, _P, _I]),
        "orc_decode": (_I, [_P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _D, _I, _P, _I]),
        "orc_decode_window": (_I, [_P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _P, _P, _P, _I, _D, _I, _P, _I]),
        "orc_max_threads": (_I, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(x):
    """fp16/fp32/fp64 -> contiguous fp64 (exact widening)."""
    return np.ascontiguousarray(np.asarray(x), dtype=np.float64)


# ---------------------------------------------------------------- primitives
def splitmix64(seed: int, tag: int, count: int) -> np.ndarray:
    out = np.empty(count, np.uint64)
    lib().orc_splitmix64(seed, tag, count, _ptr(out))
    return out


def uniform(seed: int, tag: int, count: int) -> np.ndarray:
    out = np.empty(count, np.float64)
    lib().orc_uniform(seed, tag, count, _ptr(out))
    return out


def gaussian(seed: int, tag: int, count: int) -> np.ndarray:
    out = np.empty(count, np.float64)
    lib().orc_gaussian(seed, tag, count, _ptr(out))
    return out


def signs(seed: int, tag: int, count: int) -> np.ndarray:
    out = np.empty(count, np.int8)
    lib().orc_signs(seed, tag, count, _ptr(out))
    return out


def haar(d: int, seed: int) -> np.ndarray:
    out = np.empty((d, d), np.float64)
    lib().orc_haar(d, seed, _ptr(out))
    return out


def fwht(x) -> np.ndarray:
    y = _f64(x).copy()
    lib().orc_fwht(y.shape[-1], _ptr(y))
    return y


def hadamard_matrix(D) -> np.ndarray:
    D = np.ascontiguousarray(D, np.int8)
    d = D.shape[0]
    out = np.empty((d, d), np.float64)
    lib().orc_hadamard_matrix(d, _ptr(D), _ptr(out))
    return out


def lloyd_max(bits: int):
    L = 1 << bits
    c = np.empty(L, np.float64)
    t = np.empty(max(L - 1, 1), np.float64)
    lib().orc_lloyd_max(bits, _ptr(c), _ptr(t))
    return c, t[: L - 1]


def lloyd_max_beta(d: int, bits: int):
    """Exact-d Lloyd-Max codebook of v = sqrt(d) u_1, u uniform on the sphere."""
    L = 1 << bits
    c = np.empty(L, np.float64)
    t = np.empty(max(L - 1, 1), np.float64)
    lib().orc_lloyd_max_beta(d, bits, _ptr(c), _ptr(t))
    return c, t[: L - 1]


def pack(codes, width: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.int32)
    n = codes.size
    out = np.empty(n * width // 8, np.uint8)
    lib().orc_pack(_ptr(codes), n, width, _ptr(out))
    return out


def unpack(data, n: int, width: int) -> np.ndarray:
    data = np.ascontiguousarray(data, np.uint8)
    out = np.empty(n, np.int32)
    lib().orc_unpack(_ptr(data), n, width, _ptr(out))
    return out


def max_threads() -> int:
    return lib().orc_max_threads()


# ---------------------------------------------------------------- parameters
class Oracle:
    """Parameters of one compressor instance (R, S, codebooks) and its operations."""

    def __init__(self, d: int = 128, bits: int = 4, seed: int = 0, rot: int = ROT_HAAR,
                 key_mode: int = KEY_PROD, nthreads: int = 0, beta: bool = False, dense3: bool = False):
        self.d, self.bits, self.seed, self.rot, self.key_mode = d, bits, seed, rot, key_mode
        self.beta, self.dense3 = bool(beta), bool(dense3)
        self.nthreads = nthreads
        self._h = lib().orc_create_ex(d, bits, seed, rot, key_mode, int(beta), int(dense3))
        if not self._h:
            raise ValueError("unsupported oracle parameters")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lib is not None:
            _lib.orc_destroy(h)
            self._h = None

    # parameters
    @property
    def R(self) -> np.ndarray:
        out = np.empty((self.d, self.d), np.float64)
        lib().orc_get_rotation(self._h, _ptr(out))
        return out

    @property
    def S(self) -> np.ndarray:
        out = np.empty((self.d, self.d), np.int8)
        lib().orc_get_S(self._h, _ptr(out))
        return out

    @property
    def hadamard_signs(self):
        out = np.empty(self.d, np.int8)
        if lib().orc_get_hadamard_signs(self._h, _ptr(out)) != 0:
            return None
        return out

    def codebook(self, kind: int):
        b = self.code_bits(kind)
        c = np.empty(1 << b, np.float64)
        t = np.empty(max((1 << b) - 1, 1), np.float64)
        lib().orc_get_codebook(self._h, kind, _ptr(c), _ptr(t))
        return c, t[: (1 << b) - 1]

    def code_bits(self, kind: int) -> int:
        return lib().orc_code_bits(self._h, kind)

    def chunk_bytes(self, kind: int) -> int:
        return lib().orc_chunk_bytes(self._h, kind)

    def is_prod(self, kind: int) -> bool:
        return kind == KIND_KEY and self.key_mode == KEY_PROD

    # vectors
    def compress_vectors(self, kind: int, x, diagnostics: bool = False):
        """x [N, d] -> dict(codes [N,d], signs [N,d] or None, norm [N], gamma [N] or None,
        v [N,d] = sqrt(d)*u (diag), sk [N,d] = (S r)/n (diag))."""
        x = _f64(x).reshape(-1, self.d)
        N = x.shape[0]
        codes = np.empty((N, self.d), np.int32)
        prod = self.is_prod(kind)
        sg = np.empty((N, self.d), np.int32) if prod else None
        norms = np.empty(N, np.float64)
        gam = np.empty(N, np.float64) if prod else None
        vd = np.empty((N, self.d), np.float64) if diagnostics else None
        sk = np.empty((N, self.d), np.float64) if (diagnostics and prod) else None
        lib().orc_compress_vectors(self._h, kind, _ptr(x), N, _ptr(codes), _ptr(sg), _ptr(norms), _ptr(gam),
                                   _ptr(vd), _ptr(sk), self.nthreads)
        return {"codes": codes, "signs": sg, "norm": norms, "gamma": gam, "v": vd, "sk": sk}

    def decompress_vectors(self, kind: int, codes, signs, norms, gammas=None) -> np.ndarray:
        codes = np.ascontiguousarray(codes, np.int32).reshape(-1, self.d)
        N = codes.shape[0]
        prod = self.is_prod(kind)
        sg = np.ascontiguousarray(signs, np.int32).reshape(-1, self.d) if prod else None
        norms = _f64(norms).reshape(N)
        gam = _f64(gammas).reshape(N) if prod else None
        out = np.empty((N, self.d), np.float64)
        lib().orc_decompress_vectors(self._h, kind, _ptr(codes), _ptr(sg), _ptr(norms), _ptr(gam), N,
                                     _ptr(out), self.nthreads)
        return out

    # paged cache
    def new_cache(self, kind: int, num_blocks: int, H: int) -> np.ndarray:
        return np.zeros((num_blocks, H, self.chunk_bytes(kind)), np.uint8)

    def compress_paged(self, kind: int, x, slot_mapping, cache: np.ndarray) -> int:
        """x [T, H, d]; writes into cache [num_blocks, H, chunk]; returns #out-of-range slots."""
        x = _f64(x)
        T, H, d = x.shape
        assert d == self.d
        sm = np.ascontiguousarray(slot_mapping, np.int32)
        assert cache.flags.c_contiguous and cache.dtype == np.uint8
        return lib().orc_compress_paged(self._h, kind, _ptr(x), T, H, _ptr(sm), _ptr(cache), cache.shape[0],
                                        self.nthreads)

    def read_paged(self, kind: int, cache, slot_mapping, H: int):
        sm = np.ascontiguousarray(slot_mapping, np.int32)
        cache = np.ascontiguousarray(cache, np.uint8)
        T = sm.shape[0]
        prod = self.is_prod(kind)
        codes = np.empty((T, H, self.d), np.int32)
        sg = np.empty((T, H, self.d), np.int32) if prod else None
        norms = np.empty((T, H), np.float64)
        gam = np.empty((T, H), np.float64) if prod else None
        lib().orc_read_paged(self._h, kind, _ptr(cache), T, H, _ptr(sm), _ptr(codes), _ptr(sg), _ptr(norms),
                             _ptr(gam))
        return {"codes": codes, "signs": sg, "norm": norms, "gamma": gam}

    def decompress_paged(self, kind: int, cache, slot_mapping, H: int) -> np.ndarray:
        sm = np.ascontiguousarray(slot_mapping, np.int32)
        cache = np.ascontiguousarray(cache, np.uint8)
        T = sm.shape[0]
        out = np.empty((T, H, self.d), np.float64)
        lib().orc_decompress_paged(self._h, kind, _ptr(cache), T, H, _ptr(sm), _ptr(out), self.nthreads)
        return out

    def decode(self, q, kcache, vcache, block_table, seq_lens, Hkv: int, scale=None, form: int = 1,
               tail_k=None, tail_v=None, tail_lens=None):
        """Decode attention over the paged cache; with tail_k / tail_v [B, W, Hkv, d]
        and tail_lens [B], the last tail_lens[b] tokens of sequence b are uncompressed
        (the residual window) and join the same softmax."""
        if tail_k is not None:
            return self._decode_window(q, kcache, vcache, block_table, seq_lens, Hkv, scale, form,
                                       tail_k, tail_v, tail_lens)
        q = _f64(q)
        B, Hq, d = q.shape
        assert d == self.d and Hq % Hkv == 0
        kcache = np.ascontiguousarray(kcache, np.uint8)
        vcache = np.ascontiguousarray(vcache, np.uint8)
        bt = np.ascontiguousarray(block_table, np.int32)
        sl = np.ascontiguousarray(seq_lens, np.int32)
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        out = np.empty((B, Hq, d), np.float64)
        rc = lib().orc_decode(self._h, _ptr(q), _ptr(kcache), _ptr(vcache), kcache.shape[0], _ptr(bt),
                              bt.shape[1], _ptr(sl), B, Hq, Hkv, float(scale), form, _ptr(out), self.nthreads)
        if rc != 0:
            raise ValueError("block id or sequence length out of range")
        return out

    def prefill(self, q, kcache, vcache, block_table, q_start: int, Hkv: int, scale=None):
        """Causal prefill attention of one sequence over its paged cache: q [Tq, Hq, d]
        are the queries at positions q_start .. q_start + Tq - 1, whose keys and values
        are already in the cache; query i attends to the tokens 0 .. q_start + i with the
        decode estimator.  It is the decode of Tq sequences that share the block table,
        query i's of length q_start + i + 1."""
        q = _f64(q)
        Tq = q.shape[0]
        bt = np.tile(np.ascontiguousarray(block_table, np.int32).reshape(1, -1), (Tq, 1))
        lens = (q_start + 1 + np.arange(Tq)).astype(np.int32)
        return self.decode(q, kcache, vcache, bt, lens, Hkv, scale)

    def _decode_window(self, q, kcache, vcache, block_table, seq_lens, Hkv, scale, form, tail_k, tail_v, tail_lens):
        q = _f64(q)
        B, Hq, d = q.shape
        assert d == self.d and Hq % Hkv == 0
        tk = _f64(tail_k)
        tv = _f64(tail_v)
        assert tk.shape == tv.shape and tk.shape[0] == B and tk.shape[2] == Hkv and tk.shape[3] == d
        kcache = np.ascontiguousarray(kcache, np.uint8)
        vcache = np.ascontiguousarray(vcache, np.uint8)
        bt = np.ascontiguousarray(block_table, np.int32)
        sl = np.ascontiguousarray(seq_lens, np.int32)
        tl = np.ascontiguousarray(tail_lens, np.int32)
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        out = np.empty((B, Hq, d), np.float64)
        rc = lib().orc_decode_window(self._h, _ptr(q), _ptr(kcache), _ptr(vcache), kcache.shape[0], _ptr(bt),
                                     bt.shape[1], _ptr(sl), B, Hq, Hkv, _ptr(tk), _ptr(tv), _ptr(tl), tk.shape[1],
                                     float(scale), form, _ptr(out), self.nthreads)
        if rc != 0:
            raise ValueError("block id, sequence length or window length out of range")
        return out
