"""CPU oracle for paged KV-cache decode attention (plain C, fp64) and its ctypes loader.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import this package.  The product path (the CUDA library and
the ``paged_kv_cache_427_b200`` binding) never imports, links or calls it, and it shares no code
with that path.

The C source ``pa_oracle.c`` states what each routine computes and which page and section of
the vLLM tutorials it follows.  This module only compiles it with gcc, loads it and marshals
numpy arrays; it holds no arithmetic of its own.

Element types are named ``"f32"``, ``"bf16"`` and ``"f16"``.  bf16 and f16 arrays are passed as
their raw 16-bit patterns (``numpy.uint16`` or ``numpy.float16``); the C code widens them to
double exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "pa_oracle.c")
LIBRARY = os.path.join(_HERE, "libpa_oracle.so")

DTYPE_CODE = {"f32": 0, "bf16": 1, "f16": 2, "fp8": 3}
ELT_BYTES = {"f32": 4, "bf16": 2, "f16": 2, "fp8": 1}

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int
_D = ctypes.c_double


def build(source: str = SOURCE, output: str = LIBRARY, extra_flags=()) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE double) into a shared library."""
    cmd = [
        "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
        "-ffp-contract=off", *extra_flags, source, "-o", output, "-lm",
    ]
    subprocess.run(cmd, check=True)
    return output


def _stale(lib: str, src: str) -> bool:
    return (not os.path.exists(lib)) or os.path.getmtime(lib) < os.path.getmtime(src)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_P)


def _raw(a: np.ndarray, dtype: str) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.itemsize != ELT_BYTES[dtype]:
        raise TypeError(f"array itemsize {a.itemsize} does not match element type {dtype}")
    return a


class Oracle:
    """ctypes front end of one compiled copy of the oracle library."""

    def __init__(self, path: str = LIBRARY):
        self.path = path
        lib = ctypes.CDLL(path)
        lib.pao_reshape_and_cache.argtypes = [_P, _P, _P, _P, _P, _I64, _I64, _I32, _I32, _I32, _I32]
        lib.pao_reshape_and_cache.restype = _I32
        lib.pao_copy_blocks.argtypes = [_P, _P, _P, _I64, _I64, _I32, _I32, _I32, _I32]
        lib.pao_copy_blocks.restype = _I32
        lib.pao_swap_blocks.argtypes = [_P, _P, _I64, _P, _P, _I64, _P, _I64, _I32, _I32, _I32, _I32]
        lib.pao_swap_blocks.restype = _I32
        lib.pao_decode_range.argtypes = [
            _P, _P, _P, _P, _I32, _P, _P, _I32, _P, _I64, _P, _I64, _I32, _I32, _I32, _I32, _I64,
            _D, _I64, _I64, _I32,
        ]
        lib.pao_decode_range.restype = _I32
        lib.pao_decode_range_scaled.argtypes = lib.pao_decode_range.argtypes + [_P, _P]
        lib.pao_decode_range_scaled.restype = _I32
        lib.pao_prefill.argtypes = [_P, _P, _I32, _P, _P, _I32, _P, _I64, _P, _P, _I64, _I32,
                                    _I32, _I32, _I32, _I64, _D, _I32]
        lib.pao_prefill.restype = _I32
        lib.pao_fp8_encode.argtypes = [_P, _I32, _I64, ctypes.c_float, _P]
        lib.pao_fp8_encode.restype = None
        lib.pao_fp8_decode.argtypes = [_P, _I64, _P]
        lib.pao_fp8_decode.restype = None
        lib.pao_reshape_and_cache_fp8.argtypes = [_P, _P, _I32, _P, _P, _P, _I64, _I64, _I32, _I32,
                                                  _I32, _P, _P]
        lib.pao_reshape_and_cache_fp8.restype = _I32
        lib.pao_lse_combine.argtypes = [_P, _P, _P, _P, _I64, _I32]
        lib.pao_lse_combine.restype = None
        lib.pao_max_threads.argtypes = []
        lib.pao_max_threads.restype = _I32
        self._lib = lib

    def max_threads(self) -> int:
        return int(self._lib.pao_max_threads())

    def reshape_and_cache(self, key, value, key_cache, value_cache, slot_mapping, dtype: str) -> int:
        """Store new tokens' K/V rows in place into the caches.  Returns skipped-token count."""
        nb, hkv, bs, d = key_cache.shape
        for c in (key_cache, value_cache):
            if not c.flags.c_contiguous:
                raise ValueError("caches must be C-contiguous (they are written in place)")
        key = _raw(key, dtype)
        value = _raw(value, dtype)
        slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        return int(self._lib.pao_reshape_and_cache(
            _ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache), _ptr(slots),
            slots.shape[0], nb, hkv, bs, d, DTYPE_CODE[dtype]))

    def copy_blocks(self, key_cache, value_cache, block_mapping, dtype: str) -> int:
        """Copy whole blocks dst <- src in place.  Returns skipped-pair count."""
        nb, hkv, bs, d = key_cache.shape
        bm = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
        return int(self._lib.pao_copy_blocks(
            _ptr(key_cache), _ptr(value_cache), _ptr(bm), bm.shape[0], nb, hkv, bs, d,
            DTYPE_CODE[dtype]))

    def swap_blocks(self, src_key, src_value, dst_key, dst_value, block_mapping, dtype: str) -> int:
        """Move whole blocks dst pool[dst] <- src pool[src].  Returns skipped-pair count."""
        snb, hkv, bs, d = src_key.shape
        dnb = dst_key.shape[0]
        if dst_key.shape[1:] != src_key.shape[1:]:
            raise ValueError("pools differ in block shape")
        bm = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
        return int(self._lib.pao_swap_blocks(
            _ptr(src_key), _ptr(src_value), snb, _ptr(dst_key), _ptr(dst_value), dnb, _ptr(bm),
            bm.shape[0], hkv, bs, d, DTYPE_CODE[dtype]))

    def fp8_encode(self, x, dtype: str, scale: float) -> np.ndarray:
        """FP8 E4M3 codes of x / scale (x of element type dtype, divided in fp32)."""
        raw = _raw(x, dtype)
        out = np.empty(raw.shape, dtype=np.uint8)
        self._lib.pao_fp8_encode(_ptr(raw), DTYPE_CODE[dtype], raw.size, float(scale), _ptr(out))
        return out

    def fp8_decode(self, codes) -> np.ndarray:
        c = np.ascontiguousarray(codes, dtype=np.uint8)
        out = np.empty(c.shape, dtype=np.float64)
        self._lib.pao_fp8_decode(_ptr(c), c.size, _ptr(out))
        return out

    def reshape_and_cache_fp8(self, key, value, dtype: str, key_cache, value_cache, slot_mapping,
                              k_scale, v_scale) -> int:
        """Quantise new tokens' K/V rows (element type dtype) into FP8 caches in place, kv head
        h with k_scale[h] / v_scale[h].  Returns skipped-token count."""
        nb, hkv, bs, d = key_cache.shape
        for c in (key_cache, value_cache):
            if not c.flags.c_contiguous or c.dtype != np.uint8:
                raise ValueError("FP8 caches must be C-contiguous uint8 (written in place)")
        key = _raw(key, dtype)
        value = _raw(value, dtype)
        slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        ks = np.ascontiguousarray(k_scale, dtype=np.float32)
        vs = np.ascontiguousarray(v_scale, dtype=np.float32)
        return int(self._lib.pao_reshape_and_cache_fp8(
            _ptr(key), _ptr(value), DTYPE_CODE[dtype], _ptr(key_cache), _ptr(value_cache),
            _ptr(slots), slots.shape[0], nb, hkv, bs, d, _ptr(ks), _ptr(vs)))

    def decode_range(self, query, key_cache, value_cache, block_tables, context_lens, scale,
                     dtype: str, t_begin: int, t_end: int, q_dtype: str | None = None,
                     num_threads: int = 0, k_scale=None, v_scale=None):
        """Attention restricted to context positions [t_begin, t_end).  With k_scale/v_scale
        ([Hkv] fp32) the keys and values of kv head g are multiplied by them (FP8 caches).

        Returns (out [S,Hq,D] float64, m [S,Hq] float64, l [S,Hq] float64).
        """
        q_dtype = q_dtype or dtype
        nb, hkv, bs, d = key_cache.shape
        s, hq, dq = query.shape
        if dq != d:
            raise ValueError("head_dim mismatch")
        q = _raw(query, q_dtype)
        kc = _raw(key_cache, dtype)
        vc = _raw(value_cache, dtype)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        out = np.empty((s, hq, d), dtype=np.float64)
        m = np.empty((s, hq), dtype=np.float64)
        l = np.empty((s, hq), dtype=np.float64)
        ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
        vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
        rc = self._lib.pao_decode_range_scaled(
            _ptr(out), _ptr(m), _ptr(l), _ptr(q), DTYPE_CODE[q_dtype], _ptr(kc), _ptr(vc),
            DTYPE_CODE[dtype], _ptr(bt), bt.shape[1] if bt.ndim == 2 else 0, _ptr(cl), s, hq, hkv,
            d, bs, nb, float(scale), int(t_begin), int(t_end), int(num_threads),
            None if ks is None else _ptr(ks), None if vs is None else _ptr(vs))
        if rc != 0:
            raise ValueError(f"oracle decode failed with status {rc}")
        return out, m, l

    def decode(self, query, key_cache, value_cache, block_tables, context_lens, scale,
               dtype: str, q_dtype: str | None = None, num_threads: int = 0, k_scale=None,
               v_scale=None) -> np.ndarray:
        """softmax(scale * q K^T) V over each sequence's whole context: [S, Hq, D] float64."""
        out, _, _ = self.decode_range(query, key_cache, value_cache, block_tables, context_lens,
                                      scale, dtype, 0, np.iinfo(np.int64).max, q_dtype,
                                      num_threads, k_scale, v_scale)
        return out

    def prefill(self, query, key_cache, value_cache, block_tables, context_lens, query_start,
                scale, dtype: str, q_dtype: str | None = None, num_threads: int = 0) -> np.ndarray:
        """Causal attention of each sequence's new tokens (query rows query_start[s] ..
        query_start[s+1]-1, the last positions of its context): [total new, Hq, D] float64."""
        q_dtype = q_dtype or dtype
        nb, hkv, bs, d = key_cache.shape
        tq, hq, dq = query.shape
        q = _raw(query, q_dtype)
        kc = _raw(key_cache, dtype)
        vc = _raw(value_cache, dtype)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        qs = np.ascontiguousarray(query_start, dtype=np.int32)
        out = np.zeros((tq, hq, d), dtype=np.float64)
        rc = self._lib.pao_prefill(
            _ptr(out), _ptr(q), DTYPE_CODE[q_dtype], _ptr(kc), _ptr(vc), DTYPE_CODE[dtype], _ptr(bt),
            bt.shape[1] if bt.ndim == 2 else 0, _ptr(cl), _ptr(qs), cl.shape[0], hq, hkv, d, bs,
            nb, float(scale), int(num_threads))
        if rc != 0:
            raise ValueError(f"oracle prefill failed with status {rc}")
        return out

    def lse_combine(self, o_parts, m, l) -> np.ndarray:
        """Merge partial results of one row: o_parts [P, D], m [P], l [P] -> [D] float64."""
        o = np.ascontiguousarray(o_parts, dtype=np.float64)
        mm = np.ascontiguousarray(m, dtype=np.float64)
        ll = np.ascontiguousarray(l, dtype=np.float64)
        out = np.empty(o.shape[1], dtype=np.float64)
        self._lib.pao_lse_combine(_ptr(out), _ptr(o), _ptr(mm), _ptr(ll), o.shape[0], o.shape[1])
        return out


_DEFAULT: Oracle | None = None


def load(path: str | None = None) -> Oracle:
    """Load (building first if missing or older than its source) the oracle library."""
    global _DEFAULT
    if path is not None:
        return Oracle(path)
    if _DEFAULT is None:
        if _stale(LIBRARY, SOURCE):
            build()
        _DEFAULT = Oracle(LIBRARY)
    return _DEFAULT
