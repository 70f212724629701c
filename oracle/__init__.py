"""fp64 CPU oracle for the paged KV-cache decode path (ctypes wrapper).

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package. The product path never
does; it shares no code with the CUDA library.

The arithmetic lives in ``pa_oracle.c`` (plain C, fp64). This module compiles
it with gcc on first use (or when the source is newer than the library) and
marshals numpy arrays. Element arrays are passed as raw 16-bit patterns
(``numpy.uint16``) plus a dtype code, so fp16 and bf16 share one path.

Every function cites the passage it follows in ``pa_oracle.c``'s header. All
pins are in ``tests/test_oracle_pins.py`` and ``tests/test_oracle_mutants.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "pa_oracle.c")
LIBRARY = os.path.join(HERE, "liboracle.so")

F16 = 0
BF16 = 1
KV_FORMATS = {"e4m3": 0, "int8": 1}   # 8-bit cache formats of the *_kv8 functions
_DTYPE_CODES = {"f16": F16, "fp16": F16, "float16": F16, "bf16": BF16, "bfloat16": BF16}


def build(source: str = SOURCE, library: str = LIBRARY, force: bool = False) -> str:
    """Compile the oracle C source into a shared library (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(library)
            and os.path.getmtime(library) >= os.path.getmtime(source)):
        return library
    tmp = library + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
           "-std=c99", source, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, library)
    return library


def dtype_code(dtype) -> int:
    if isinstance(dtype, int):
        return dtype
    return _DTYPE_CODES[str(dtype).replace("torch.", "")]


_P = ctypes.c_void_p
_I = ctypes.c_int


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """Handle on one compiled oracle library (the default one, or a test copy)."""

    def __init__(self, library: str):
        self.lib = ctypes.CDLL(library)
        L = self.lib
        L.oracle_to_double.restype = ctypes.c_double
        L.oracle_to_double.argtypes = [ctypes.c_uint16, _I]
        L.oracle_max_threads.restype = _I
        L.oracle_max_threads.argtypes = []
        L.oracle_paged_attention.restype = None
        L.oracle_paged_attention.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                             ctypes.c_double, _I, _I]
        L.oracle_reshape_and_cache.restype = None
        L.oracle_reshape_and_cache.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I]
        L.oracle_copy_blocks.restype = None
        L.oracle_copy_blocks.argtypes = [_P, _I, _P, _I, ctypes.c_size_t]
        L.oracle_swap_blocks.restype = None
        L.oracle_swap_blocks.argtypes = [_P, _P, _I, _P, _I, ctypes.c_size_t]
        L.oracle_e4m3_to_double.restype = ctypes.c_double
        L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_paged_attention_fp8.restype = None
        L.oracle_paged_attention_fp8.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                                 ctypes.c_double, _I, ctypes.c_double, ctypes.c_double, _I]
        L.oracle_reshape_and_cache_fp8.restype = None
        L.oracle_reshape_and_cache_fp8.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I,
                                                   ctypes.c_float, ctypes.c_float]
        L.oracle_int8_to_double.restype = ctypes.c_double
        L.oracle_int8_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_int8_encode.restype = ctypes.c_uint8
        L.oracle_int8_encode.argtypes = [ctypes.c_float]
        L.oracle_paged_attention_kv8.restype = None
        L.oracle_paged_attention_kv8.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                                 ctypes.c_double, _I, _I, _P, _P, _I]
        L.oracle_reshape_and_cache_kv8.restype = None
        L.oracle_reshape_and_cache_kv8.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]
        L.oracle_paged_attention_kv8_blocks.restype = None
        L.oracle_paged_attention_kv8_blocks.argtypes = L.oracle_paged_attention_kv8.argtypes
        L.oracle_reshape_and_cache_kv8_blocks.restype = None
        L.oracle_reshape_and_cache_kv8_blocks.argtypes = L.oracle_reshape_and_cache_kv8.argtypes
        L.oracle_slot_mapping.restype = None
        L.oracle_slot_mapping.argtypes = [_P, _P, _I, _P, _P, _I, _I]

    # -- element decoding -------------------------------------------------
    def to_double(self, bits, dtype) -> np.ndarray:
        code = dtype_code(dtype)
        flat = np.ascontiguousarray(bits, dtype=np.uint16).ravel()
        f = self.lib.oracle_to_double
        return np.array([f(int(b), code) for b in flat], dtype=np.float64).reshape(np.shape(bits))

    def e4m3_to_double(self, codes) -> np.ndarray:
        flat = np.ascontiguousarray(codes, dtype=np.uint8).ravel()
        f = self.lib.oracle_e4m3_to_double
        return np.array([f(int(c)) for c in flat], dtype=np.float64).reshape(np.shape(codes))

    def e4m3_encode(self, values) -> np.ndarray:
        flat = np.ascontiguousarray(values, dtype=np.float32).ravel()
        f = self.lib.oracle_e4m3_encode
        return np.array([f(float(v)) for v in flat], dtype=np.uint8).reshape(np.shape(values))

    def paged_attention_fp8(self, q, k_pool, v_pool, block_tables, context_lens, scale, q_dtype,
                            k_scale, v_scale, num_threads: int = 0) -> np.ndarray:
        """out[s][h][:] in fp64 over E4M3 pools (uint8 codes) with per-tensor scales."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        k_pool = np.ascontiguousarray(k_pool, dtype=np.uint8)
        v_pool = np.ascontiguousarray(v_pool, dtype=np.uint8)
        block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        B, H, D = q.shape
        NB, Hkv, bs, D2 = k_pool.shape
        assert D2 == D and v_pool.shape == k_pool.shape and H % Hkv == 0
        for s in range(B):
            n = int(context_lens[s])
            pages = -(-n // bs)
            assert 0 <= n and pages <= block_tables.shape[1]
            if pages:
                used = block_tables[s, :pages]
                assert used.min() >= 0 and used.max() < NB
        out = np.zeros((B, H, D), dtype=np.float64)
        self.lib.oracle_paged_attention_fp8(
            _ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), _ptr(context_lens),
            B, H, Hkv, D, bs, block_tables.shape[1], float(scale), dtype_code(q_dtype), float(k_scale),
            float(v_scale), int(num_threads))
        return out

    def reshape_and_cache_fp8(self, k, v, k_pool, v_pool, slot_mapping, dtype, k_scale, v_scale) -> None:
        """In place on uint8 E4M3 pools: code = encode(x / scale) in fp32."""
        for a in (k_pool, v_pool):
            assert a.dtype == np.uint8 and a.flags.c_contiguous
        k = np.ascontiguousarray(k, dtype=np.uint16)
        v = np.ascontiguousarray(v, dtype=np.uint16)
        slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        T, Hkv, D = k.shape
        NB, Hkv2, bs, D2 = k_pool.shape
        assert Hkv2 == Hkv and D2 == D and v.shape == k.shape and slot_mapping.shape == (T,)
        assert slot_mapping.max(initial=-1) < NB * bs
        self.lib.oracle_reshape_and_cache_fp8(_ptr(k), _ptr(v), _ptr(k_pool), _ptr(v_pool), _ptr(slot_mapping),
                                              T, Hkv, D, bs, dtype_code(dtype), float(k_scale), float(v_scale))

    def int8_to_double(self, codes) -> np.ndarray:
        flat = np.ascontiguousarray(codes, dtype=np.uint8).ravel()
        f = self.lib.oracle_int8_to_double
        return np.array([f(int(c)) for c in flat], dtype=np.float64).reshape(np.shape(codes))

    def int8_encode(self, values) -> np.ndarray:
        flat = np.ascontiguousarray(values, dtype=np.float32).ravel()
        f = self.lib.oracle_int8_encode
        return np.array([f(float(v)) for v in flat], dtype=np.uint8).reshape(np.shape(values))

    def paged_attention_kv8(self, q, k_pool, v_pool, block_tables, context_lens, scale, q_dtype, kv_format,
                            k_scales, v_scales, num_threads: int = 0) -> np.ndarray:
        """out[s][h][:] in fp64 over an 8-bit cache (uint8 codes; kv_format "e4m3" or
        "int8") with one scale per KV head (k_scales, v_scales: [num_kv_heads]) or
        one per (physical block, KV head) ([num_blocks][num_kv_heads])."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        k_pool = np.ascontiguousarray(k_pool, dtype=np.uint8)
        v_pool = np.ascontiguousarray(v_pool, dtype=np.uint8)
        block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        B, H, D = q.shape
        NB, Hkv, bs, D2 = k_pool.shape
        assert D2 == D and v_pool.shape == k_pool.shape and H % Hkv == 0
        ks = np.ascontiguousarray(k_scales, dtype=np.float64)
        vs = np.ascontiguousarray(v_scales, dtype=np.float64)
        per_block = ks.ndim == 2
        assert ks.shape == vs.shape and ks.shape in ((Hkv,), (NB, Hkv))
        for s in range(B):
            n = int(context_lens[s])
            pages = -(-n // bs)
            assert 0 <= n and pages <= block_tables.shape[1]
            if pages:
                used = block_tables[s, :pages]
                assert used.min() >= 0 and used.max() < NB
        out = np.zeros((B, H, D), dtype=np.float64)
        fn = self.lib.oracle_paged_attention_kv8_blocks if per_block else self.lib.oracle_paged_attention_kv8
        fn(
            _ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), _ptr(context_lens),
            B, H, Hkv, D, bs, block_tables.shape[1], float(scale), dtype_code(q_dtype), KV_FORMATS[kv_format],
            _ptr(ks), _ptr(vs), int(num_threads))
        return out

    def reshape_and_cache_kv8(self, k, v, k_pool, v_pool, slot_mapping, dtype, kv_format, k_scales,
                              v_scales) -> None:
        """In place on uint8 pools: code = encode(x / scale) in fp32, the scale of
        KV head h ([num_kv_heads] arrays) or of (the slot's block, h)
        ([num_blocks][num_kv_heads])."""
        for a in (k_pool, v_pool):
            assert a.dtype == np.uint8 and a.flags.c_contiguous
        k = np.ascontiguousarray(k, dtype=np.uint16)
        v = np.ascontiguousarray(v, dtype=np.uint16)
        slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        T, Hkv, D = k.shape
        NB, Hkv2, bs, D2 = k_pool.shape
        assert Hkv2 == Hkv and D2 == D and v.shape == k.shape and slot_mapping.shape == (T,)
        assert slot_mapping.max(initial=-1) < NB * bs
        ks = np.ascontiguousarray(k_scales, dtype=np.float32)
        vs = np.ascontiguousarray(v_scales, dtype=np.float32)
        per_block = ks.ndim == 2
        assert ks.shape == vs.shape and ks.shape in ((Hkv,), (NB, Hkv))
        fn = self.lib.oracle_reshape_and_cache_kv8_blocks if per_block else self.lib.oracle_reshape_and_cache_kv8
        fn(_ptr(k), _ptr(v), _ptr(k_pool), _ptr(v_pool), _ptr(slot_mapping), T, Hkv, D, bs, dtype_code(dtype),
           KV_FORMATS[kv_format], _ptr(ks), _ptr(vs))

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    # -- paged attention ----------------------------------------------------
    def paged_attention(self, q, k_pool, v_pool, block_tables, context_lens, scale,
                        dtype, num_threads: int = 0) -> np.ndarray:
        """out[s][h][:] in fp64. q [B][H][D], pools [NB][Hkv][bs][D] (uint16 bits)."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        k_pool = np.ascontiguousarray(k_pool, dtype=np.uint16)
        v_pool = np.ascontiguousarray(v_pool, dtype=np.uint16)
        block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        B, H, D = q.shape
        NB, Hkv, bs, D2 = k_pool.shape
        assert D2 == D and v_pool.shape == k_pool.shape and H % Hkv == 0
        assert block_tables.shape[0] == B and context_lens.shape == (B,)
        # The oracle trusts its inputs; check here the indices it will follow.
        for s in range(B):
            n = int(context_lens[s])
            pages = -(-n // bs)
            assert 0 <= n and pages <= block_tables.shape[1]
            if pages:
                used = block_tables[s, :pages]
                assert used.min() >= 0 and used.max() < NB
        out = np.zeros((B, H, D), dtype=np.float64)
        self.lib.oracle_paged_attention(
            _ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables),
            _ptr(context_lens), B, H, Hkv, D, bs, block_tables.shape[1],
            float(scale), dtype_code(dtype), int(num_threads))
        return out

    # -- data movers ----------------------------------------------------------
    def reshape_and_cache(self, k, v, k_pool, v_pool, slot_mapping) -> None:
        """In place on k_pool / v_pool (uint16 [NB][Hkv][bs][D])."""
        for a in (k_pool, v_pool):
            assert a.dtype == np.uint16 and a.flags.c_contiguous
        k = np.ascontiguousarray(k, dtype=np.uint16)
        v = np.ascontiguousarray(v, dtype=np.uint16)
        slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        T, Hkv, D = k.shape
        NB, Hkv2, bs, D2 = k_pool.shape
        assert Hkv2 == Hkv and D2 == D and v.shape == k.shape and slot_mapping.shape == (T,)
        assert slot_mapping.max(initial=-1) < NB * bs
        self.lib.oracle_reshape_and_cache(_ptr(k), _ptr(v), _ptr(k_pool), _ptr(v_pool),
                                          _ptr(slot_mapping), T, Hkv, D, bs)

    def copy_blocks(self, pools, src_dst_pairs, block_bytes: int) -> None:
        """In place on each pool (any contiguous numpy array), whole blocks."""
        pairs = np.ascontiguousarray(src_dst_pairs, dtype=np.int64).reshape(-1, 2)
        for a in pools:
            assert a.flags.c_contiguous
            nblocks = a.nbytes // block_bytes
            assert pairs.size == 0 or (pairs.min() >= 0 and pairs.max() < nblocks)
        arr = (ctypes.c_void_p * max(1, len(pools)))(*[a.ctypes.data for a in pools])
        self.lib.oracle_copy_blocks(arr, len(pools), _ptr(pairs), pairs.shape[0],
                                    int(block_bytes))

    def swap_blocks(self, dst_pools, src_pools, src_dst_pairs, block_bytes: int) -> None:
        """In place on each dst pool: dst_pools[i][dst] = src_pools[i][src] per pair."""
        pairs = np.ascontiguousarray(src_dst_pairs, dtype=np.int64).reshape(-1, 2)
        assert len(dst_pools) == len(src_pools)
        for d, s_ in zip(dst_pools, src_pools):
            assert d.flags.c_contiguous and s_.flags.c_contiguous
            if pairs.size:
                assert pairs[:, 0].min() >= 0 and pairs[:, 0].max() < s_.nbytes // block_bytes
                assert pairs[:, 1].min() >= 0 and pairs[:, 1].max() < d.nbytes // block_bytes
        n = max(1, len(dst_pools))
        darr = (ctypes.c_void_p * n)(*[a.ctypes.data for a in dst_pools])
        sarr = (ctypes.c_void_p * n)(*[a.ctypes.data for a in src_pools])
        self.lib.oracle_swap_blocks(darr, sarr, len(dst_pools), _ptr(pairs), pairs.shape[0], int(block_bytes))

    def slot_mapping(self, block_tables, seq_ids, positions, block_size: int) -> np.ndarray:
        block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        seq_ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
        positions = np.ascontiguousarray(positions, dtype=np.int32)
        n = seq_ids.shape[0]
        slots = np.zeros(n, dtype=np.int64)
        self.lib.oracle_slot_mapping(_ptr(slots), _ptr(block_tables), block_tables.shape[1],
                                     _ptr(seq_ids), _ptr(positions), n, int(block_size))
        return slots


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from ``pa_oracle.c`` in this directory."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def paged_attention(*args, **kwargs):
    return get().paged_attention(*args, **kwargs)


def reshape_and_cache(*args, **kwargs):
    return get().reshape_and_cache(*args, **kwargs)


def copy_blocks(*args, **kwargs):
    return get().copy_blocks(*args, **kwargs)


def slot_mapping(*args, **kwargs):
    return get().slot_mapping(*args, **kwargs)


def swap_blocks(*args, **kwargs):
    return get().swap_blocks(*args, **kwargs)


def paged_attention_fp8(*args, **kwargs):
    return get().paged_attention_fp8(*args, **kwargs)


def reshape_and_cache_fp8(*args, **kwargs):
    return get().reshape_and_cache_fp8(*args, **kwargs)


def paged_attention_kv8(*args, **kwargs):
    return get().paged_attention_kv8(*args, **kwargs)


def reshape_and_cache_kv8(*args, **kwargs):
    return get().reshape_and_cache_kv8(*args, **kwargs)


def to_double(*args, **kwargs):
    return get().to_double(*args, **kwargs)


def max_threads() -> int:
    return get().max_threads()
