"""fp64 CPU oracle for paged attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product library (``scatter_kv_b200``) never imports it, and this package
imports nothing from there.

The arithmetic lives in ``pa_oracle.c`` (plain C, fp64); this module only
compiles it with gcc, loads it with ctypes and marshals numpy arrays.  See
that file's header for the definitions it follows (FlexAttention operator
doc, "FlexAttention Computation" and "Grouped Query Attention (GQA)"; ONNX
Runtime PR "[WebGPU] Initial PagedAttention implementation (1/n)", section
"FlashAttention: optional seqlens_q input").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "libpa_oracle.so")
_lib = None

F16 = 0
F64 = 1
BF16 = 2


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into libpa_oracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_scatter_kv.argtypes = [P, P, P, P, P, i64, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int]
        lib.oracle_slot_mapping.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            i64, P]
        lib.oracle_kv_slots.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
        lib.oracle_kv_slots.restype = i64
        lib.oracle_attention.argtypes = [P, P, P, P, P, P, ctypes.c_int, i64, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, P, i64, P, i64, P]
        lib.oracle_token_positions.argtypes = [P, P, ctypes.c_int, i64, P]
        lib.oracle_rotary.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, i64, P, P, P,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_sparse_attention.argtypes = [P, P, P, P, P, P, ctypes.c_int, i64, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, P, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_double, ctypes.c_int, P, P, P]
        lib.oracle_quantize_int4.argtypes = [ctypes.c_float, ctypes.c_float]
        lib.oracle_quantize_int4.restype = ctypes.c_int
        lib.oracle_scatter_kv_int4.argtypes = [P, P, P, P, P, P, P, i64, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int]
        lib.oracle_dequantize_int4.argtypes = [P, P, i64, ctypes.c_int, ctypes.c_int, P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def max_threads() -> int:
    """Threads the oracle's OpenMP loop uses (OMP_NUM_THREADS, else all cores)."""
    return int(_load().oracle_max_threads())


def half_to_double(bits: int) -> float:
    return float(_load().oracle_half_to_double(int(bits) & 0xFFFF))


def bf16_to_double(bits: int) -> float:
    return float(_load().oracle_bf16_to_double(int(bits) & 0xFFFF))


def _elem_type(a: np.ndarray, bf16: bool) -> int:
    if bf16:
        if a.dtype != np.uint16:
            raise TypeError("bfloat16 arrays are passed as uint16 bit patterns")
        return BF16
    if a.dtype == np.float16:
        return F16
    if a.dtype == np.float64:
        return F64
    raise TypeError("oracle takes float16, float64 or (bf16=True) uint16 arrays")


def scatter_kv(key, value, slot_mapping, key_cache, value_cache) -> None:
    """In place: key_cache[slot // bs, slot % bs] = key[t] (and value), slot >= 0."""
    lib = _load()
    assert key_cache.flags.c_contiguous and value_cache.flags.c_contiguous
    assert key_cache.dtype == key.dtype == value.dtype == value_cache.dtype
    key = _c(key, key.dtype)
    value = _c(value, value.dtype)
    slots = _c(slot_mapping, np.int32)
    nb, bs, kvh, d = key_cache.shape
    lib.oracle_scatter_kv(_ptr(key), _ptr(value), _ptr(slots), _ptr(key_cache), _ptr(value_cache),
                          key.shape[0], kvh, d, bs, key.dtype.itemsize)


def slot_mapping(block_table, cu_seqlens_q, seqlens_kv, block_size: int) -> np.ndarray:
    lib = _load()
    bt = _c(block_table, np.int32)
    cu = _c(cu_seqlens_q, np.int32)
    skv = _c(seqlens_kv, np.int32)
    token_count = int(cu[-1])
    out = np.empty(token_count, dtype=np.int32)
    lib.oracle_slot_mapping(_ptr(bt), _ptr(cu), _ptr(skv), len(skv), bt.shape[1], block_size,
                            token_count, _ptr(out))
    return out


def kv_slots(block_table, seqlens_kv, block_size: int) -> np.ndarray:
    """Slots of logical positions [0, seqlens_kv[b]) for every sequence b."""
    lib = _load()
    bt = _c(block_table, np.int32)
    skv = _c(seqlens_kv, np.int32)
    out = np.empty(int(skv.astype(np.int64).sum()), dtype=np.int32)
    n = lib.oracle_kv_slots(_ptr(bt), _ptr(skv), len(skv), bt.shape[1], block_size, _ptr(out))
    assert n == out.size
    return out


def attention(query, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv,
              scale: float, causal: bool = True, rows=None, softcap: float = 0.0,
              window: int = -1, bf16: bool = False) -> np.ndarray:
    """fp64 paged attention.

    query [token_count, q_heads, head_size]; caches [num_blocks, block_size,
    kv_heads, head_size]; all float16, all float64, or (bf16=True) all
    bfloat16 bit patterns held as uint16.  ``rows``: optional int64 [n, 2]
    array of (token, q_head) pairs to compute; the result is then
    [n, head_size], else [token_count, q_heads, head_size] (float64).
    ``softcap`` > 0 caps the scaled scores at c * tanh(s / c); ``window`` >= 0
    lets query position P see only keys [P - window, P].
    """
    lib = _load()
    dtype = _elem_type(query, bf16)
    assert key_cache.dtype == value_cache.dtype == query.dtype
    q = _c(query, query.dtype)
    kc = key_cache if key_cache.flags.c_contiguous else np.ascontiguousarray(key_cache)
    vc = value_cache if value_cache.flags.c_contiguous else np.ascontiguousarray(value_cache)
    bt = _c(block_table, np.int32)
    cu = _c(cu_seqlens_q, np.int32)
    skv = _c(seqlens_kv, np.int32)
    token_count, q_heads, head_size = q.shape
    nb, bs, kv_heads, d2 = kc.shape
    assert d2 == head_size
    max_keys = max(1, int(skv.max()) if skv.size else 1)
    nthreads = max_threads()
    scratch = np.empty(nthreads * max_keys, dtype=np.float64)
    if rows is None:
        out = np.empty((token_count, q_heads, head_size), dtype=np.float64)
        rows_p, nrows = None, token_count * q_heads
    else:
        rows = _c(rows, np.int64).reshape(-1, 2)
        out = np.empty((rows.shape[0], head_size), dtype=np.float64)
        rows_p, nrows = _ptr(rows), rows.shape[0]
    if nrows:
        lib.oracle_attention(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), _ptr(cu), _ptr(skv), len(skv),
                             token_count, q_heads, kv_heads, head_size, bs, bt.shape[1],
                             float(scale), float(softcap), int(window), 1 if causal else 0, dtype,
                             rows_p, nrows, _ptr(scratch), max_keys, _ptr(out))
    return out


def token_positions(cu_seqlens_q, seqlens_kv) -> np.ndarray:
    """Position past_len_b + i of every packed token (int64 [token_count])."""
    lib = _load()
    cu = _c(cu_seqlens_q, np.int32)
    skv = _c(seqlens_kv, np.int32)
    out = np.empty(int(cu[-1]), dtype=np.int64)
    lib.oracle_token_positions(_ptr(cu), _ptr(skv), len(skv), out.size, _ptr(out))
    return out


def rotary(x, positions, cos_cache, sin_cache, rotary_dim: int, interleaved: bool,
           bf16: bool = False) -> np.ndarray:
    """Rotary embedding of x [token_count, heads, head_size] (any row stride
    over tokens; heads contiguous) at the given positions; cos/sin caches
    [max_position, rotary_dim / 2] of x's element type.  Returns float64."""
    lib = _load()
    dtype = _elem_type(x, bf16)
    assert cos_cache.dtype == sin_cache.dtype == x.dtype
    T, H, d = x.shape
    assert x.strides[2] == x.itemsize and x.strides[1] == d * x.itemsize
    assert rotary_dim % 2 == 0 and 0 <= rotary_dim <= d
    assert cos_cache.shape[1] == rotary_dim // 2 and cos_cache.shape == sin_cache.shape
    pos = _c(positions, np.int64)
    assert pos.size == T and (T == 0 or (pos.min() >= 0 and pos.max() < cos_cache.shape[0]))
    cc = _c(cos_cache, cos_cache.dtype)
    sc = _c(sin_cache, sin_cache.dtype)
    out = np.empty((T, H, d), dtype=np.float64)
    if T:
        base = x.ctypes.data_as(ctypes.c_void_p)
        lib.oracle_rotary(base, T, H, d, x.strides[0] // x.itemsize, _ptr(pos), _ptr(cc), _ptr(sc),
                          rotary_dim, 1 if interleaved else 0, dtype, _ptr(out))
    return out


def quantize_int4(x: float, scale: float) -> int:
    """Code of one value: round(x / scale) (binary32, ties to even) clamped to [-8, 7]."""
    return int(_load().oracle_quantize_int4(float(x), float(scale)))


def scatter_kv_int4(key, value, slot_mapping, k_scale, v_scale, key_cache, value_cache,
                    bf16: bool = False) -> None:
    """In place: quantise token t's K/V rows with the per-channel scales
    [kv_heads, head_size] and pack them into INT4 cache slot slot_mapping[t]
    (caches uint8 [num_blocks, block_size, kv_heads, head_size // 2])."""
    lib = _load()
    dtype = _elem_type(key, bf16)
    assert key_cache.dtype == value_cache.dtype == np.uint8
    assert key_cache.flags.c_contiguous and value_cache.flags.c_contiguous
    key = _c(key, key.dtype)
    value = _c(value, value.dtype)
    T, kvh, d = key.shape
    assert key_cache.shape[2:] == (kvh, d // 2)
    ks = _c(k_scale, np.float32).reshape(kvh, d)
    vs = _c(v_scale, np.float32).reshape(kvh, d)
    slots = _c(slot_mapping, np.int32)
    lib.oracle_scatter_kv_int4(_ptr(key), _ptr(value), _ptr(slots), _ptr(ks), _ptr(vs),
                               _ptr(key_cache), _ptr(value_cache), T, kvh, d, dtype)


def dequantize_int4(cache, scale) -> np.ndarray:
    """float64 [num_blocks, block_size, kv_heads, head_size] values of an INT4 cache."""
    lib = _load()
    nb, bs, kvh, half = cache.shape
    d = 2 * half
    c = _c(cache, np.uint8)
    sc = _c(scale, np.float32).reshape(kvh, d)
    out = np.empty((nb, bs, kvh, d), dtype=np.float64)
    lib.oracle_dequantize_int4(_ptr(c), _ptr(sc), nb * bs, kvh, d, _ptr(out))
    return out


def sparse_attention(query, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv,
                     selected, local_window: int, scale: float, bf16: bool = False) -> np.ndarray:
    """Local-plus-selected attention: token t and KV head h see keys
    [P - local_window, P] plus the selected positions selected[t, h, :] that
    are in [0, P] (int32 [token_count, kv_heads, num_selected]; -1 pads),
    each key once.  Returns float64 [token_count, q_heads, head_size]."""
    lib = _load()
    dtype = _elem_type(query, bf16)
    q = _c(query, query.dtype)
    kc = key_cache if key_cache.flags.c_contiguous else np.ascontiguousarray(key_cache)
    vc = value_cache if value_cache.flags.c_contiguous else np.ascontiguousarray(value_cache)
    bt = _c(block_table, np.int32)
    cu = _c(cu_seqlens_q, np.int32)
    skv = _c(seqlens_kv, np.int32)
    sel = _c(selected, np.int32)
    T, qh, d = q.shape
    nb, bs, kvh, _ = kc.shape
    assert sel.shape[:2] == (T, kvh) and local_window >= 0
    max_keys = max(1, int(skv.max()) if skv.size else 1)
    mark = np.empty(max_keys, dtype=np.uint8)
    scores = np.empty(max_keys, dtype=np.float64)
    out = np.empty((T, qh, d), dtype=np.float64)
    if T:
        lib.oracle_sparse_attention(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), _ptr(cu), _ptr(skv),
                                    len(skv), T, qh, kvh, d, bs, bt.shape[1], _ptr(sel),
                                    sel.shape[2], int(local_window), float(scale), dtype,
                                    _ptr(mark), _ptr(scores), _ptr(out))
    return out
