"""Paged attention for continuous batching on NVIDIA B200 (sm_100a).

A thin ctypes binding of ``libpagedattn.so`` (declared in
``include/pagedattn.h``): the functions below carry the C names and only
marshal arguments -- shapes and raw device pointers of torch tensors -- into
the C calls.  All computation runs in the library's CUDA kernels; there is
no Python or CPU fallback, and importing this package fails loudly when the
library has not been built (``python scatter_kv_b200/build.py``).

Calls:
  pa_scatter_kv            new K/V tokens -> paged cache (in place)
  pa_compute_slot_mapping  cache slot of every new token
  pa_attention             causal GQA attention over the paged cache
  pa_attention_workspace_size, pa_get_status, pa_trace_*  (plumbing)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_OK = 0
PA_ERR_INVALID_ARGUMENT = 1
PA_ERR_NOT_IMPLEMENTED = 2
PA_ERR_CUDA = 3

PA_DTYPE_F16 = 0
PA_DTYPE_BF16 = 1

PA_DEV_BAD_CU_SEQLENS = 1 << 0
PA_DEV_QLEN_GT_KV = 1 << 1
PA_DEV_KV_TOO_LONG = 1 << 2
PA_DEV_BAD_BLOCK = 1 << 3
PA_DEV_BAD_SLOT = 1 << 4
PA_DEV_TIMEOUT = 1 << 5
PA_DEV_HINT_EXCEEDED = 1 << 6
PA_DEV_BAD_POSITION = 1 << 7
PA_DEV_BAD_SELECTION = 1 << 8

PA_KERNEL_SCATTER = 0
PA_KERNEL_SLOT_MAPPING = 1
PA_KERNEL_DECODE = 2
PA_KERNEL_COMBINE = 3
PA_KERNEL_PREFILL = 4
PA_KERNEL_QKV_ROTARY = 5
PA_KERNEL_SPARSE = 6
PA_TRACE_CAPACITY = 4096


class pa_dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("token_count", ctypes.c_int64),
        ("q_heads", ctypes.c_int32),
        ("kv_heads", ctypes.c_int32),
        ("head_size", ctypes.c_int32),
        ("num_blocks", ctypes.c_int64),
        ("block_size", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
        ("max_seqlen_q_hint", ctypes.c_int32),
        ("max_seqlen_kv_hint", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("min_seqlen_q_hint", ctypes.c_int32),
        ("softcap", ctypes.c_float),
        ("local_window", ctypes.c_int32),
        ("local_window_size", ctypes.c_int32),
    ]


class pa_rotary(ctypes.Structure):
    _fields_ = [
        ("rotary_dim", ctypes.c_int32),
        ("interleaved", ctypes.c_int32),
        ("max_position", ctypes.c_int64),
    ]


class pa_trace_record(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("ms", ctypes.c_float)]


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_status_name(status)}: {message}")
        self.status = status


EXPORTS = [
    "pa_scatter_kv", "pa_compute_slot_mapping", "pa_attention_workspace_size", "pa_attention",
    "pa_get_status", "pa_status_string", "pa_last_error", "pa_trace_enable", "pa_trace_read",
    "pa_kernel_name", "pa_attention_noalloc", "pa_split_qkv_rotary_scatter",
    "pa_scatter_kv_int4", "pa_attention_int4", "pa_sparse_attention", "pa_selftest_wait_timeout",
]

# Bytes of the fixed scratch array behind pa_attention_noalloc.
NOALLOC_SCRATCH_BYTES = 8 << 20


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python scatter_kv_b200/build.py` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32P = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)
    D = ctypes.POINTER(pa_dims)
    lib.pa_scatter_kv.argtypes = [P, P, P, P, P, D, P, P]
    lib.pa_scatter_kv.restype = ctypes.c_int
    lib.pa_compute_slot_mapping.argtypes = [P, P, P, P, D, P, P]
    lib.pa_compute_slot_mapping.restype = ctypes.c_int
    lib.pa_attention_workspace_size.argtypes = [D, ctypes.POINTER(ctypes.c_size_t)]
    lib.pa_attention_workspace_size.restype = ctypes.c_int
    lib.pa_attention.argtypes = [P, P, P, P, P, P, ctypes.c_float, P, D, P, ctypes.c_size_t, P, P]
    lib.pa_attention.restype = ctypes.c_int
    lib.pa_attention_noalloc.argtypes = [P, P, P, P, P, P, ctypes.c_float, P, D, P, P]
    lib.pa_attention_noalloc.restype = ctypes.c_int
    lib.pa_selftest_wait_timeout.argtypes = [P, P]
    lib.pa_selftest_wait_timeout.restype = ctypes.c_int
    lib.pa_split_qkv_rotary_scatter.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int64, P, P,
                                                ctypes.POINTER(pa_rotary), P, P, P, P, P, P, P,
                                                D, P, P]
    lib.pa_split_qkv_rotary_scatter.restype = ctypes.c_int
    lib.pa_scatter_kv_int4.argtypes = [P, P, P, P, P, P, P, D, P, P]
    lib.pa_scatter_kv_int4.restype = ctypes.c_int
    lib.pa_attention_int4.argtypes = [P, P, P, P, P, P, P, P, ctypes.c_float, P, D, P,
                                      ctypes.c_size_t, P, P]
    lib.pa_attention_int4.restype = ctypes.c_int
    lib.pa_sparse_attention.argtypes = [P, P, P, P, P, P, P, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_float, P, D, P, P]
    lib.pa_sparse_attention.restype = ctypes.c_int
    lib.pa_get_status.argtypes = [P, I32P, P]
    lib.pa_get_status.restype = ctypes.c_int
    lib.pa_status_string.argtypes = [ctypes.c_int]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_last_error.argtypes = []
    lib.pa_last_error.restype = ctypes.c_char_p
    lib.pa_trace_enable.argtypes = [ctypes.c_int]
    lib.pa_trace_enable.restype = ctypes.c_int
    lib.pa_trace_read.argtypes = [ctypes.POINTER(pa_trace_record), ctypes.c_int]
    lib.pa_trace_read.restype = ctypes.c_int
    lib.pa_kernel_name.argtypes = [ctypes.c_int32]
    lib.pa_kernel_name.restype = ctypes.c_char_p
    return lib


lib = _load()


def _status_name(st: int) -> str:
    return lib.pa_status_string(int(st)).decode()


def _check(st: int):
    if st != PA_OK:
        raise PagedAttentionError(st, lib.pa_last_error().decode())


def _ptr(t):
    """Device (or host) address of a torch tensor; None -> NULL; ints pass through."""
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


def make_dims(query=None, key_cache=None, block_table=None, cu_seqlens_q=None, *, batch=None,
              token_count=None, q_heads=None, kv_heads=None, head_size=None, num_blocks=None,
              block_size=None, max_blocks_per_seq=None, max_seqlen_q=0, max_seqlen_kv=0,
              min_seqlen_q=0, dtype=PA_DTYPE_F16, softcap=0.0, window=None) -> pa_dims:
    """pa_dims from tensor shapes (query [T, qh, d], cache [nb, bs, kvh, d],
    block table [B, maxblk], cu_seqlens_q [B + 1]); keywords override.
    ``softcap`` > 0 caps the scaled scores; ``window`` = w (an int >= 0) lets
    the query at position P see only keys [P - w, P] (None: no window)."""
    d = pa_dims()
    if query is not None:
        d.token_count, d.q_heads, d.head_size = query.shape
    if key_cache is not None:
        d.num_blocks, d.block_size, d.kv_heads, hs = key_cache.shape
        d.head_size = hs
    if block_table is not None:
        d.batch, d.max_blocks_per_seq = block_table.shape
    if cu_seqlens_q is not None:
        d.batch = cu_seqlens_q.shape[0] - 1
    for name, val in (("batch", batch), ("token_count", token_count), ("q_heads", q_heads),
                      ("kv_heads", kv_heads), ("head_size", head_size), ("num_blocks", num_blocks),
                      ("block_size", block_size), ("max_blocks_per_seq", max_blocks_per_seq)):
        if val is not None:
            setattr(d, name, int(val))
    d.max_seqlen_q_hint = int(max_seqlen_q)
    d.max_seqlen_kv_hint = int(max_seqlen_kv)
    d.min_seqlen_q_hint = int(min_seqlen_q)
    d.dtype = int(dtype)
    d.softcap = float(softcap)
    d.local_window = 0 if window is None else 1
    d.local_window_size = 0 if window is None else int(window)
    return d


def pa_scatter_kv(key, value, slot_mapping, key_cache, value_cache, dims: pa_dims,
                  dev_status=None, stream=None) -> None:
    _check(lib.pa_scatter_kv(_ptr(key), _ptr(value), _ptr(slot_mapping), _ptr(key_cache),
                             _ptr(value_cache), ctypes.byref(dims), _ptr(dev_status),
                             _stream(stream)))


def pa_compute_slot_mapping(block_table, cu_seqlens_q, seqlens_kv, slot_mapping, dims: pa_dims,
                            dev_status=None, stream=None) -> None:
    _check(lib.pa_compute_slot_mapping(_ptr(block_table), _ptr(cu_seqlens_q), _ptr(seqlens_kv),
                                       _ptr(slot_mapping), ctypes.byref(dims), _ptr(dev_status),
                                       _stream(stream)))


def pa_attention_workspace_size(dims: pa_dims) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.pa_attention_workspace_size(ctypes.byref(dims), ctypes.byref(n)))
    return int(n.value)


def pa_attention(query, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv, scale,
                 out, dims: pa_dims, workspace=None, workspace_bytes=None, dev_status=None,
                 stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None or isinstance(workspace, int) else \
            workspace.numel() * workspace.element_size()
    _check(lib.pa_attention(_ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_table),
                            _ptr(cu_seqlens_q), _ptr(seqlens_kv), float(scale), _ptr(out),
                            ctypes.byref(dims), _ptr(workspace), int(workspace_bytes),
                            _ptr(dev_status), _stream(stream)))


def pa_attention_noalloc(query, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv,
                         scale, out, dims: pa_dims, dev_status=None, stream=None) -> None:
    """pa_attention without a workspace argument, for callers that cannot
    allocate device memory: the split-KV scratch is a fixed 8 MiB array inside
    the library (dims needing more are rejected).  Calls that overlap on the
    GPU share that array and race; the first call on a device looks up the
    array's address and should come before any stream capture."""
    _check(lib.pa_attention_noalloc(_ptr(query), _ptr(key_cache), _ptr(value_cache),
                                    _ptr(block_table), _ptr(cu_seqlens_q), _ptr(seqlens_kv),
                                    float(scale), _ptr(out), ctypes.byref(dims), _ptr(dev_status),
                                    _stream(stream)))


def pa_split_qkv_rotary_scatter(query, key, value, q_token_stride, kv_token_stride, cos_cache,
                                sin_cache, rotary: pa_rotary, block_table, cu_seqlens_q,
                                seqlens_kv, query_out, key_cache, value_cache, slot_mapping,
                                dims: pa_dims, dev_status=None, stream=None) -> None:
    """query / key / value: tensors or raw device addresses (ints), with the
    token strides in elements (0 = dense)."""
    _check(lib.pa_split_qkv_rotary_scatter(
        _ptr(query), _ptr(key), _ptr(value), int(q_token_stride), int(kv_token_stride),
        _ptr(cos_cache), _ptr(sin_cache), ctypes.byref(rotary) if rotary is not None else None,
        _ptr(block_table), _ptr(cu_seqlens_q), _ptr(seqlens_kv), _ptr(query_out), _ptr(key_cache),
        _ptr(value_cache), _ptr(slot_mapping), ctypes.byref(dims), _ptr(dev_status),
        _stream(stream)))


def pa_scatter_kv_int4(key, value, slot_mapping, k_scale, v_scale, key_cache, value_cache,
                       dims: pa_dims, dev_status=None, stream=None) -> None:
    _check(lib.pa_scatter_kv_int4(_ptr(key), _ptr(value), _ptr(slot_mapping), _ptr(k_scale),
                                  _ptr(v_scale), _ptr(key_cache), _ptr(value_cache),
                                  ctypes.byref(dims), _ptr(dev_status), _stream(stream)))


def pa_attention_int4(query, key_cache, value_cache, k_scale, v_scale, block_table, cu_seqlens_q,
                      seqlens_kv, scale, out, dims: pa_dims, workspace=None, workspace_bytes=None,
                      dev_status=None, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None or isinstance(workspace, int) else \
            workspace.numel() * workspace.element_size()
    _check(lib.pa_attention_int4(_ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(k_scale),
                                 _ptr(v_scale), _ptr(block_table), _ptr(cu_seqlens_q),
                                 _ptr(seqlens_kv), float(scale), _ptr(out), ctypes.byref(dims),
                                 _ptr(workspace), int(workspace_bytes), _ptr(dev_status),
                                 _stream(stream)))


def pa_sparse_attention(query, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv,
                        selected, num_selected, local_window, scale, out, dims: pa_dims,
                        dev_status=None, stream=None) -> None:
    _check(lib.pa_sparse_attention(_ptr(query), _ptr(key_cache), _ptr(value_cache),
                                   _ptr(block_table), _ptr(cu_seqlens_q), _ptr(seqlens_kv),
                                   _ptr(selected), int(num_selected), int(local_window),
                                   float(scale), _ptr(out), ctypes.byref(dims), _ptr(dev_status),
                                   _stream(stream)))


def packed_qkv_views(qkv, dims: pa_dims):
    """(query, key, value, stride) addresses of a packed QKV tensor
    [token_count, q_heads + 2 kv_heads, head_size] for
    pa_split_qkv_rotary_scatter."""
    esz = qkv.element_size()
    base = qkv.data_ptr()
    hd = dims.head_size
    stride = (dims.q_heads + 2 * dims.kv_heads) * hd
    return (base, base + dims.q_heads * hd * esz,
            base + (dims.q_heads + dims.kv_heads) * hd * esz, stride)


def pa_get_status(dev_status, stream=None) -> int:
    code = ctypes.c_int32(0)
    _check(lib.pa_get_status(_ptr(dev_status), ctypes.byref(code), _stream(stream)))
    return int(code.value)


def pa_selftest_wait_timeout(dev_status, stream=None) -> None:
    """Launch the kernel whose bounded waits must time out (see the header)."""
    _check(lib.pa_selftest_wait_timeout(_ptr(dev_status), _stream(stream)))


def pa_trace_enable(on: bool = True) -> None:
    _check(lib.pa_trace_enable(1 if on else 0))


def pa_trace_read():
    """[(kernel name, ms), ...] of the launches since the last read."""
    buf = (pa_trace_record * PA_TRACE_CAPACITY)()
    n = lib.pa_trace_read(buf, PA_TRACE_CAPACITY)
    return [(lib.pa_kernel_name(buf[i].kernel).decode(), float(buf[i].ms)) for i in range(n)]


@dataclass
class Workspace:
    """Device buffers one paged-attention call needs, sized for ``dims``."""

    out: object
    workspace: object
    status: object
    slot_mapping: object


def allocate(dims: pa_dims, device="cuda", out=None):
    """Allocate output, workspace, status word and slot-mapping buffers with torch."""
    import torch
    nbytes = pa_attention_workspace_size(dims)
    if out is None:
        out = torch.empty((dims.token_count, dims.q_heads, dims.head_size),
                          dtype=torch.bfloat16 if dims.dtype == PA_DTYPE_BF16 else torch.float16,
                          device=device)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    status = torch.zeros(4, dtype=torch.int32, device=device)
    slots = torch.empty(max(dims.token_count, 1), dtype=torch.int32, device=device)
    return Workspace(out, ws, status, slots)


def step(query, key, value, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv,
         scale, dims: pa_dims, buffers: Workspace, stream=None, fused: bool = False):
    """One pass of the hot path: slot mapping, scatter of the new K/V, then
    attention.  ``fused``: slot mapping and scatter in one kernel
    (pa_split_qkv_rotary_scatter without a query output); otherwise
    pa_compute_slot_mapping then pa_scatter_kv.  Both write
    ``buffers.slot_mapping``.  Returns ``buffers.out``."""
    if fused:
        pa_split_qkv_rotary_scatter(None, key, value, 0, 0, None, None, None, block_table,
                                    cu_seqlens_q, seqlens_kv, None, key_cache, value_cache,
                                    buffers.slot_mapping, dims, buffers.status, stream)
    else:
        pa_compute_slot_mapping(block_table, cu_seqlens_q, seqlens_kv, buffers.slot_mapping, dims,
                                buffers.status, stream)
        pa_scatter_kv(key, value, buffers.slot_mapping, key_cache, value_cache, dims,
                      buffers.status, stream)
    pa_attention(query, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv, scale,
                 buffers.out, dims, buffers.workspace, None, buffers.status, stream)
    return buffers.out
