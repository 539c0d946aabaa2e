"""Thin ctypes binding of libpa.so.

Every function here has the name of the C entry point it calls and only
marshals arguments: it reads shapes, dtypes and device pointers off torch
tensors, checks that they are CUDA tensors laid out as the C ABI expects,
calls the library on the current (or given) stream, and raises PAError on a
non-zero status.  All computation happens in the library's CUDA kernels;
there is no other code path.  If libpa.so has not been built the import of
this module fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_F32, PA_BF16 = 0, 1
_STATUS = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_WORKSPACE",
           4: "PA_ERR_CUDA", 5: "PA_ERR_BAD_BLOCK_ID", 6: "PA_ERR_TIMEOUT"}
_DTYPES = {torch.float32: PA_F32, torch.bfloat16: PA_BF16}

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_355_b200.build` "
                      "(or __graft_entry__.build()); there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH)
_P, _I, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "pa_status_string": ([_I], ctypes.c_char_p),
    "pa_version": ([], ctypes.c_char_p),
    "pa_read_error_flag": ([_P], _I),
    "pa_selftest_wait_timeout": ([ctypes.c_uint32, _P], _I),
    "pa_hbm_read_probe": ([_P, _SZ, _P], _I),
    "pa_slot_mapping": ([_P, _I, _I, _P, _P, _I64, _I, _P, _P], _I),
    "pa_decode_slot_mapping": ([_P, _I, _P, _I, _I, _P, _P], _I),
    "pa_reshape_and_cache": ([_P, _P, _P, _P, _P, _I64, _I, _I, _I, _I64, _I, _P], _I),
    "pa_reshape_and_cache_decode": ([_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I64, _I, _P, _P], _I),
    "pa_copy_blocks": ([_P, _P, _P, _I64, _I, _I, _I, _I64, _I, _P], _I),
    "pa_swap_blocks": ([_P, _P, _P, _P, _P, _I64, _I, _I, _I, _I64, _I64, _I, _P], _I),
    "pa_paged_attention_partition_size": ([_I, _I, _I, _I, _I, _I, ctypes.POINTER(_I)], _I),
    "pa_paged_attention_workspace_size": ([_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "pa_paged_attention_decode": ([_P, _P, _P, _P, _I, _P, _I, _F, _I, _P, _I, _I, _I, _I, _I, _I64, _I, _I, _P,
                                   _SZ, _P], _I),
    "pa_paged_attention_decode_append": ([_P, _P, _P, _P, _P, _P, _I, _P, _I, _F, _I, _P, _I, _I, _I, _I, _I, _I64, _I,
                                          _I, _P, _SZ, _P, _P], _I),
    "pa_paged_attention_shared_prefix_workspace_size": ([_I, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                                                        ctypes.POINTER(_SZ)], _I),
    "pa_paged_attention_decode_shared_prefix": ([_P, _P, _P, _P, _I, _P, _I, _F, _I, _P, _I, _I, _I, _I, _I, _I64,
                                                 _I, _P, _P, _I, _I, _I, _I, _P, _SZ, _P], _I),
    "pa_paged_attention_decode_contiguous": ([_P, _P, _P, _I64, _P, _I, _F, _I, _P, _I, _I, _I, _I, _I, _I, _I, _P,
                                              _SZ, _P], _I),
    "pa_paged_attention_prefill": ([_P, _P, _P, _P, _I, _P, _P, _I, _F, _I, _P, _I, _I, _I, _I, _I, _I64, _I64, _I,
                                    _P], _I),
    "pa_paged_attention_decode_static_scratch": ([_P, _P, _P, _P, _I, _P, _I, _F, _I, _P, _I, _I, _I, _I, _I, _I64,
                                                  _I, _I, _P], _I),
    # host-side block manager (host pointers)
    "pa_bm_create": ([_I64, _I], _P),
    "pa_bm_destroy": ([_P], None),
    "pa_bm_add_sequence": ([_P, _I64], _I),
    "pa_bm_append_tokens": ([_P, _P, _I64, _P, _P, _P], _I),
    "pa_bm_fork": ([_P, _I64, _I64], _I),
    "pa_bm_free_sequence": ([_P, _I64], _I),
    "pa_bm_num_free": ([_P], _I64),
    "pa_bm_refcount": ([_P, _I64], _I),
    "pa_bm_length": ([_P, _I64], _I64),
    "pa_bm_block_tables": ([_P, _P, _I64, _I, _P, _P], _I),
    "pa_bm_free_list": ([_P, _P, _I64, _P], _I),
    "pa_bm_shared_prefix_groups": ([_P, _P, _I64, _P, _P, _P, _P, _P], _I),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGS)


class PAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {_STATUS.get(status, status)}")


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise PAError(fn, status)


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _kv_dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported element type {t.dtype}: use float32 or bfloat16")
    return _DTYPES[t.dtype]


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def pa_status_string(status: int) -> str:
    return _lib.pa_status_string(status).decode()


def pa_version() -> str:
    return _lib.pa_version().decode()


def pa_read_error_flag(stream=None) -> int:
    """Synchronise the stream and return (then clear) the device error word."""
    return int(_lib.pa_read_error_flag(_stream(stream)))


def pa_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _check("pa_selftest_wait_timeout", _lib.pa_selftest_wait_timeout(limit_us, _stream(stream)))


def pa_hbm_read_probe(buffer, stream=None) -> None:
    """Stream every byte of a CUDA tensor through shared memory and discard
    it (the device's HBM read ceiling; nothing is written)."""
    nbytes = buffer.numel() * buffer.element_size()
    _check("pa_hbm_read_probe", _lib.pa_hbm_read_probe(_dev(buffer, "buffer"), nbytes, _stream(stream)))


def pa_slot_mapping(block_tables, seq_ids, positions, block_size: int, slot_mapping, stream=None) -> None:
    B, MBS = block_tables.shape
    n = seq_ids.numel()
    _check("pa_slot_mapping", _lib.pa_slot_mapping(
        _dev(block_tables, "block_tables", torch.int32), MBS, B, _dev(seq_ids, "seq_ids", torch.int32),
        _dev(positions, "positions", torch.int32), n, block_size, _dev(slot_mapping, "slot_mapping", torch.int64),
        _stream(stream)))


def pa_decode_slot_mapping(block_tables, context_lens, block_size: int, slot_mapping, stream=None) -> None:
    B, MBS = block_tables.shape
    _check("pa_decode_slot_mapping", _lib.pa_decode_slot_mapping(
        _dev(block_tables, "block_tables", torch.int32), MBS, _dev(context_lens, "context_lens", torch.int32), B,
        block_size, _dev(slot_mapping, "slot_mapping", torch.int64), _stream(stream)))


def pa_reshape_and_cache(key, value, k_pool, v_pool, slot_mapping, stream=None) -> None:
    T, Hkv, D = key.shape
    NB, Hkv2, bs, D2 = k_pool.shape
    if (Hkv2, D2) != (Hkv, D) or value.shape != key.shape or v_pool.shape != k_pool.shape:
        raise ValueError("key/value and pool shapes disagree")
    dt = _kv_dtype(key)
    for t, n in ((value, "value"), (k_pool, "k_pool"), (v_pool, "v_pool")):
        _dev(t, n, key.dtype)
    _check("pa_reshape_and_cache", _lib.pa_reshape_and_cache(
        _dev(key, "key"), value.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
        _dev(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D, bs, NB, dt, _stream(stream)))


def pa_reshape_and_cache_decode(key, value, k_pool, v_pool, block_tables, context_lens, slot_mapping=None,
                                stream=None) -> None:
    B, Hkv, D = key.shape
    NB, Hkv2, bs, D2 = k_pool.shape
    if (Hkv2, D2) != (Hkv, D) or value.shape != key.shape or v_pool.shape != k_pool.shape:
        raise ValueError("key/value and pool shapes disagree")
    if block_tables.shape[0] != B or context_lens.numel() != B:
        raise ValueError("block_tables / context_lens do not match the batch of key")
    dt = _kv_dtype(key)
    for t, n in ((value, "value"), (k_pool, "k_pool"), (v_pool, "v_pool")):
        _dev(t, n, key.dtype)
    slots = 0 if slot_mapping is None else _dev(slot_mapping, "slot_mapping", torch.int64)
    _check("pa_reshape_and_cache_decode", _lib.pa_reshape_and_cache_decode(
        _dev(key, "key"), value.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), B, Hkv, D, bs, NB, dt, slots or None, _stream(stream)))


def pa_copy_blocks(k_pool, v_pool, block_mapping, stream=None) -> None:
    NB, Hkv, bs, D = k_pool.shape
    _dev(v_pool, "v_pool", k_pool.dtype)
    P = block_mapping.numel() // 2
    _check("pa_copy_blocks", _lib.pa_copy_blocks(
        _dev(k_pool, "k_pool"), v_pool.data_ptr(), _dev(block_mapping, "block_mapping", torch.int64), P, Hkv, D, bs,
        NB, _kv_dtype(k_pool), _stream(stream)))


def _addr(t: torch.Tensor, name: str, dtype=None) -> int:
    """Pointer of a CUDA tensor or of a pinned host tensor (device-addressable)."""
    if not isinstance(t, torch.Tensor) or not (t.is_cuda or t.is_pinned()):
        raise TypeError(f"{name} must be a CUDA tensor or a pinned host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def pa_swap_blocks(src_k, src_v, dst_k, dst_v, block_mapping, stream=None) -> None:
    """dst block m[p][1] := src block m[p][0] (K and V); pools on the device or
    in pinned host memory, block_mapping likewise."""
    sNB, Hkv, bs, D = src_k.shape
    dNB = dst_k.shape[0]
    if tuple(dst_k.shape[1:]) != (Hkv, bs, D) or src_v.shape != src_k.shape or dst_v.shape != dst_k.shape:
        raise ValueError("pool shapes disagree")
    for t, n in ((src_v, "src_v"), (dst_k, "dst_k"), (dst_v, "dst_v")):
        _addr(t, n, src_k.dtype)
    _check("pa_swap_blocks", _lib.pa_swap_blocks(
        _addr(src_k, "src_k"), src_v.data_ptr(), dst_k.data_ptr(), dst_v.data_ptr(),
        _addr(block_mapping, "block_mapping", torch.int64), block_mapping.numel() // 2, Hkv, D, bs, sNB, dNB,
        _kv_dtype(src_k), _stream(stream)))


def pa_paged_attention_partition_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                      block_size) -> int:
    out = _I(0)
    _check("pa_paged_attention_partition_size", _lib.pa_paged_attention_partition_size(
        batch, num_q_heads, num_kv_heads, head_dim, max_context_len, block_size, ctypes.byref(out)))
    return out.value


def pa_paged_attention_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, block_size,
                                      partition_size: int = 0) -> int:
    out = _SZ(0)
    _check("pa_paged_attention_workspace_size", _lib.pa_paged_attention_workspace_size(
        batch, num_q_heads, num_kv_heads, head_dim, max_context_len, block_size, partition_size, ctypes.byref(out)))
    return out.value


def _workspace(workspace, nbytes: int, device, stream) -> tuple[int, int]:
    """Device pointer and size of the split-KV scratch.

    If the caller gives none, one is taken from torch's caching allocator and
    tied to the stream the kernels run on, so it is not reused before they
    finish.  Callers that launch on a raw stream handle should pass their own.
    """
    if workspace is None:
        if nbytes == 0:
            return 0, 0
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        if isinstance(stream, torch.cuda.Stream):
            workspace.record_stream(stream)
    _dev(workspace, "workspace")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def pa_paged_attention_decode(q, k_pool, v_pool, block_tables, context_lens, max_context_len: int, scale: float,
                              out, partition_size: int = 0, workspace=None, stream=None) -> None:
    """out[b, h] = softmax(scale * q[b, h] . K_b^T) V_b over the paged cache."""
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or v_pool.shape != k_pool.shape or tuple(out.shape) != (B, Hq, D):
        raise ValueError("q / pool / out shapes disagree")
    MBS = block_tables.shape[1]
    dt = _kv_dtype(q)
    _dev(k_pool, "k_pool", q.dtype)
    _dev(v_pool, "v_pool", q.dtype)
    need = pa_paged_attention_workspace_size(B, Hq, Hkv, D, max_context_len, bs, partition_size)
    ws, ws_bytes = _workspace(workspace, need, q.device, stream)
    _check("pa_paged_attention_decode", _lib.pa_paged_attention_decode(
        _dev(q, "q"), k_pool.data_ptr(), v_pool.data_ptr(), _dev(block_tables, "block_tables", torch.int32), MBS,
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len), float(scale), bs, _dev(out, "out"),
        _kv_dtype(out), B, Hq, Hkv, D, NB, dt, partition_size, ws, ws_bytes, _stream(stream)))


def pa_paged_attention_decode_append(q, key, value, k_pool, v_pool, block_tables, context_lens, max_context_len: int,
                                     scale: float, out, partition_size: int = 0, workspace=None, slot_mapping=None,
                                     stream=None) -> None:
    """One decode step: write each sequence's new token (position
    context_lens[b] - 1) into the pool, then attend over the lengths that
    include it."""
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or v_pool.shape != k_pool.shape or tuple(out.shape) != (B, Hq, D):
        raise ValueError("q / pool / out shapes disagree")
    if tuple(key.shape) != (B, Hkv, D) or value.shape != key.shape:
        raise ValueError("key / value must be [batch, num_kv_heads, head_dim]")
    MBS = block_tables.shape[1]
    dt = _kv_dtype(q)
    for t, n in ((key, "key"), (value, "value"), (k_pool, "k_pool"), (v_pool, "v_pool")):
        _dev(t, n, q.dtype)
    need = pa_paged_attention_workspace_size(B, Hq, Hkv, D, max_context_len, bs, partition_size)
    ws, ws_bytes = _workspace(workspace, need, q.device, stream)
    slots = _dev(slot_mapping, "slot_mapping", torch.int64) if slot_mapping is not None else None
    _check("pa_paged_attention_decode_append", _lib.pa_paged_attention_decode_append(
        _dev(q, "q"), key.data_ptr(), value.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(),
        _dev(block_tables, "block_tables", torch.int32), MBS, _dev(context_lens, "context_lens", torch.int32),
        int(max_context_len), float(scale), bs, _dev(out, "out"), _kv_dtype(out), B, Hq, Hkv, D, NB, dt,
        partition_size, ws, ws_bytes, slots, _stream(stream)))


def pa_paged_attention_shared_prefix_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                                    block_size, num_groups, max_group_size, max_prefix_len,
                                                    partition_size=0) -> int:
    n = ctypes.c_size_t(0)
    _check("pa_paged_attention_shared_prefix_workspace_size", _lib.pa_paged_attention_shared_prefix_workspace_size(
        batch, num_q_heads, num_kv_heads, head_dim, int(max_context_len), block_size, num_groups, max_group_size,
        int(max_prefix_len), partition_size, ctypes.byref(n)))
    return n.value


def pa_paged_attention_decode_shared_prefix(q, k_pool, v_pool, block_tables, context_lens, max_context_len: int,
                                            scale: float, out, group_starts, group_prefix_lens, max_prefix_len: int,
                                            max_group_size: int, partition_size: int = 0, workspace=None,
                                            stream=None) -> None:
    """Decode attention for groups of consecutive sequences that share their
    first group_prefix_lens[g] tokens (whole blocks, equal table entries):
    sequences group_starts[g] .. group_starts[g + 1] - 1 form group g
    (int32 device tensors of num_groups + 1 and num_groups entries)."""
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or v_pool.shape != k_pool.shape or tuple(out.shape) != (B, Hq, D):
        raise ValueError("q / pool / out shapes disagree")
    G = group_prefix_lens.numel()
    if group_starts.numel() != G + 1:
        raise ValueError("group_starts needs num_groups + 1 entries")
    dt = _kv_dtype(q)
    _dev(k_pool, "k_pool", q.dtype)
    _dev(v_pool, "v_pool", q.dtype)
    need = pa_paged_attention_shared_prefix_workspace_size(B, Hq, Hkv, D, max_context_len, bs, G, max_group_size,
                                                           max_prefix_len, partition_size)
    ws, ws_bytes = _workspace(workspace, need, q.device, stream)
    _check("pa_paged_attention_decode_shared_prefix", _lib.pa_paged_attention_decode_shared_prefix(
        _dev(q, "q"), k_pool.data_ptr(), v_pool.data_ptr(), _dev(block_tables, "block_tables", torch.int32),
        block_tables.shape[1], _dev(context_lens, "context_lens", torch.int32), int(max_context_len), float(scale), bs,
        _dev(out, "out"), _kv_dtype(out), B, Hq, Hkv, D, NB, dt, _dev(group_starts, "group_starts", torch.int32),
        _dev(group_prefix_lens, "group_prefix_lens", torch.int32), G, int(max_group_size), int(max_prefix_len),
        partition_size, ws, ws_bytes, _stream(stream)))


def pa_paged_attention_decode_contiguous(q, k_c, v_c, context_lens, max_context_len: int, scale: float, out,
                                         block_size: int = 16, partition_size: int = 0, workspace=None,
                                         stream=None) -> None:
    """The same attention over a contiguous cache k_c, v_c: [B, Hkv, L_pad, D]."""
    B, Hq, D = q.shape
    B2, Hkv, L_pad, D2 = k_c.shape
    if B2 != B or D2 != D or v_c.shape != k_c.shape or tuple(out.shape) != (B, Hq, D):
        raise ValueError("q / cache / out shapes disagree")
    dt = _kv_dtype(q)
    _dev(k_c, "k_c", q.dtype)
    _dev(v_c, "v_c", q.dtype)
    need = pa_paged_attention_workspace_size(B, Hq, Hkv, D, max_context_len, block_size, partition_size)
    ws, ws_bytes = _workspace(workspace, need, q.device, stream)
    _check("pa_paged_attention_decode_contiguous", _lib.pa_paged_attention_decode_contiguous(
        _dev(q, "q"), k_c.data_ptr(), v_c.data_ptr(), L_pad, _dev(context_lens, "context_lens", torch.int32),
        int(max_context_len), float(scale), block_size, _dev(out, "out"), _kv_dtype(out), B, Hq, Hkv, D, dt,
        partition_size, ws, ws_bytes, _stream(stream)))


STATIC_SCRATCH_BYTES = 16 << 20  # PA_STATIC_SCRATCH_BYTES in include/pa.h


def pa_paged_attention_decode_static_scratch(q, k_pool, v_pool, block_tables, context_lens, max_context_len: int,
                                             scale: float, out, partition_size: int = 0, stream=None) -> None:
    """pa_paged_attention_decode without a workspace argument, for callers
    that cannot allocate device memory: the split-KV scratch is a fixed array
    of STATIC_SCRATCH_BYTES inside libpa, shared by all calls (calls that
    overlap on the GPU race on it).  Raises PAError(PA_ERR_WORKSPACE) when the
    sizes need more scratch than that.  The first call on a device looks up the
    array's address and should come before any stream capture."""
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or v_pool.shape != k_pool.shape or tuple(out.shape) != (B, Hq, D):
        raise ValueError("q / pool / out shapes disagree")
    MBS = block_tables.shape[1]
    dt = _kv_dtype(q)
    _dev(k_pool, "k_pool", q.dtype)
    _dev(v_pool, "v_pool", q.dtype)
    _check("pa_paged_attention_decode_static_scratch", _lib.pa_paged_attention_decode_static_scratch(
        _dev(q, "q"), k_pool.data_ptr(), v_pool.data_ptr(), _dev(block_tables, "block_tables", torch.int32), MBS,
        _dev(context_lens, "context_lens", torch.int32), int(max_context_len), float(scale), bs, _dev(out, "out"),
        _kv_dtype(out), B, Hq, Hkv, D, NB, dt, partition_size, _stream(stream)))


def pa_paged_attention_prefill(q, k_pool, v_pool, block_tables, context_lens, query_start, max_query_len: int,
                               scale: float, out, stream=None) -> None:
    """Causal multi-query attention: q rows query_start[b]..query_start[b+1]-1
    are the last tokens of sequence b (lengths context_lens, counting them)."""
    T, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    if D2 != D or v_pool.shape != k_pool.shape or tuple(out.shape) != (T, Hq, D):
        raise ValueError("q / pool / out shapes disagree")
    B = context_lens.numel()
    if query_start.numel() != B + 1:
        raise ValueError("query_start needs batch + 1 entries")
    _dev(k_pool, "k_pool", q.dtype)
    _dev(v_pool, "v_pool", q.dtype)
    _check("pa_paged_attention_prefill", _lib.pa_paged_attention_prefill(
        _dev(q, "q"), k_pool.data_ptr(), v_pool.data_ptr(), _dev(block_tables, "block_tables", torch.int32),
        block_tables.shape[1], _dev(context_lens, "context_lens", torch.int32),
        _dev(query_start, "query_start", torch.int32), int(max_query_len), float(scale), bs, _dev(out, "out"),
        _kv_dtype(out), B, Hq, Hkv, D, T, NB, _kv_dtype(q), _stream(stream)))
