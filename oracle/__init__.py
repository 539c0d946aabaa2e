"""CPU oracle for the paged KV-cache decode path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product package
``paged_kv_cache_355_b200`` never does, and shares no code with it.

The arithmetic lives in ``pa_oracle.c`` (plain C, fp64 accumulation, OpenMP
across independent rows); this module only marshals numpy arrays into it.
``brute.py`` is an independent pure-Python check of the same definition that
never builds a block pool, and ``block_manager.py`` is the host-side model of
the pages' allocator (free list, block tables, reference counts,
copy-on-write).

Data conventions (the pages fix none of them):
  * k_pool, v_pool: [num_blocks, Hkv, block_size, D], fp32 (numpy float32)
    or bf16 passed as raw 16-bit words (numpy uint16);
  * q: [B, Hq, D] with the same element type; block_tables int32 [B, MBS];
    context_lens int32 [B]; query head h reads kv head h // (Hq // Hkv).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = [
            "gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
            "-shared", "-std=c11", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm",
        ]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # PA_ORACLE_LIB lets the mutation tests load a deliberately broken
            # build of pa_oracle.c; normally the library next to this file is used.
            override = os.environ.get("PA_ORACLE_LIB")
            lib = ctypes.CDLL(override if override else build())
            P = ctypes.c_void_p
            i32, i64, f32 = ctypes.c_int, ctypes.c_int64, ctypes.c_float
            lib.oracle_paged_decode.argtypes = [P, P, P, P, i32, P, f32, i32, i32, i32, i32, i32, i64, i32, P]
            lib.oracle_paged_decode_rows.argtypes = [P, P, P, P, i32, P, f32, i32, i32, i32, i32, i32, i64, i32, P, P, i64, P]
            lib.oracle_contiguous_decode.argtypes = [P, P, P, i32, P, f32, i32, i32, i32, i32, i32, P]
            lib.oracle_paged_prefill.argtypes = [P, P, P, P, i32, P, P, f32, i32, i32, i32, i32, i32, i64, i32, P]
            lib.oracle_slot_mapping.argtypes = [P, i32, i32, P, P, i64, i32, P]
            lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32]
            lib.oracle_copy_blocks.argtypes = [P, P, P, i64, i32, i32, i32, i64, i32]
            lib.oracle_round_bf16.argtypes = [P, i64, P]
            lib.oracle_round_bf16.restype = None
            lib.oracle_num_threads.argtypes = []
            for name in ("oracle_paged_decode", "oracle_paged_decode_rows", "oracle_contiguous_decode",
                         "oracle_paged_prefill",
                         "oracle_slot_mapping", "oracle_reshape_and_cache", "oracle_copy_blocks",
                         "oracle_num_threads"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS, else all cores)."""
    return int(_load().oracle_num_threads())


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle takes float32 or bf16-as-uint16 arrays, got {a.dtype}")


def _c(a: np.ndarray, dtype=None) -> np.ndarray:
    a = np.asarray(a)
    return np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def paged_decode(q, k_pool, v_pool, block_tables, context_lens, scale, block_size):
    """All rows of paged decode attention, float64 [B, Hq, D]."""
    q, k_pool, v_pool = _c(q), _c(k_pool), _c(v_pool)
    bt, lens = _c(block_tables, np.int32), _c(context_lens, np.int32)
    dt = _dtype_code(q)
    assert _dtype_code(k_pool) == dt and _dtype_code(v_pool) == dt
    B, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_pool.shape
    assert D2 == D and bs == block_size and v_pool.shape == k_pool.shape
    out = np.zeros((B, Hq, D), np.float64)
    rc = _load().oracle_paged_decode(_ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(bt), bt.shape[1] if bt.ndim == 2 else 0,
                                     _ptr(lens), float(np.float32(scale)), block_size, B, Hq, Hkv, D, NB, dt, _ptr(out))
    if rc:
        raise ValueError("oracle_paged_decode rejected its arguments")
    return out


def paged_decode_rows(q, k_pool, v_pool, block_tables, context_lens, scale, block_size, rows_b, rows_h):
    """Selected rows (rows_b[i], rows_h[i]) of paged decode attention, float64 [n, D]."""
    q, k_pool, v_pool = _c(q), _c(k_pool), _c(v_pool)
    bt, lens = _c(block_tables, np.int32), _c(context_lens, np.int32)
    rb, rh = _c(rows_b, np.int32), _c(rows_h, np.int32)
    dt = _dtype_code(q)
    B, Hq, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    assert bs == block_size
    out = np.zeros((rb.shape[0], D), np.float64)
    rc = _load().oracle_paged_decode_rows(_ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(bt), bt.shape[1],
                                          _ptr(lens), float(np.float32(scale)), block_size, B, Hq, Hkv, D, NB, dt,
                                          _ptr(rb), _ptr(rh), rb.shape[0], _ptr(out))
    if rc:
        raise ValueError("oracle_paged_decode_rows rejected its arguments")
    return out


def paged_prefill(q, k_pool, v_pool, block_tables, context_lens, query_start, scale, block_size):
    """Causal multi-query attention, float64 [T, Hq, D]; sequence b owns query
    rows query_start[b] .. query_start[b + 1] - 1, its last tokens."""
    q, k_pool, v_pool = _c(q), _c(k_pool), _c(v_pool)
    bt, lens, qs = _c(block_tables, np.int32), _c(context_lens, np.int32), _c(query_start, np.int32)
    dt = _dtype_code(q)
    T, Hq, D = q.shape
    NB, Hkv, bs, _ = k_pool.shape
    assert bs == block_size and qs.shape[0] == lens.shape[0] + 1 and qs[-1] == T
    out = np.zeros((T, Hq, D), np.float64)
    rc = _load().oracle_paged_prefill(_ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(bt), bt.shape[1], _ptr(lens), _ptr(qs),
                                      float(np.float32(scale)), block_size, lens.shape[0], Hq, Hkv, D, NB, dt, _ptr(out))
    if rc:
        raise ValueError("oracle_paged_prefill rejected its arguments")
    return out


def contiguous_decode(q, k_c, v_c, context_lens, scale):
    """Decode attention over a contiguous cache k_c, v_c: [B, Hkv, L_pad, D]."""
    q, k_c, v_c = _c(q), _c(k_c), _c(v_c)
    lens = _c(context_lens, np.int32)
    dt = _dtype_code(q)
    B, Hq, D = q.shape
    _, Hkv, L_pad, _ = k_c.shape
    out = np.zeros((B, Hq, D), np.float64)
    rc = _load().oracle_contiguous_decode(_ptr(q), _ptr(k_c), _ptr(v_c), L_pad, _ptr(lens), float(np.float32(scale)),
                                          B, Hq, Hkv, D, dt, _ptr(out))
    if rc:
        raise ValueError("oracle_contiguous_decode rejected its arguments")
    return out


def slot_mapping(block_tables, seq_ids, positions, block_size):
    """int64 slot of each (sequence, position) token."""
    bt = _c(block_tables, np.int32)
    sid, pos = _c(seq_ids, np.int32), _c(positions, np.int32)
    slots = np.zeros(sid.shape[0], np.int64)
    rc = _load().oracle_slot_mapping(_ptr(bt), bt.shape[1], bt.shape[0], _ptr(sid), _ptr(pos), sid.shape[0],
                                     block_size, _ptr(slots))
    if rc:
        raise ValueError("oracle_slot_mapping rejected its arguments")
    return slots


def reshape_and_cache(key, value, k_pool, v_pool, slots):
    """Write key/value [T, Hkv, D] into the pools in place; slot < 0 skips."""
    key, value = _c(key), _c(value)
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    sl = _c(slots, np.int64)
    dt = _dtype_code(key)
    NB, Hkv, bs, D = k_pool.shape
    rc = _load().oracle_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_pool), _ptr(v_pool), _ptr(sl),
                                          sl.shape[0], Hkv, D, bs, NB, dt)
    if rc:
        raise ValueError("oracle_reshape_and_cache rejected its arguments")


def copy_blocks(k_pool, v_pool, block_mapping):
    """For each (src, dst) pair in order, duplicate block src into block dst."""
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    bm = _c(np.asarray(block_mapping).reshape(-1, 2), np.int64)
    dt = _dtype_code(k_pool)
    NB, Hkv, bs, D = k_pool.shape
    rc = _load().oracle_copy_blocks(_ptr(k_pool), _ptr(v_pool), _ptr(bm), bm.shape[0], Hkv, D, bs, NB, dt)
    if rc:
        raise ValueError("oracle_copy_blocks rejected its arguments")


def round_bf16(x) -> np.ndarray:
    """Round float64 values once to bfloat16; returns the uint16 bit patterns."""
    x = _c(np.asarray(x, np.float64))
    out = np.zeros(x.shape, np.uint16)
    _load().oracle_round_bf16(_ptr(x), x.size, _ptr(out))
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    bits = np.asarray(bits, np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
