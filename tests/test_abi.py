"""The C ABI without a GPU: the library loads, exports every entry point that
include/pa.h declares, and rejects bad arguments on the host before any
launch (these calls never reach the CUDA runtime)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3


def declared_entry_points(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_355_b200 import build

    path = build.build()
    return ctypes.CDLL(path)


def test_every_declared_symbol_is_exported(lib):
    names = declared_entry_points()
    assert len(names) >= 10
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_timeline_build_exports_the_same_abi_and_its_readers(lib):
    """libpa_timeline.so (the decode and prefill kernels with per-CTA stamps)
    exports everything include/pa.h declares plus include/pa_timeline.h's
    readers; libpa.so has none of the readers."""
    from paged_kv_cache_355_b200 import build

    tl = ctypes.CDLL(build.TIMELINE_LIB)
    readers = declared_entry_points(os.path.join(ROOT, "include", "pa_timeline.h"))
    assert sorted(readers) == ["pa_timeline_clear", "pa_timeline_clear_prefill", "pa_timeline_read",
                               "pa_timeline_read_prefill"]
    missing = [n for n in declared_entry_points() + readers if not hasattr(tl, n)]
    assert not missing, missing
    assert not any(hasattr(lib, n) for n in readers)


def test_binding_wraps_every_declared_symbol(lib):
    import paged_kv_cache_355_b200 as pa
    from paged_kv_cache_355_b200 import block_manager

    assert sorted(pa.EXPORTED) == declared_entry_points()
    for name in declared_entry_points():
        if name.startswith("pa_bm_"):
            # the host block manager is wrapped as a class over its handle
            assert callable(getattr(block_manager.BlockManager, name[len("pa_bm_"):], None)) or name in (
                "pa_bm_create", "pa_bm_destroy", "pa_bm_append_tokens", "pa_bm_block_tables", "pa_bm_free_list")
        else:
            assert callable(getattr(pa, name))


def test_status_strings(lib):
    lib.pa_status_string.restype = ctypes.c_char_p
    names = [lib.pa_status_string(i).decode() for i in range(7)]
    assert names == ["PA_OK", "PA_ERR_INVALID_ARG", "PA_ERR_UNSUPPORTED", "PA_ERR_WORKSPACE", "PA_ERR_CUDA",
                     "PA_ERR_BAD_BLOCK_ID", "PA_ERR_TIMEOUT"]
    assert lib.pa_status_string(99).decode() == "PA_ERR_UNKNOWN"


def _decode(lib, **kw):
    args = dict(q=16, k=16, v=16, bt=16, mbs=8, lens=16, maxlen=100, scale=0.1, bs=16, out=16, out_dtype=0,
                batch=2, hq=8, hkv=2, d=128, nb=10, kv_dtype=1, part=0, ws=0, ws_bytes=0, stream=None)
    args.update(kw)
    P = ctypes.c_void_p
    return lib.pa_paged_attention_decode(
        P(args["q"]), P(args["k"]), P(args["v"]), P(args["bt"]), args["mbs"], P(args["lens"]), args["maxlen"],
        ctypes.c_float(args["scale"]), args["bs"], P(args["out"]), args["out_dtype"], args["batch"], args["hq"],
        args["hkv"], args["d"], ctypes.c_int64(args["nb"]), args["kv_dtype"], args["part"], P(args["ws"]),
        ctypes.c_size_t(args["ws_bytes"]), P(args["stream"]))


def test_decode_rejects_bad_shapes(lib):
    assert _decode(lib, hq=6, hkv=4) == INVALID            # Hq % Hkv != 0
    assert _decode(lib, hq=64, hkv=2) == UNSUPPORTED       # group of 32
    assert _decode(lib, hq=32, hkv=2, kv_dtype=0) == UNSUPPORTED  # group of 16 needs bf16
    assert _decode(lib, d=96) == UNSUPPORTED
    assert _decode(lib, bs=64) == UNSUPPORTED
    assert _decode(lib, kv_dtype=7) == INVALID
    assert _decode(lib, out_dtype=3) == INVALID
    assert _decode(lib, maxlen=8 * 16 + 1) == INVALID      # longer than the table can map
    assert _decode(lib, q=0) == INVALID
    assert _decode(lib, bt=0) == INVALID
    assert _decode(lib, k=24) == INVALID                   # not 16-byte aligned
    assert _decode(lib, part=48) == INVALID                # not a multiple of 32
    assert _decode(lib, part=16384) == INVALID             # above 8192
    assert _decode(lib, batch=-1) == INVALID
    assert _decode(lib, batch=0, q=0, k=0, v=0) == OK      # nothing to do, nothing launched


def test_decode_requires_workspace_for_splits(lib):
    # 100 tokens cut into 32-token splits need scratch for the partial results
    assert _decode(lib, part=32) == WORKSPACE
    assert _decode(lib, part=32, ws=16, ws_bytes=64) == WORKSPACE


def test_workspace_size(lib):
    sz = ctypes.c_size_t(0)
    assert lib.pa_paged_attention_workspace_size(4, 8, 2, 128, 100, 16, 32, ctypes.byref(sz)) == OK
    rows = 4 * 8 * 4  # batch * Hq * ceil(100 / 32)
    expect = -(-rows * 128 * 4 // 256) * 256 + -(-rows * 2 * 4 // 256) * 256
    assert sz.value == expect
    assert lib.pa_paged_attention_workspace_size(4, 8, 2, 128, 100, 16, 128, ctypes.byref(sz)) == OK
    assert sz.value == 0
    assert lib.pa_paged_attention_workspace_size(4, 8, 2, 128, 100, 16, 33, ctypes.byref(sz)) == INVALID
    part = ctypes.c_int(0)
    assert lib.pa_paged_attention_partition_size(64, 32, 32, 128, 2048, 16, ctypes.byref(part)) == OK
    assert part.value % 32 == 0 and 256 <= part.value <= 8192


def test_cache_kernels_reject_bad_arguments(lib):
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    assert lib.pa_reshape_and_cache(P(16), P(16), P(16), P(16), P(16), I64(4), 2, 96, 16, I64(8), 1, None) == UNSUPPORTED
    assert lib.pa_reshape_and_cache(P(16), P(16), P(16), P(16), P(16), I64(4), 2, 128, 12, I64(8), 1, None) == UNSUPPORTED
    assert lib.pa_reshape_and_cache(P(0), P(16), P(16), P(16), P(16), I64(4), 2, 128, 16, I64(8), 1, None) == INVALID
    assert lib.pa_reshape_and_cache(P(16), P(16), P(16), P(16), P(16), I64(-1), 2, 128, 16, I64(8), 1, None) == INVALID
    assert lib.pa_reshape_and_cache(P(0), P(0), P(0), P(0), P(0), I64(0), 2, 128, 16, I64(8), 1, None) == OK
    assert lib.pa_copy_blocks(P(16), P(16), P(0), I64(3), 2, 128, 16, I64(8), 1, None) == INVALID
    assert lib.pa_copy_blocks(P(16), P(16), P(16), I64(3), 2, 128, 16, I64(8), 5, None) == INVALID
    assert lib.pa_copy_blocks(P(0), P(0), P(0), I64(0), 2, 128, 16, I64(8), 1, None) == OK
    assert lib.pa_slot_mapping(P(0), 4, 2, P(16), P(16), I64(3), 16, P(16), None) == INVALID
    assert lib.pa_slot_mapping(P(16), 4, 2, P(16), P(16), I64(3), 0, P(16), None) == INVALID
    assert lib.pa_decode_slot_mapping(P(16), 4, P(0), 2, 16, P(16), None) == INVALID


def test_selftest_rejects_bad_limits(lib):
    assert lib.pa_selftest_wait_timeout(0, None) == INVALID
    assert lib.pa_selftest_wait_timeout(2_000_001, None) == INVALID


def test_static_scratch_size_constant_matches_the_header():
    """The binding's STATIC_SCRATCH_BYTES is the header's PA_STATIC_SCRATCH_BYTES."""
    text = open(HEADER).read()
    m = re.search(r"#define\s+PA_STATIC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m, "PA_STATIC_SCRATCH_BYTES not found in include/pa.h"
    import paged_kv_cache_355_b200 as pa

    assert pa.STATIC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_read_probe_rejects_bad_arguments(lib):
    P = ctypes.c_void_p
    lib.pa_hbm_read_probe.argtypes = [P, ctypes.c_size_t, P]
    assert lib.pa_hbm_read_probe(P(16), 17, None) == INVALID   # not a multiple of 16 bytes
    assert lib.pa_hbm_read_probe(P(24), 16, None) == INVALID   # not 16-byte aligned
    assert lib.pa_hbm_read_probe(P(0), 16, None) == INVALID
    assert lib.pa_hbm_read_probe(P(16), 0, None) == OK         # nothing to read, nothing launched


def _shared(lib, **kw):
    args = dict(q=16, k=16, v=16, bt=16, mbs=8, lens=16, maxlen=100, scale=0.1, bs=16, out=16, out_dtype=0,
                batch=4, hq=8, hkv=2, d=128, nb=10, kv_dtype=1, gs=16, gl=16, ng=2, mg=2, mp=32, part=0, ws=0,
                ws_bytes=0, stream=None)
    args.update(kw)
    P = ctypes.c_void_p
    return lib.pa_paged_attention_decode_shared_prefix(
        P(args["q"]), P(args["k"]), P(args["v"]), P(args["bt"]), args["mbs"], P(args["lens"]), args["maxlen"],
        ctypes.c_float(args["scale"]), args["bs"], P(args["out"]), args["out_dtype"], args["batch"], args["hq"],
        args["hkv"], args["d"], ctypes.c_int64(args["nb"]), args["kv_dtype"], P(args["gs"]), P(args["gl"]),
        args["ng"], args["mg"], args["mp"], args["part"], P(args["ws"]), ctypes.c_size_t(args["ws_bytes"]),
        P(args["stream"]))


def test_shared_prefix_rejects_bad_arguments(lib):
    assert _shared(lib, kv_dtype=0) == UNSUPPORTED        # bf16 only
    assert _shared(lib, ng=0) == INVALID                  # no group
    assert _shared(lib, ng=5) == INVALID                  # more groups than sequences
    assert _shared(lib, mg=0) == INVALID
    assert _shared(lib, mp=101) == INVALID                # prefix bound above max_context_len
    assert _shared(lib, mp=-1) == INVALID
    assert _shared(lib, gs=0) == INVALID
    assert _shared(lib, gl=0) == INVALID
    assert _shared(lib) == WORKSPACE                      # always needs scratch (prefix lengths at least)
    assert _shared(lib, batch=0, q=0) == OK


def test_shared_prefix_workspace_size(lib):
    sz = ctypes.c_size_t(0)
    f = lib.pa_paged_attention_shared_prefix_workspace_size
    # no prefix, one suffix split: only the per-sequence prefix lengths
    assert f(4, 8, 2, 128, 100, 16, 2, 2, 0, 128, ctypes.byref(sz)) == OK
    assert sz.value == 256
    # a prefix: prefix splits + suffix splits per row, then the lengths and
    # (head_dim 128, one prefix split and one own split: the prefix pass runs
    # last) its exit counter
    assert f(4, 8, 2, 128, 100, 16, 2, 2, 64, 128, ctypes.byref(sz)) == OK
    rows = 4 * 8 * 2
    assert sz.value == -(-rows * 128 * 4 // 256) * 256 + -(-rows * 2 * 4 // 256) * 256 + 256 + 256
    # head_dim 64 keeps the prefix pass first: no counter
    assert f(4, 8, 2, 64, 100, 16, 2, 2, 64, 128, ctypes.byref(sz)) == OK
    assert sz.value == -(-rows * 64 * 4 // 256) * 256 + -(-rows * 2 * 4 // 256) * 256 + 256
    assert f(4, 8, 2, 128, 100, 16, 0, 2, 64, 128, ctypes.byref(sz)) == INVALID
    assert f(4, 8, 2, 128, 100, 16, 2, 2, 101, 128, ctypes.byref(sz)) == INVALID


def test_nvtx_ranges_leave_the_calls_unchanged(lib):
    """With PA_NVTX=1 every launching entry point opens and closes an NVTX
    range; with no profiler attached that changes nothing the caller sees."""
    import subprocess
    import sys

    code = ("import ctypes; lib = ctypes.CDLL(%r); P = ctypes.c_void_p; "
            "lib.pa_hbm_read_probe.argtypes = [P, ctypes.c_size_t, P]; "
            "print(lib.pa_hbm_read_probe(P(24), 16, None), lib.pa_hbm_read_probe(P(16), 0, None), "
            "lib.pa_copy_blocks(P(16), P(16), P(0), ctypes.c_int64(3), 2, 128, 16, ctypes.c_int64(8), 1, None))"
            % os.path.join(ROOT, "paged_kv_cache_355_b200", "libpa.so"))
    outs = []
    for flag in ("0", "1"):
        env = dict(os.environ, PA_NVTX=flag)
        outs.append(subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                                   check=True).stdout.split())
    assert outs[0] == outs[1] == [str(INVALID), str(OK), str(INVALID)]
