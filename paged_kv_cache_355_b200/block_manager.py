"""Python handle on libpa's native (C++) KV block manager.

Argument marshalling only (numpy host arrays in and out); the allocator
itself -- FIFO free list, per-sequence block tables, reference counts,
fork and copy-on-write -- is pa_bm_* in libpa (see include/pa.h).
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _binding

_lib = _binding._lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class OutOfBlocks(RuntimeError):
    pass


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int):
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        self._h = _lib.pa_bm_create(self.num_blocks, self.block_size)
        if not self._h:
            raise ValueError("pa_bm_create rejected its sizes")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            _lib.pa_bm_destroy(h)
            self._h = None

    def _check(self, fn, rc):
        if rc == 3:
            raise OutOfBlocks("no free KV block left")
        if rc != 0:
            raise _binding.PAError(fn, rc)

    def add_sequence(self, seq: int) -> None:
        self._check("pa_bm_add_sequence", _lib.pa_bm_add_sequence(self._h, int(seq)))

    def append_tokens(self, seq_ids):
        """Append one token per entry; returns (slots int64 [n], cow pairs int64 [k, 2])."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, np.int64))
        n = ids.shape[0]
        slots = np.empty(n, np.int64)
        pairs = np.empty((max(n, 1), 2), np.int64)
        k = ctypes.c_int64(0)
        rc = _lib.pa_bm_append_tokens(self._h, _p(ids), n, _p(slots), _p(pairs), ctypes.byref(k))
        self._check("pa_bm_append_tokens", rc)
        return slots, pairs[: k.value].copy()

    def append_token(self, seq: int):
        slots, pairs = self.append_tokens([seq])
        return int(slots[0]), [tuple(int(x) for x in p) for p in pairs]

    def fork(self, parent: int, child: int) -> None:
        self._check("pa_bm_fork", _lib.pa_bm_fork(self._h, int(parent), int(child)))

    def free_sequence(self, seq: int) -> None:
        self._check("pa_bm_free_sequence", _lib.pa_bm_free_sequence(self._h, int(seq)))

    def num_free(self) -> int:
        return int(_lib.pa_bm_num_free(self._h))

    def refcount(self, block: int) -> int:
        return int(_lib.pa_bm_refcount(self._h, int(block)))

    def length(self, seq: int) -> int:
        return int(_lib.pa_bm_length(self._h, int(seq)))

    def block_tables(self, seq_ids, max_blocks_per_seq: int):
        """(int32 [n, max_blocks_per_seq] tables padded with -1, int32 [n] lengths)."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, np.int64))
        tables = np.empty((ids.shape[0], max_blocks_per_seq), np.int32)
        lens = np.empty(ids.shape[0], np.int32)
        self._check("pa_bm_block_tables", _lib.pa_bm_block_tables(self._h, _p(ids), ids.shape[0],
                                                                  max_blocks_per_seq, _p(tables), _p(lens)))
        return tables, lens

    def block_table(self, seq: int) -> list[int]:
        n = -(-self.length(seq) // self.block_size)
        t, _ = self.block_tables([seq], max(n, 1))
        return [int(x) for x in t[0] if x >= 0]

    def free_list(self) -> list[int]:
        n = ctypes.c_int64(0)
        out = np.empty(self.num_blocks, np.int64)
        self._check("pa_bm_free_list", _lib.pa_bm_free_list(self._h, _p(out), self.num_blocks, ctypes.byref(n)))
        return out[: n.value].tolist()

    def shared_prefix_groups(self, seq_ids):
        """(group_starts int32 [G + 1], prefix_lens int32 [G], max_group_size,
        max_prefix_len) of a batch in the order given: the inputs of
        pa_paged_attention_decode_shared_prefix (copy the two arrays to the
        device)."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, np.int64))
        n = ids.shape[0]
        starts = np.empty(n + 1, np.int32)
        plens = np.empty(max(n, 1), np.int32)
        ng, mg, mp = ctypes.c_int64(0), ctypes.c_int32(0), ctypes.c_int32(0)
        self._check("pa_bm_shared_prefix_groups", _lib.pa_bm_shared_prefix_groups(
            self._h, _p(ids), n, _p(starts), _p(plens), ctypes.byref(ng), ctypes.byref(mg), ctypes.byref(mp)))
        g = ng.value
        return starts[: g + 1].copy(), plens[:g].copy(), int(mg.value), int(mp.value)
