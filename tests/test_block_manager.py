"""Pins for the host block manager (free list, tables, refcounts, CoW)."""
from __future__ import annotations

import json
import os

import pytest

from oracle.block_manager import BlockManager, OutOfBlocks

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_toy_allocator_trace():
    g = json.load(open(os.path.join(GOLDEN, "toy_allocator_trace.json")))
    bs = g["block_size"]
    bm = BlockManager(g["total_blocks"], bs)
    for seq, first, last, expected_block in g["segments"]:
        for length in range(first, last + 1):
            assert bm.lengths.get(seq, 0) == length - 1
            bm.append_token(seq)
            assert bm.block_table(seq)[-1] == expected_block, (seq, length)
    for seq, table in g["final_tables"].items():
        assert bm.block_table(seq) == table
    assert bm.free[0] == g["final_free_head"]


def test_block_size_one_takes_a_block_per_token():
    bm = BlockManager(10, 1)
    for _ in range(4):
        bm.append_token("s")
    assert bm.block_table("s") == [0, 1, 2, 3]
    assert [bm.slot("s", p) for p in range(4)] == [0, 1, 2, 3]


def test_waste_is_below_one_block_per_sequence():
    bm = BlockManager(1000, 16)
    lengths = {"a": 1, "b": 16, "c": 17, "d": 100}
    for s, n in lengths.items():
        for _ in range(n):
            bm.append_token(s)
    for s, n in lengths.items():
        reserved = len(bm.block_table(s)) * 16
        assert 0 <= reserved - n <= 15


def test_fork_shares_blocks_and_cow_on_first_write():
    bs = 4
    bm = BlockManager(20, bs)
    for _ in range(6):  # one full block + a partial one
        bm.append_token("p")
    for i in range(3):
        bm.fork("p", f"c{i}")
    shared = bm.block_table("p")
    assert all(bm.refcount[b] == 4 for b in shared)
    slot, pairs = bm.append_token("c0")
    assert len(pairs) == 1 and pairs[0][0] == shared[1]
    new = pairs[0][1]
    assert bm.block_table("c0") == [shared[0], new]
    assert slot == new * bs + 2
    assert bm.refcount[shared[1]] == 3 and bm.refcount[new] == 1
    # the others still point at the original partial block
    for s in ("p", "c1", "c2"):
        assert bm.block_table(s) == shared


def test_last_sharer_writes_in_place():
    bm = BlockManager(10, 4)
    for _ in range(3):
        bm.append_token("p")
    bm.fork("p", "c")
    blk = bm.block_table("p")[0]
    _, pairs = bm.append_token("c")
    assert pairs and bm.refcount[blk] == 1
    _, pairs = bm.append_token("p")
    assert pairs == [] and bm.block_table("p") == [blk]


def test_free_returns_blocks_when_count_drops_to_zero():
    bm = BlockManager(8, 2)
    for _ in range(4):
        bm.append_token("p")
    bm.fork("p", "c")
    assert bm.num_free() == 6
    bm.free_sequence("p")
    assert bm.num_free() == 6
    bm.free_sequence("c")
    assert bm.num_free() == 8
    assert list(bm.free)[-2:] == [0, 1]


def test_running_out_of_blocks_raises():
    bm = BlockManager(2, 2)
    for _ in range(4):
        bm.append_token("a")
    with pytest.raises(OutOfBlocks):
        bm.append_token("a")


def test_parallel_sampling_without_sharing_costs_n_times_the_prefix():
    # n = 8 samples of a 1000-token prompt: shared prefix blocks vs private copies
    bs, n, prompt = 16, 8, 1000
    bm = BlockManager(4000, bs)
    for _ in range(prompt):
        bm.append_token(0)
    for i in range(1, n):
        bm.fork(0, i)
    used_shared = 4000 - bm.num_free()
    private = BlockManager(4000, bs)
    for i in range(n):
        for _ in range(prompt):
            private.append_token(i)
    used_private = 4000 - private.num_free()
    assert used_private == n * used_shared
