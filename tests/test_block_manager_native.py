"""libpa's native block manager against the oracle's host model: the same
operation sequences must give identical slots, copy-on-write pairs, block
tables, reference counts and free lists (integer work: bit-exact)."""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

from oracle.block_manager import BlockManager as RefManager
from oracle.block_manager import OutOfBlocks as RefOut

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def native():
    from paged_kv_cache_355_b200 import build

    build.build()
    from paged_kv_cache_355_b200 import block_manager

    return block_manager


def _same_state(nat, ref, seqs):
    assert nat.num_free() == len(ref.free)
    assert nat.free_list() == list(ref.free)
    for b in range(ref.num_blocks):
        assert nat.refcount(b) == ref.refcount[b]
    for s in seqs:
        if s in ref.tables:
            assert nat.block_table(s) == ref.block_table(s)
            assert nat.length(s) == ref.lengths[s]
        else:
            assert nat.length(s) == -1


@pytest.mark.parametrize("bs", [1, 2, 8, 16])
def test_random_operation_sequences_match_the_oracle(native, bs):
    rng = np.random.default_rng(bs)
    nb = 300
    nat, ref = native.BlockManager(nb, bs), RefManager(nb, bs)
    live, next_id = [0], 1
    for step in range(1500):
        op = rng.random()
        if op < 0.75 and live:
            s = int(rng.choice(live))
            try:
                want = ref.append_token(s)
            except RefOut:
                with pytest.raises(native.OutOfBlocks):
                    nat.append_token(s)
                continue
            assert nat.append_token(s) == want
        elif op < 0.85 and live:
            p = int(rng.choice(live))
            ref.fork(p, next_id)
            nat.fork(p, next_id)
            live.append(next_id)
            next_id += 1
        elif op < 0.95 and len(live) > 1:
            s = int(rng.choice(live))
            ref.free_sequence(s)
            nat.free_sequence(s)
            live.remove(s)
        else:
            ref.add_sequence(next_id)
            nat.add_sequence(next_id)
            live.append(next_id)
            next_id += 1
        if step % 100 == 0:
            _same_state(nat, ref, range(next_id))
    _same_state(nat, ref, range(next_id))


def test_batched_appends_equal_one_by_one(native):
    a, b = native.BlockManager(100, 4), native.BlockManager(100, 4)
    for m in (a, b):
        for _ in range(6):
            m.append_token(0)
        m.fork(0, 1)
        m.fork(0, 2)
    ids = [1, 2, 0, 1, 1, 3, 3, 2]
    slots, pairs = a.append_tokens(ids)
    one = [b.append_token(s) for s in ids]
    assert slots.tolist() == [s for s, _ in one]
    assert [tuple(p) for p in pairs.tolist()] == [p for _, ps in one for p in ps]


def test_toy_allocator_trace(native):
    g = json.load(open(os.path.join(GOLDEN, "toy_allocator_trace.json")))
    bm = native.BlockManager(g["total_blocks"], g["block_size"])
    names = {"a": 0, "b": 1}
    for seq, first, last, expected in g["segments"]:
        for _ in range(first, last + 1):
            bm.append_token(names[seq])
            assert bm.block_table(names[seq])[-1] == expected
    for seq, table in g["final_tables"].items():
        assert bm.block_table(names[seq]) == table
    assert bm.free_list()[0] == g["final_free_head"]


def test_dense_tables_feed_the_decode_kernel(native):
    bm = native.BlockManager(20, 4)
    for s, n in ((0, 5), (1, 9), (2, 1)):
        for _ in range(n):
            bm.append_token(s)
    tables, lens = bm.block_tables([2, 0, 1], 4)
    assert lens.tolist() == [1, 5, 9]
    assert tables.tolist() == [bm.block_table(2) + [-1] * 3, bm.block_table(0) + [-1] * 2, bm.block_table(1) + [-1]]
    with pytest.raises(Exception):
        bm.block_tables([1], 2)  # table wider than the requested width


def test_bad_arguments(native):
    with pytest.raises(ValueError):
        native.BlockManager(0, 16)
    bm = native.BlockManager(4, 2)
    bm.add_sequence(7)
    with pytest.raises(Exception):
        bm.add_sequence(7)
    with pytest.raises(Exception):
        bm.fork(99, 100)
    with pytest.raises(Exception):
        bm.free_sequence(99)
    for _ in range(8):
        bm.append_token(7)
    with pytest.raises(native.OutOfBlocks):
        bm.append_token(7)


def _check_groups(nat, order, starts, plens, mg, mp):
    """The defining properties of the shared-prefix description."""
    bs = nat.block_size
    tables = [nat.block_table(s) for s in order]
    lens = [nat.length(s) for s in order]
    n = len(order)
    assert starts[0] == 0 and starts[-1] == n and all(a < b for a, b in zip(starts[:-1], starts[1:]))
    assert len(plens) == len(starts) - 1
    assert mg == max(b - a for a, b in zip(starts[:-1], starts[1:])) and mp == max(plens)
    for g, (a, e) in enumerate(zip(starts[:-1], starts[1:])):
        members = range(a, e)
        first = tables[a][0] if tables[a] else None
        # members begin on the same block; the next group does not
        if e - a > 1:
            assert first is not None and all(tables[m] and tables[m][0] == first for m in members)
        if e < n and first is not None and tables[e]:
            assert tables[e][0] != first
        # the prefix: whole blocks, equal in every member, full in every member, and maximal
        P = int(plens[g])
        k = P // bs
        assert P % bs == 0
        assert all(tables[m][:k] == tables[a][:k] and lens[m] >= P for m in members)
        extendable = all(len(tables[m]) > k and len(tables[a]) > k and tables[m][k] == tables[a][k]
                         and lens[m] >= (k + 1) * bs for m in members)
        assert not extendable


@pytest.mark.parametrize("bs", [1, 4, 16])
def test_shared_prefix_groups_on_random_fork_trees(native, bs):
    rng = np.random.default_rng(40 + bs)
    nat = native.BlockManager(4000, bs)
    seqs, next_id = [], 0
    for prompt in range(12):
        root = next_id
        next_id += 1
        nat.add_sequence(root)
        for _ in range(int(rng.integers(0, 120))):
            nat.append_token(root)
        family = [root]
        for _ in range(int(rng.integers(0, 6))):  # samples forked from the prompt or from each other
            nat.fork(int(rng.choice(family)), next_id)
            family.append(next_id)
            next_id += 1
        for _ in range(200):
            nat.append_token(int(rng.choice(family)))
        seqs += family
    for trial in range(3):
        order = list(seqs) if trial == 0 else [int(x) for x in rng.permutation(seqs)]
        starts, plens, mg, mp = nat.shared_prefix_groups(order)
        _check_groups(nat, order, starts.tolist(), plens.tolist(), mg, mp)


def test_shared_prefix_groups_of_parallel_samples(native):
    """3 prompts of 40 tokens (bs 16: 2 full blocks + 8 tokens) x 4 samples,
    each sample then writing its own tokens: the samples of a prompt form a
    group sharing the 32 tokens of the full prompt blocks (the partial block
    is copied on the first write)."""
    nat = native.BlockManager(200, 16)
    order = []
    for p in range(3):
        root = 10 * p
        nat.add_sequence(root)
        for _ in range(40):
            nat.append_token(root)
        order.append(root)
        for s in range(1, 4):
            nat.fork(root, root + s)
            order.append(root + s)
    for s in order:
        for _ in range(1 + s % 5):
            nat.append_token(s)
    starts, plens, mg, mp = nat.shared_prefix_groups(order)
    assert starts.tolist() == [0, 4, 8, 12] and plens.tolist() == [32, 32, 32] and (mg, mp) == (4, 32)
    _check_groups(nat, order, starts.tolist(), plens.tolist(), mg, mp)
    # a sequence that shares nothing is a group of one with prefix 0
    nat.add_sequence(99)
    nat.append_token(99)
    starts, plens, _, _ = nat.shared_prefix_groups(order[:4] + [99] + order[4:])
    assert starts.tolist() == [0, 4, 5, 9, 13] and plens.tolist() == [32, 0, 32, 32]
