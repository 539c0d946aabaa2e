"""Pins for the oracle's slot mapping, cache write, block copy and bf16 rounding."""
from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.block_manager import BlockManager

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_mapping_from_the_pages():
    g = json.load(open(os.path.join(GOLDEN, "worked_mapping.json")))
    bs = g["block_size"]
    bt = np.array([g["block_table"]], np.int32)
    positions = np.arange(2 * bs, dtype=np.int32)
    slots = oracle.slot_mapping(bt, np.zeros_like(positions), positions, bs)
    for logical, physical in g["logical_to_physical"]:
        for pos in range(logical * bs, (logical + 1) * bs):
            assert slots[pos] // bs == physical
            assert slots[pos] % bs == pos - logical * bs
    # position 17 is offset 1 of logical block 1, i.e. physical block 105
    assert slots[17] == 105 * 16 + 1 == 1681


def test_slot_mapping_matches_block_manager():
    rng = np.random.default_rng(20)
    for bs in (1, 2, 8, 16, 32):
        bm = BlockManager(400, bs)
        seqs = list(range(6))
        slots_bm, sid, pos = [], [], []
        for _ in range(150):
            s = int(rng.integers(0, len(seqs)))
            p = bm.lengths.get(s, 0)
            slot, pairs = bm.append_token(s)
            assert pairs == []
            slots_bm.append(slot)
            sid.append(s)
            pos.append(p)
        width = max(len(bm.block_table(s)) for s in bm.tables)
        bt = np.full((len(seqs), width), -1, np.int32)
        for s in bm.tables:
            bt[s, : len(bm.block_table(s))] = bm.block_table(s)
        got = oracle.slot_mapping(bt, np.array(sid, np.int32), np.array(pos, np.int32), bs)
        assert got.tolist() == slots_bm


def test_slot_mapping_rejects_unmapped_position():
    bt = np.array([[3, -1]], np.int32)
    with pytest.raises(ValueError):
        oracle.slot_mapping(bt, [0], [5], 4)  # logical block 1 is unmapped
    with pytest.raises(ValueError):
        oracle.slot_mapping(bt, [0], [8], 4)  # beyond the table


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_reshape_and_cache_matches_explicit_loops(dtype):
    rng = np.random.default_rng(21)
    NB, Hkv, bs, D, T = 9, 3, 8, 16, 20
    mk = (lambda a: a.astype(np.float32)) if dtype == "f32" else (
        lambda a: rng.integers(0, 2 ** 16, size=a.shape, dtype=np.uint16))
    k_pool = mk(rng.standard_normal((NB, Hkv, bs, D)))
    v_pool = mk(rng.standard_normal((NB, Hkv, bs, D)))
    key = mk(rng.standard_normal((T, Hkv, D)))
    val = mk(rng.standard_normal((T, Hkv, D)))
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
    slots[[2, 11]] = -1
    exp_k, exp_v = k_pool.copy(), v_pool.copy()
    for i in range(T):
        if slots[i] < 0:
            continue
        blk, off = divmod(int(slots[i]), bs)
        for h in range(Hkv):
            for d in range(D):
                exp_k[blk, h, off, d] = key[i, h, d]
                exp_v[blk, h, off, d] = val[i, h, d]
    oracle.reshape_and_cache(key, val, k_pool, v_pool, slots)
    assert k_pool.tobytes() == exp_k.tobytes()
    assert v_pool.tobytes() == exp_v.tobytes()


def test_reshape_and_cache_rejects_slot_outside_pool():
    k_pool = np.zeros((2, 1, 4, 8), np.float32)
    v_pool = np.zeros_like(k_pool)
    with pytest.raises(ValueError):
        oracle.reshape_and_cache(np.ones((1, 1, 8), np.float32), np.ones((1, 1, 8), np.float32),
                                 k_pool, v_pool, np.array([8], np.int64))


@pytest.mark.parametrize("dtype", [np.float32, np.uint16])
def test_copy_blocks_matches_numpy(dtype):
    rng = np.random.default_rng(22)
    NB, Hkv, bs, D = 12, 2, 16, 8
    if dtype == np.float32:
        k_pool = rng.standard_normal((NB, Hkv, bs, D)).astype(np.float32)
        v_pool = rng.standard_normal((NB, Hkv, bs, D)).astype(np.float32)
    else:
        k_pool = rng.integers(0, 2 ** 16, size=(NB, Hkv, bs, D), dtype=np.uint16)
        v_pool = rng.integers(0, 2 ** 16, size=(NB, Hkv, bs, D), dtype=np.uint16)
    pairs = [(0, 5), (3, 7), (0, 11), (9, 2)]
    exp_k, exp_v = k_pool.copy(), v_pool.copy()
    for s, d in pairs:
        exp_k[d] = exp_k[s]
        exp_v[d] = exp_v[s]
    oracle.copy_blocks(k_pool, v_pool, pairs)
    assert k_pool.tobytes() == exp_k.tobytes() and v_pool.tobytes() == exp_v.tobytes()


def test_round_bf16_matches_torch_on_float32_values():
    rng = np.random.default_rng(23)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        rng.standard_normal(1000) * 1e-39]).astype(np.float32)
    ours = oracle.round_bf16(x.astype(np.float64))
    theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def test_round_bf16_ties_go_to_even():
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 1 + 2.0 ** -8 + 2.0 ** -40, 0.0, -0.0])
    got = oracle.bf16_bits_to_f64(oracle.round_bf16(x))
    assert got.tolist() == [1.0, 1 + 2.0 ** -6, -1.0, 1 + 2.0 ** -7, 0.0, -0.0]
    assert np.signbit(got[-1])
