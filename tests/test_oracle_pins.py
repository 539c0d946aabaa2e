"""Pins for the CPU oracle's attention: brute force, closed forms, invariants.

Each check is chosen so that a plausible slip in the oracle (a wrong sign in
the exponent, a dropped normalisation or scale, a wrong head or in-block
index, a transposed pool layout) makes at least one of them fail;
test_oracle_mutants.py plants those slips and checks exactly that.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
from oracle import brute
from tests.helpers import f32_to_bf16_bits, pad_tables, place_logical, random_tables, to_logical_lists

pytestmark = pytest.mark.filterwarnings("ignore")


def _random_case(rng, lengths, Hq, Hkv, D, bs, extra_blocks=3):
    B = len(lengths)
    logical_k = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lengths]
    logical_v = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lengths]
    nb = sum(-(-L // bs) for L in lengths) + extra_blocks
    tables = random_tables(rng, lengths, bs, nb)
    k_pool, v_pool = place_logical(logical_k, logical_v, tables, nb, bs, fill=np.nan)
    bt = pad_tables(tables, max(len(t) for t in tables) + 1)
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    return q, logical_k, logical_v, k_pool, v_pool, bt, np.array(lengths, np.int32)


# ---------------------------------------------------------------------------
# brute force over logical lists (never paged)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("bs", [1, 2, 8, 16])
@pytest.mark.parametrize("G", [1, 2])
def test_oracle_matches_brute_force(bs, G):
    rng = np.random.default_rng(100 + bs * 7 + G)
    for trial in range(3):
        B = int(rng.integers(1, 5))
        lengths = [int(x) for x in rng.integers(1, 41, size=B)]
        Hkv, D = 2, 8
        Hq = Hkv * G
        scale = float(np.float32(1.0 / math.sqrt(D)))
        q, lk, lv, kp, vp, bt, lens = _random_case(rng, lengths, Hq, Hkv, D, bs)
        got = oracle.paged_decode(q, kp, vp, bt, lens, scale, bs)
        want = brute.decode_logical(q.astype(np.float64).tolist(), to_logical_lists(lk), to_logical_lists(lv),
                                    float(np.float32(scale)))
        np.testing.assert_allclose(got, np.array(want), rtol=0, atol=1e-12)


def test_oracle_rows_match_full():
    rng = np.random.default_rng(7)
    q, lk, lv, kp, vp, bt, lens = _random_case(rng, [5, 17, 33], 4, 2, 8, 8)
    full = oracle.paged_decode(q, kp, vp, bt, lens, 0.3, 8)
    rb = np.array([0, 1, 2, 2, 1], np.int32)
    rh = np.array([3, 0, 1, 2, 2], np.int32)
    rows = oracle.paged_decode_rows(q, kp, vp, bt, lens, 0.3, 8, rb, rh)
    np.testing.assert_array_equal(rows, full[rb, rh])


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------
def _single_seq(k_rows, v_rows, q_rows, bs=4, scale=1.0, G=1):
    """One sequence; k_rows/v_rows [L, Hkv, D]; q_rows [Hq, D]."""
    L = k_rows.shape[0]
    nb = -(-L // bs) + 2
    tables = [list(range(nb - 1, nb - 1 - (-(-L // bs)), -1))]  # reversed placement
    kp, vp = place_logical([k_rows], [v_rows], tables, nb, bs, fill=np.nan)
    bt = pad_tables(tables, len(tables[0]))
    return oracle.paged_decode(q_rows[None].astype(np.float32), kp, vp, bt, np.array([L], np.int32), scale, bs)[0]


def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(1)
    k = rng.standard_normal((1, 1, 16)).astype(np.float32)
    v = rng.standard_normal((1, 1, 16)).astype(np.float32)
    q = rng.standard_normal((1, 16)).astype(np.float32) * 50
    out = _single_seq(k, v, q, scale=0.7)
    assert np.array_equal(out[0], v[0, 0].astype(np.float64))


def test_zero_query_gives_mean_value():
    rng = np.random.default_rng(2)
    L = 37
    k = rng.standard_normal((L, 1, 8)).astype(np.float32)
    v = rng.standard_normal((L, 1, 8)).astype(np.float32)
    out = _single_seq(k, v, np.zeros((1, 8), np.float32))
    np.testing.assert_allclose(out[0], v[:, 0].astype(np.float64).mean(axis=0), rtol=0, atol=1e-13)


def test_identical_keys_give_mean_value():
    rng = np.random.default_rng(3)
    L = 21
    k = np.repeat(rng.standard_normal((1, 1, 8)).astype(np.float32), L, axis=0)
    v = rng.standard_normal((L, 1, 8)).astype(np.float32)
    q = rng.standard_normal((1, 8)).astype(np.float32)
    out = _single_seq(k, v, q, scale=0.9)
    np.testing.assert_allclose(out[0], v[:, 0].astype(np.float64).mean(axis=0), rtol=0, atol=1e-13)


@pytest.mark.parametrize("scale,mult", [(1.0, 1.0), (0.5, 2.0), (0.125, 8.0)])
def test_weights_one_two_three(scale, mult):
    # keys along e0 with scale*<q,k> = 0, ln 2, ln 3  ->  softmax weights 1/6, 2/6, 3/6
    D = 4
    c = np.array([0.0, math.log(2.0), math.log(3.0)]) * mult
    k = np.zeros((3, 1, D), np.float32)
    k[:, 0, 0] = c
    v = np.array([[1, 0, 0, 6], [0, 1, 0, 6], [0, 0, 1, 6]], np.float32)[:, None, :]
    q = np.zeros((1, D), np.float32)
    q[0, 0] = 1.0
    out = _single_seq(k, v, q, bs=2, scale=scale)
    np.testing.assert_allclose(out[0], [1 / 6, 2 / 6, 3 / 6, 6.0], rtol=0, atol=2e-7)


def test_dominant_score_selects_its_value():
    rng = np.random.default_rng(4)
    L, D = 40, 8
    k = rng.standard_normal((L, 1, D)).astype(np.float32) * 0.01
    v = rng.standard_normal((L, 1, D)).astype(np.float32)
    q = np.zeros((1, D), np.float32)
    q[0, 0] = 1.0
    k[23, 0, 0] = 80.0  # score gap >= 60 against every other token
    out = _single_seq(k, v, q, bs=8, scale=1.0)
    np.testing.assert_allclose(out[0], v[23, 0].astype(np.float64), rtol=1e-20, atol=1e-20)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (8, 1), (16, 4)])
def test_grouped_heads_read_kv_head_h_div_g(Hq, Hkv):
    # one token, a distinct value per kv head: query head h must return v[h // G]
    D = 8
    G = Hq // Hkv
    k = np.ones((1, Hkv, D), np.float32)
    v = np.arange(Hkv * D, dtype=np.float32).reshape(1, Hkv, D)
    q = np.ones((Hq, D), np.float32)
    out = _single_seq(k, v, q, bs=4, G=G)
    for h in range(Hq):
        assert np.array_equal(out[h], v[0, h // G].astype(np.float64)), h


def test_empty_sequence_gives_zero_row():
    rng = np.random.default_rng(5)
    q, lk, lv, kp, vp, bt, lens = _random_case(rng, [3, 9], 2, 2, 8, 4)
    lens[0] = 0
    out = oracle.paged_decode(q, kp, vp, bt, lens, 0.5, 4)
    assert np.all(out[0] == 0.0)
    assert np.all(np.isfinite(out[1]))


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------
def test_physical_block_permutation_is_invisible():
    rng = np.random.default_rng(6)
    lengths = [1, 7, 16, 33, 40]
    q, lk, lv, kp, vp, bt, lens = _random_case(rng, lengths, 4, 2, 8, 8, extra_blocks=9)
    base = oracle.paged_decode(q, kp, vp, bt, lens, 0.35, 8)
    perm = rng.permutation(kp.shape[0])  # new id of old block i is perm[i]
    kp2 = np.empty_like(kp)
    vp2 = np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    again = oracle.paged_decode(q, kp2, vp2, bt2, lens, 0.35, 8)
    assert np.array_equal(base, again)


def test_block_size_is_invisible():
    rng = np.random.default_rng(8)
    lengths = [1, 15, 16, 17, 64, 70]
    Hkv, D = 2, 8
    lk = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lengths]
    lv = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lengths]
    q = rng.standard_normal((len(lengths), 4, D)).astype(np.float32)
    results = []
    for bs in (1, 2, 8, 16, 32):
        nb = sum(-(-L // bs) for L in lengths) + 2
        tables = random_tables(rng, lengths, bs, nb)
        kp, vp = place_logical(lk, lv, tables, nb, bs, fill=np.nan)
        bt = pad_tables(tables, max(len(t) for t in tables))
        results.append(oracle.paged_decode(q, kp, vp, bt, np.array(lengths, np.int32), 0.3, bs))
    for r in results[1:]:
        assert np.array_equal(results[0], r)


def test_contiguous_layout_gives_identical_result():
    rng = np.random.default_rng(9)
    lengths = [4, 19, 32]
    Hkv, D, bs, L_pad = 2, 8, 8, 40
    q, lk, lv, kp, vp, bt, lens = _random_case(rng, lengths, 4, Hkv, D, bs)
    k_c = np.full((len(lengths), Hkv, L_pad, D), np.nan, np.float32)
    v_c = np.full((len(lengths), Hkv, L_pad, D), np.nan, np.float32)
    for b, L in enumerate(lengths):
        k_c[b, :, :L] = lk[b].transpose(1, 0, 2)
        v_c[b, :, :L] = lv[b].transpose(1, 0, 2)
    paged = oracle.paged_decode(q, kp, vp, bt, lens, 0.4, bs)
    contig = oracle.contiguous_decode(q, k_c, v_c, lens, 0.4)
    assert np.array_equal(paged, contig)


def test_shared_prefix_blocks_equal_private_copies():
    rng = np.random.default_rng(10)
    bs, Hkv, D, n = 8, 2, 8, 4
    prefix = 19  # 2 full shared blocks + a partial one
    total = prefix + 5
    pk = rng.standard_normal((prefix, Hkv, D)).astype(np.float32)
    pv = rng.standard_normal((prefix, Hkv, D)).astype(np.float32)
    lk = [np.concatenate([pk, rng.standard_normal((5, Hkv, D)).astype(np.float32)]) for _ in range(n)]
    lv = [np.concatenate([pv, rng.standard_normal((5, Hkv, D)).astype(np.float32)]) for _ in range(n)]
    q = rng.standard_normal((n, 4, D)).astype(np.float32)
    lens = np.full(n, total, np.int32)
    # private: every sample owns all of its blocks
    nb = n * 3 + 4
    priv_tables = random_tables(rng, [total] * n, bs, nb)
    kp, vp = place_logical(lk, lv, priv_tables, nb, bs)
    out_priv = oracle.paged_decode(q, kp, vp, pad_tables(priv_tables, 3), lens, 0.3, bs)
    # shared: the two full prefix blocks are one physical pair for all samples
    shared = [0, 1]
    tables = [shared + [2 + 2 * i, 3 + 2 * i] for i in range(n)]
    kp2, vp2 = place_logical(lk, lv, tables, 2 + 2 * n, bs)
    out_shared = oracle.paged_decode(q, kp2, vp2, pad_tables(tables, 4), lens, 0.3, bs)
    assert np.array_equal(out_priv, out_shared)


def test_copy_on_write_isolates_the_other_sharers():
    rng = np.random.default_rng(11)
    bs, Hkv, D = 4, 2, 8
    k_pool = rng.standard_normal((6, Hkv, bs, D)).astype(np.float32)
    v_pool = rng.standard_normal((6, Hkv, bs, D)).astype(np.float32)
    # three sequences share blocks 0 and 1 (length 7: block 1 is partial)
    bt = np.array([[0, 1], [0, 1], [0, 1]], np.int32)
    lens = np.array([7, 7, 7], np.int32)
    q = rng.standard_normal((3, 2, D)).astype(np.float32)
    before = oracle.paged_decode(q, k_pool, v_pool, bt, lens, 0.5, bs)
    snapshot_k, snapshot_v = k_pool.copy(), v_pool.copy()
    # sequence 2 writes token 7: copy block 1 to block 4 first, then write there
    oracle.copy_blocks(k_pool, v_pool, [(1, 4)])
    bt[2, 1] = 4
    slot = oracle.slot_mapping(bt, [2], [7], bs)
    assert slot[0] == 4 * bs + 3
    oracle.reshape_and_cache(np.full((1, Hkv, D), 9.0, np.float32), np.full((1, Hkv, D), -9.0, np.float32),
                             k_pool, v_pool, slot)
    lens[2] = 8
    after = oracle.paged_decode(q, k_pool, v_pool, bt, lens, 0.5, bs)
    assert np.array_equal(k_pool[:4], snapshot_k[:4]) and np.array_equal(v_pool[:4], snapshot_v[:4])
    assert np.array_equal(after[:2], before[:2])
    assert not np.array_equal(after[2], before[2])


# ---------------------------------------------------------------------------
# element types and argument checks
# ---------------------------------------------------------------------------
def test_bf16_inputs_widen_exactly():
    rng = np.random.default_rng(12)
    q, lk, lv, kp, vp, bt, lens = _random_case(rng, [6, 13], 4, 2, 8, 4)
    kp = np.nan_to_num(kp)
    vp = np.nan_to_num(vp)
    qb, kb, vb = f32_to_bf16_bits(q), f32_to_bf16_bits(kp), f32_to_bf16_bits(vp)
    via_bf16 = oracle.paged_decode(qb, kb, vb, bt, lens, 0.25, 4)
    via_f32 = oracle.paged_decode(oracle.bf16_bits_to_f64(qb).astype(np.float32),
                                  oracle.bf16_bits_to_f64(kb).astype(np.float32),
                                  oracle.bf16_bits_to_f64(vb).astype(np.float32), bt, lens, 0.25, 4)
    assert np.array_equal(via_bf16, via_f32)


def test_rejects_block_id_outside_pool():
    rng = np.random.default_rng(13)
    q, lk, lv, kp, vp, bt, lens = _random_case(rng, [9], 2, 2, 8, 4)
    bt[0, 1] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle.paged_decode(q, kp, vp, bt, lens, 0.5, 4)


def test_rejects_length_beyond_table():
    rng = np.random.default_rng(14)
    q, lk, lv, kp, vp, bt, lens = _random_case(rng, [9], 2, 2, 8, 4)
    lens[0] = bt.shape[1] * 4 + 1
    with pytest.raises(ValueError):
        oracle.paged_decode(q, kp, vp, bt, lens, 0.5, 4)
