"""Pins for the oracle's causal multi-query (chunked prefill) attention."""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
from oracle import brute
from tests.helpers import pad_tables, place_logical, random_tables, to_logical_lists


def _case(rng, lengths, news, Hq, Hkv, D, bs):
    lk = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lengths]
    lv = [rng.standard_normal((L, Hkv, D)).astype(np.float32) for L in lengths]
    nb = sum(-(-L // bs) for L in lengths) + 2
    tables = random_tables(rng, lengths, bs, nb)
    kp, vp = place_logical(lk, lv, tables, nb, bs, fill=np.nan)
    bt = pad_tables(tables, max(len(t) for t in tables))
    qs = np.concatenate([[0], np.cumsum(news)]).astype(np.int32)
    q = rng.standard_normal((int(qs[-1]), Hq, D)).astype(np.float32)
    return q, lk, lv, kp, vp, bt, np.array(lengths, np.int32), qs


@pytest.mark.parametrize("bs,G", [(1, 1), (4, 2), (8, 1), (16, 4)])
def test_prefill_matches_brute_force(bs, G):
    rng = np.random.default_rng(bs + 10 * G)
    lengths, news = [5, 23, 40], [5, 7, 1]
    Hkv, D = 2, 8
    q, lk, lv, kp, vp, bt, lens, qs = _case(rng, lengths, news, Hkv * G, Hkv, D, bs)
    got = oracle.paged_prefill(q, kp, vp, bt, lens, qs, 0.3, bs)
    qlists = [[[list(map(float, q[r, h])) for h in range(Hkv * G)] for r in range(qs[b], qs[b + 1])]
              for b in range(len(lengths))]
    want = brute.prefill_logical(qlists, to_logical_lists(lk), to_logical_lists(lv), float(np.float32(0.3)))
    flat = np.array([row for seq in want for row in seq])
    np.testing.assert_allclose(got, flat, rtol=0, atol=1e-12)


def test_each_query_equals_a_decode_call_at_its_own_length():
    rng = np.random.default_rng(3)
    lengths, news = [17, 33], [9, 33]
    q, lk, lv, kp, vp, bt, lens, qs = _case(rng, lengths, news, 8, 2, 16, 8)
    got = oracle.paged_prefill(q, kp, vp, bt, lens, qs, 0.25, 8)
    for b, (L, n) in enumerate(zip(lengths, news)):
        for i in range(n):
            row = qs[b] + i
            one = oracle.paged_decode(q[row][None], kp, vp, bt[b][None], np.array([L - n + i + 1], np.int32), 0.25, 8)
            assert np.array_equal(got[row], one[0])


def test_first_position_sees_only_itself():
    # a chunk that is the whole sequence: query 0 sits at position 0, out = v_0
    rng = np.random.default_rng(4)
    q, lk, lv, kp, vp, bt, lens, qs = _case(rng, [12], [12], 4, 4, 8, 4)
    got = oracle.paged_prefill(q * 50, kp, vp, bt, lens, qs, 1.0, 4)
    for h in range(4):
        assert np.array_equal(got[0, h], lv[0][0, h].astype(np.float64))


def test_single_new_token_is_decode():
    rng = np.random.default_rng(5)
    q, lk, lv, kp, vp, bt, lens, qs = _case(rng, [7, 30, 1], [1, 1, 1], 8, 2, 16, 8)
    assert np.array_equal(oracle.paged_prefill(q, kp, vp, bt, lens, qs, 0.5, 8),
                          oracle.paged_decode(q, kp, vp, bt, lens, 0.5, 8))


def test_rejects_more_queries_than_tokens():
    rng = np.random.default_rng(6)
    q, lk, lv, kp, vp, bt, lens, qs = _case(rng, [4], [4], 2, 2, 8, 4)
    lens = np.array([3], np.int32)
    with pytest.raises(ValueError):
        oracle.paged_prefill(q, kp, vp, bt, lens, qs, 0.5, 4)
