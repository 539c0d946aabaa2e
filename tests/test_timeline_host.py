"""Host side of the timeline tool (paged_kv_cache_355_b200/timeline.py), on
the CPU: the launch order it attributes pass-1 CTAs with, and the summary it
computes from the stamp arrays."""
from __future__ import annotations

import numpy as np

from paged_kv_cache_355_b200.timeline import KERNELS, TL_CTAS, TL_SLOTS, TT_CTAS, TT_EVENTS, TT_TILES, _summary, \
    launch_order


def test_launch_order_is_longest_first_by_64_length_buckets_then_index():
    max_len = 4096
    lengths = np.array([5, 100, 100, 3000, 7, 4096, 0, 3000, 64])
    order = launch_order(lengths, max_len)
    assert sorted(order.tolist()) == list(range(len(lengths)))
    bucket = lambda L: min(63, (min(max(L, 0), max_len) * 64) // (max_len + 1))
    # ranks go by decreasing bucket; within a bucket by increasing index
    keys = [(-bucket(lengths[b]), b) for b in order]
    assert keys == sorted(keys)
    assert order[0] == 5 and order[1] == 3 and order[2] == 7
    # 5, 7, 0 and 64 tokens share the lowest bucket: index order among them
    assert order[-4:].tolist() == [0, 4, 6, 8]
    # lengths above max_len count as max_len; beyond the ranking's batch limit, index order
    assert launch_order(np.array([9999, 10]), 100)[0] == 0
    assert launch_order(np.arange(3000), 4096).tolist() == list(range(3000))


def _stamps(n_p1, base=10_000_000):
    ev = np.zeros((len(KERNELS), TL_CTAS, TL_SLOTS), np.uint64)
    tt = np.zeros((TT_CTAS, TT_TILES, TT_EVENTS), np.uint64)
    # pass 1: CTA i enters at i us, stages its table 1 us later, first stage
    # 2 us after that, streams 0.5 us per token for 10 (i + 1) tokens,
    # epilogue 1 us
    tok = 10 * (np.arange(n_p1) + 1)
    t0 = base + 1000 * np.arange(n_p1)
    ev[2, :n_p1, 0] = t0
    ev[2, :n_p1, 1] = t0 + 1000
    ev[2, :n_p1, 3] = t0 + 3000
    ev[2, :n_p1, 4] = t0 + 3000 + 500 * tok
    ev[2, :n_p1, 2] = t0 + 4000 + 500 * tok
    return ev, tt, tok


def test_summary_phases_fit_and_resident_counts():
    n = 8
    ev, tt, tok = _stamps(n)
    r = _summary(ev, tt, lambda ids: tok[ids])
    assert r["ctas"][2] == n and sum(r["ctas"]) == n
    k = r["kernels"]["pass 1"]
    assert k["entry_us"][0] == 0.0 and k["entry_us"][-1] == 7.0
    assert r["call_end_us"] == 7.0 + 4.0 + 0.5 * 80
    ph = r["pass1_phases_us"]
    assert ph["prologue"] == [1.0] * 5 and ph["first stage"] == [2.0] * 5 and ph["epilogue"] == [1.0] * 5
    f = r["pass1_life_fit"]
    assert abs(f["fixed_us"] - 4.0) < 1e-6 and abs(f["ns_per_token"] - 500.0) < 1e-3
    # resident at t = 0 and t = 5: CTA 0, then CTAs 0..5
    res = r["resident"]["pass 1"]
    assert res[0] == 1 and res[1] == 6
    # summed lives over the most CTAs resident at once
    lives = 4.0 + 0.5 * tok
    assert abs(r["pass1_summed_life_per_slot_us"] - lives.sum() / max(res)) < 0.01


def test_summary_tile_chain_medians():
    ev, tt, tok = _stamps(2)
    ev[1, 0, 0] = ev[2, 0, 0]  # one prefix CTA
    ev[1, 0, 2] = ev[2, 0, 0] + 50_000
    base = int(ev[2, 0, 0])
    for j in range(4):
        t = base + 3000 * j
        tt[0, j, 5] = t            # K requested
        tt[0, j, 4] = t + 1000     # S issued
        tt[0, j, 0] = t + 1500     # scores ready
        tt[0, j, 1] = t + 2300     # P written
        tt[0, j, 6] = t + 500      # V requested
        tt[0, j, 3] = t + 2500     # P.V issued
    r = _summary(ev, tt, None)
    chain = r["prefix_tiles_us"]
    assert [c["tile"] for c in chain] == [1, 2, 3]
    c = chain[0]
    assert c["period"] == 3.0 and c["scores_to_P"] == 0.8 and c["P_to_PV"] == 0.2
    assert c["Vreq_to_PV"] == 2.0 and c["Kreq_to_S"] == 1.0 and c["S_to_scores"] == 0.5


def test_prefill_summary_on_synthetic_stamps():
    from paged_kv_cache_355_b200.timeline import PF_CTAS, PF_SLOTS, _prefill_summary

    ev = np.zeros((PF_CTAS, PF_SLOTS), np.uint64)
    base = 5_000_000
    # two SMs, two CTAs each: entry, ready +0.5, first S +2, last P.V (tile 0,
    # tile 1) at +20/+21, exit +23; the second CTA on an SM enters 1.5 us
    # after the first exits
    for i, (sm, start) in enumerate([(0, 0.0), (1, 0.0), (0, 24.5), (1, 24.5)]):
        t = base + int(start * 1000)
        ev[i, 0], ev[i, 1], ev[i, 2] = t, t + 500, t + 2000
        ev[i, 3], ev[i, 4], ev[i, 5] = t + 20000, t + 21000, t + 23000
        ev[i, PF_SLOTS - 1] = sm
    r = _prefill_summary(ev)
    assert r["ctas"] == 4 and r["sms"] == 2 and r["span_us"] == 47.5
    assert r["life_us"] == [23.0] * 5 and r["entry_to_first_S_us"] == [2.0] * 5
    assert r["last_PV_to_exit_us"] == [2.0] * 5 and r["exit_to_next_entry_us"] == [1.5] * 5
    assert r["ctas_per_sm"] == [2.0] * 5 and r["sm_last_exit_us"] == [47.5] * 5
    assert abs(r["first_S_to_last_PV_share"] - (4 * 19.0) / (2 * 47.5)) < 1e-4


def test_prefill_timeline_runs_the_benchmarked_workload():
    import importlib.util
    import os

    from paged_kv_cache_355_b200.timeline import PREFILL_SHAPE

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_for_timeline", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    assert PREFILL_SHAPE == bench.PREFILL_SHAPE
