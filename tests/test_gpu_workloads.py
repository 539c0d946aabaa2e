"""The named decode workloads at full size, run exactly as the benchmark runs
them (same launch configuration): cache writes and copies compared bit for
bit with the oracle, attention compared on sampled (sequence, head) rows that
the oracle computes one by one, plus properties that hold at any size."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_355_b200.workloads import make_case
from tests.helpers import assert_matches_oracle, np_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_355_b200 as pa

    assert torch.cuda.is_available()
    pa.pa_read_error_flag()
    return pa


def _sample_rows(case, n=48, seed=0):
    B, Hq = case.workload.batch, case.workload.num_q_heads
    g = torch.Generator().manual_seed(seed)
    order = torch.argsort(case.lengths)
    rb = [int(order[0]), int(order[-1])] + torch.randint(0, B, (n - 2,), generator=g).tolist()
    rh = torch.randint(0, Hq, (n,), generator=g).tolist()
    return np.array(rb, np.int32), np.array(rh, np.int32)


@pytest.mark.parametrize("name", ["llama7b", "gqa", "cow", "long16", "long32"])
def test_workload_full_size(pa, name):
    case = make_case(name, device="cuda")
    w = case.workload
    bs = w.block_size
    # --- oracle side, on host copies taken before the GPU touches the pools
    kp_h, vp_h = np_of(case.k_pool).copy(), np_of(case.v_pool).copy()
    bt_h, lens_h = np_of(case.block_tables), np_of(case.lengths)
    if case.cow_pairs.numel():
        oracle.copy_blocks(kp_h, vp_h, np_of(case.cow_pairs))
    slots_ref = oracle.slot_mapping(bt_h, np_of(case.new_seq_ids), np_of(case.new_positions), bs)
    oracle.reshape_and_cache(np_of(case.k_new), np_of(case.v_new), kp_h, vp_h, slots_ref)

    # --- GPU side: copy-on-write copies, slot mapping, cache write, attention
    bt, lens = case.block_tables.cuda(), case.lengths.cuda()
    if case.cow_pairs.numel():
        pa.pa_copy_blocks(case.k_pool, case.v_pool, case.cow_pairs.cuda())
    slots = torch.empty(case.new_seq_ids.numel(), dtype=torch.int64, device="cuda")
    pa.pa_slot_mapping(bt, case.new_seq_ids.cuda(), case.new_positions.cuda(), bs, slots)
    if not case.cow_pairs.numel():  # plain decode: the decode form gives the same slots
        slots2 = torch.empty_like(slots)
        pa.pa_decode_slot_mapping(bt, lens, bs, slots2)
        assert torch.equal(slots, slots2)
    pa.pa_reshape_and_cache(case.k_new, case.v_new, case.k_pool, case.v_pool, slots)
    out = torch.full(tuple(case.q.shape), float("nan"), device="cuda")
    pa.pa_paged_attention_decode(case.q, case.k_pool, case.v_pool, bt, lens, case.max_len, case.scale, out)
    torch.cuda.synchronize()
    assert pa.pa_read_error_flag() == 0

    assert np.array_equal(np_of(slots), slots_ref)
    assert np_of(case.k_pool).tobytes() == kp_h.tobytes()
    assert np_of(case.v_pool).tobytes() == vp_h.tobytes()

    rb, rh = _sample_rows(case)
    ref = oracle.paged_decode_rows(np_of(case.q), kp_h, vp_h, bt_h, lens_h, case.scale, bs, rb, rh)
    err = assert_matches_oracle(out[torch.from_numpy(rb).long(), torch.from_numpy(rh).long()], ref, True, name)
    print(f"{name}: max|d| over {len(rb)} sampled rows = {err:.3e}")

    # properties at full size: every row finite, bounded by the largest |V|,
    # and a second run gives identical bits
    assert torch.isfinite(out).all()
    assert out.abs().max() <= max(case.k_pool.abs().max(), case.v_pool.float().abs().max()) + 1e-3
    again = torch.empty_like(out)
    pa.pa_paged_attention_decode(case.q, case.k_pool, case.v_pool, bt, lens, case.max_len, case.scale, again)
    torch.cuda.synchronize()
    assert torch.equal(out, again)


@pytest.mark.parametrize("name", ["llama7b", "gqa", "long16", "long32"])
def test_decode_step_full_size(pa, name):
    """The call the benchmark times for these workloads,
    pa_paged_attention_decode_append (the new token's slot, its cache write
    and the attention in one launch), in the benchmark's launch configuration
    (automatic partition, caller workspace, slot output): slots and both
    pools bit for bit against the oracle's slot mapping and cache write,
    attention on 48 sampled rows plus every head of the longest and the
    shortest sequence.  The appended slots start NaN-poisoned, so a tile
    staged before the folded write would show."""
    case = make_case(name, device="cuda")
    w = case.workload
    B, Hq, Hkv, D, bs = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size
    assert case.new_seq_ids.numel() == B and not case.cow_pairs.numel()
    bt_h, lens_h = np_of(case.block_tables), np_of(case.lengths)
    for b, L in enumerate(lens_h.tolist()):
        blk = int(bt_h[b, (L - 1) // bs])
        case.k_pool[blk, :, (L - 1) % bs] = float("nan")
        case.v_pool[blk, :, (L - 1) % bs] = float("nan")
    kp_h, vp_h = np_of(case.k_pool).copy(), np_of(case.v_pool).copy()
    slots_ref = oracle.slot_mapping(bt_h, np_of(case.new_seq_ids), np_of(case.new_positions), bs)
    oracle.reshape_and_cache(np_of(case.k_new), np_of(case.v_new), kp_h, vp_h, slots_ref)

    bt, lens = case.block_tables.cuda(), case.lengths.cuda()
    part = pa.pa_paged_attention_partition_size(B, Hq, Hkv, D, case.max_len, bs)
    ws_bytes = pa.pa_paged_attention_workspace_size(B, Hq, Hkv, D, case.max_len, bs, part)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    out = torch.full((B, Hq, D), float("nan"), device="cuda")
    slots = torch.full((B,), 7, dtype=torch.int64, device="cuda")
    pa.pa_paged_attention_decode_append(case.q, case.k_new, case.v_new, case.k_pool, case.v_pool, bt, lens,
                                        case.max_len, case.scale, out, partition_size=part, workspace=ws,
                                        slot_mapping=slots)
    torch.cuda.synchronize()
    assert pa.pa_read_error_flag() == 0
    assert np.array_equal(np_of(slots), slots_ref)
    assert np_of(case.k_pool).tobytes() == kp_h.tobytes()
    assert np_of(case.v_pool).tobytes() == vp_h.tobytes()

    rb, rh = _sample_rows(case)
    order = torch.argsort(case.lengths)
    ends = [int(order[0]), int(order[-1])]
    rb = np.concatenate([rb, np.repeat(np.array(ends, np.int32), Hq)])
    rh = np.concatenate([rh, np.tile(np.arange(Hq, dtype=np.int32), 2)])
    ref = oracle.paged_decode_rows(np_of(case.q), kp_h, vp_h, bt_h, lens_h, case.scale, bs, rb, rh)
    err = assert_matches_oracle(out[torch.from_numpy(rb).long(), torch.from_numpy(rh).long()], ref, True, name)
    print(f"{name} decode step (partition {part}): max|d| over {len(rb)} rows = {err:.3e}")
    assert torch.isfinite(out).all()


def test_shared_prefix_full_size_cow(pa):
    """The shared-prefix workload at full size through the call the benchmark
    times for it (pa_paged_attention_decode_shared_prefix, automatic
    partitions): the step's copy-on-write copies and token writes first, then
    attention with each group's 992 shared prompt tokens read once; sampled
    rows plus every head of the longest and shortest sequence against the
    oracle, and every row against the plain decode call at the bar."""
    from paged_kv_cache_355_b200.workloads import shared_prefix_groups

    case = make_case("cow", device="cuda")
    w = case.workload
    B, Hq, Hkv, D, bs = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size
    kp_h, vp_h = np_of(case.k_pool).copy(), np_of(case.v_pool).copy()
    bt_h, lens_h = np_of(case.block_tables), np_of(case.lengths)
    oracle.copy_blocks(kp_h, vp_h, np_of(case.cow_pairs))
    slots_ref = oracle.slot_mapping(bt_h, np_of(case.new_seq_ids), np_of(case.new_positions), bs)
    oracle.reshape_and_cache(np_of(case.k_new), np_of(case.v_new), kp_h, vp_h, slots_ref)

    bt, lens = case.block_tables.cuda(), case.lengths.cuda()
    pa.pa_copy_blocks(case.k_pool, case.v_pool, case.cow_pairs.cuda())
    slots = torch.empty(case.new_seq_ids.numel(), dtype=torch.int64, device="cuda")
    pa.pa_slot_mapping(bt, case.new_seq_ids.cuda(), case.new_positions.cuda(), bs, slots)
    pa.pa_reshape_and_cache(case.k_new, case.v_new, case.k_pool, case.v_pool, slots)
    starts, plens = shared_prefix_groups(case)
    assert all(bt_h[b, : plens[g] // bs].tolist() == bt_h[starts[g], : plens[g] // bs].tolist()
               for g in range(len(plens)) for b in range(starts[g], starts[g + 1]))
    gs = torch.tensor(starts, dtype=torch.int32, device="cuda")
    gl = torch.tensor(plens, dtype=torch.int32, device="cuda")
    out = torch.full((B, Hq, D), float("nan"), device="cuda")
    pa.pa_paged_attention_decode_shared_prefix(case.q, case.k_pool, case.v_pool, bt, lens, case.max_len, case.scale,
                                               out, gs, gl, max(plens), w.samples)
    plain = torch.full_like(out, float("nan"))
    pa.pa_paged_attention_decode(case.q, case.k_pool, case.v_pool, bt, lens, case.max_len, case.scale, plain)
    torch.cuda.synchronize()
    assert pa.pa_read_error_flag() == 0
    assert np_of(case.k_pool).tobytes() == kp_h.tobytes() and np_of(case.v_pool).tobytes() == vp_h.tobytes()

    rb, rh = _sample_rows(case)
    order = torch.argsort(case.lengths)
    ends = [int(order[0]), int(order[-1])]
    rb = np.concatenate([rb, np.repeat(np.array(ends, np.int32), Hq)])
    rh = np.concatenate([rh, np.tile(np.arange(Hq, dtype=np.int32), 2)])
    ref = oracle.paged_decode_rows(np_of(case.q), kp_h, vp_h, bt_h, lens_h, case.scale, bs, rb, rh)
    err = assert_matches_oracle(out[torch.from_numpy(rb).long(), torch.from_numpy(rh).long()], ref, True, "cow")
    print(f"cow shared prefix: max|d| over {len(rb)} rows = {err:.3e}")
    assert_matches_oracle(out, plain.double().cpu().numpy(), True, "cow: shared prefix vs plain decode")
    again = torch.empty_like(out)
    pa.pa_paged_attention_decode_shared_prefix(case.q, case.k_pool, case.v_pool, bt, lens, case.max_len, case.scale,
                                               again, gs, gl, max(plens), w.samples)
    torch.cuda.synchronize()
    assert torch.equal(out, again)
