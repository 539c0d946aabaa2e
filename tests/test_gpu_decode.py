"""GPU parity of paged decode attention (pass 1 + split-KV merge) and of the
contiguous-cache variant against the fp64 CPU oracle, at sizes that span
several 32-token stages and ragged tails, plus the invariants the pages fix."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_355_b200.workloads import custom_case, make_case
from tests.helpers import assert_matches_oracle, np_of

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_355_b200 as pa

    assert torch.cuda.is_available()
    pa.pa_read_error_flag()
    return pa


def run_gpu(pa, case, partition=0, out_dtype=torch.float32, k_pool=None, v_pool=None, block_tables=None,
            out_offset=0):
    """Paged decode of a case's current pools (no append); out_offset > 0
    puts the output that many elements into its buffer (misaligned rows)."""
    q = case.q.cuda()
    kp = (case.k_pool if k_pool is None else k_pool).cuda()
    vp = (case.v_pool if v_pool is None else v_pool).cuda()
    bt = (case.block_tables if block_tables is None else block_tables).cuda()
    lens = case.lengths.cuda()
    buf = torch.full((q.numel() + out_offset,), float("nan"), dtype=out_dtype, device="cuda")
    out = buf[out_offset:].view(tuple(q.shape))
    pa.pa_paged_attention_decode(q, kp, vp, bt, lens, case.max_len, case.scale, out, partition_size=partition)
    torch.cuda.synchronize()
    return out


def run_oracle(case, k_pool=None, v_pool=None, block_tables=None):
    return oracle.paged_decode(np_of(case.q), np_of(case.k_pool if k_pool is None else k_pool),
                               np_of(case.v_pool if v_pool is None else v_pool),
                               np_of(case.block_tables if block_tables is None else block_tables),
                               np_of(case.lengths), case.scale, case.workload.block_size)


# ---------------------------------------------------------------------------
# the tiny configuration, whole decode step (slot mapping, cache write, attention)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("partition", [0, 32])
def test_tiny_decode_step(pa, partition):
    case = make_case("tiny")
    w = case.workload
    # oracle: slot of each sequence's new token, write it, attend
    slots_ref = oracle.slot_mapping(np_of(case.block_tables), np_of(case.new_seq_ids), np_of(case.new_positions),
                                    w.block_size)
    kp, vp = np_of(case.k_pool).copy(), np_of(case.v_pool).copy()
    oracle.reshape_and_cache(np_of(case.k_new), np_of(case.v_new), kp, vp, slots_ref)
    ref = oracle.paged_decode(np_of(case.q), kp, vp, np_of(case.block_tables), np_of(case.lengths), case.scale,
                              w.block_size)
    # GPU: the same step through the library
    gk, gv = case.k_pool.cuda(), case.v_pool.cuda()
    slots = torch.empty(w.batch, dtype=torch.int64, device="cuda")
    out = torch.empty(tuple(case.q.shape), dtype=torch.float32, device="cuda")
    pa.decode_step(case.q.cuda(), case.k_new.cuda(), case.v_new.cuda(), gk, gv, case.block_tables.cuda(),
                   case.lengths.cuda(), case.max_len, case.scale, out, slots, partition_size=partition)
    torch.cuda.synchronize()
    assert np.array_equal(np_of(slots), slots_ref)
    assert np_of(gk).tobytes() == kp.tobytes() and np_of(gv).tobytes() == vp.tobytes()
    assert_matches_oracle(out, ref, False, "tiny step")
    assert pa.pa_read_error_flag() == 0


# ---------------------------------------------------------------------------
# sweep: element type, head_dim, block size, group size, split / no split
# ---------------------------------------------------------------------------
def _ragged_lengths(bs):
    return [1, bs - 1, bs, bs + 1, 31, 32, 33, 95, 100, 257]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("partition", [0, 64])
def test_decode_sweep(pa, dtype, D, bs, G, partition):
    Hkv = 2
    case = custom_case(_ragged_lengths(bs), Hkv * G, Hkv, D, bs, DT[dtype], seed=D * 7 + bs * 3 + G)
    if dtype == "f32" and G == 16:
        with pytest.raises(pa.PAError, match="UNSUPPORTED"):
            run_gpu(pa, case, partition)
        return
    out = run_gpu(pa, case, partition)
    assert_matches_oracle(out, run_oracle(case), dtype == "bf16", f"{dtype} D{D} bs{bs} G{G} P{partition}")
    assert pa.pa_read_error_flag() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_sequence_edge_lengths(pa, dtype):
    P = 64
    for L in [0, 1, 15, 16, 17, 31, 32, 33, P - 1, P, P + 1, 2 * P + 3, 5 * P]:
        case = custom_case([L], 8, 2, 128, 16, DT[dtype], seed=L)
        for part in (0, P, 32):
            out = run_gpu(pa, case, part)
            if L == 0:
                assert torch.all(out == 0), "empty sequence must give a zero row"
            else:
                assert_matches_oracle(out, run_oracle(case), dtype == "bf16", f"L={L} P={part}")
    assert pa.pa_read_error_flag() == 0


def test_large_batch_takes_index_order(pa):
    """Above 2048 sequences the kernel skips the longest-first ranking and
    takes sequences in index order; results are the same attention."""
    rng = np.random.default_rng(21)
    lengths = [int(x) for x in rng.integers(0, 90, 2100)]
    case = custom_case(lengths, 4, 2, 64, 16, torch.bfloat16, seed=21)
    for part in (0, 32):
        out = run_gpu(pa, case, part)
        assert_matches_oracle(out, run_oracle(case), True, f"batch 2100 P={part}")
    assert pa.pa_read_error_flag() == 0


@pytest.mark.parametrize("part", [0, 512])
def test_many_splits_few_rows(pa, part):
    """Few long rows cut into many splits: the merge gives each row a whole
    CTA (eight warps)."""
    case = custom_case([30001, 17000, 1], 8, 2, 128, 16, torch.bfloat16, seed=22)
    out = run_gpu(pa, case, part)
    assert_matches_oracle(out, run_oracle(case), True, f"many splits P={part}")
    assert pa.pa_read_error_flag() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D,bs,G", [(128, 16, 1), (128, 8, 4), (64, 32, 8), (128, 16, 16), (64, 16, 2)])
@pytest.mark.parametrize("partition", [0, 32])
def test_decode_append_equals_write_then_decode(pa, dtype, D, bs, G, partition):
    """pa_paged_attention_decode_append = pa_reshape_and_cache_decode then
    pa_paged_attention_decode: pools and slots bit for bit, attention at the
    bar.  The appended slots start as NaN, so a tile staged before the write
    landed would poison the result."""
    if dtype == "f32" and G == 16:
        pytest.skip("group size 16 is bf16 only")
    Hkv = 2
    lengths = [1, 17, 0, 64, 65, 200, 33]
    case = custom_case(lengths, Hkv * G, Hkv, D, bs, DT[dtype], seed=D + bs + G)
    B = len(lengths)
    g = torch.Generator().manual_seed(7 * G + bs)
    key = torch.randn(B, Hkv, D, generator=g).to(DT[dtype])
    val = torch.randn(B, Hkv, D, generator=g).to(DT[dtype])
    kp, vp = case.k_pool.clone(), case.v_pool.clone()
    for b, L in enumerate(lengths):
        if L > 0:
            blk = int(case.block_tables[b, (L - 1) // bs])
            kp[blk, :, (L - 1) % bs] = float("nan")
            vp[blk, :, (L - 1) % bs] = float("nan")
    live = np.array([b for b, L in enumerate(lengths) if L > 0], dtype=np.int32)
    want_slots = np.full(B, -1, dtype=np.int64)
    want_slots[live] = oracle.slot_mapping(np_of(case.block_tables), live,
                                           np.array([lengths[b] - 1 for b in live], dtype=np.int32), bs)
    hk, hv = np_of(kp).copy(), np_of(vp).copy()
    oracle.reshape_and_cache(np_of(key), np_of(val), hk, hv, want_slots)
    want = oracle.paged_decode(np_of(case.q), hk, hv, np_of(case.block_tables), np_of(case.lengths), case.scale, bs)
    gk, gv = kp.cuda(), vp.cuda()
    out = torch.full(tuple(case.q.shape), float("nan"), dtype=torch.float32, device="cuda")
    slots = torch.full((B,), 7, dtype=torch.int64, device="cuda")
    pa.pa_paged_attention_decode_append(case.q.cuda(), key.cuda(), val.cuda(), gk, gv, case.block_tables.cuda(),
                                        case.lengths.cuda(), case.max_len, case.scale, out,
                                        partition_size=partition, slot_mapping=slots)
    torch.cuda.synchronize()
    assert np.array_equal(np_of(slots), want_slots)
    assert np_of(gk).tobytes() == hk.tobytes() and np_of(gv).tobytes() == hv.tobytes()
    assert_matches_oracle(out, want, dtype == "bf16", f"append {dtype} D{D} bs{bs} G{G} P{partition}")
    assert pa.pa_read_error_flag() == 0


@pytest.mark.parametrize("fault", ["length_over_max", "length_over_max_unmapped", "bad_last_block",
                                   "negative_last_block", "negative_length", "bad_middle_block"])
def test_decode_append_error_paths_match_two_calls(pa, fault):
    """Bad inputs: the one-launch step leaves the pools, the slots and the
    device error word exactly as pa_reshape_and_cache_decode followed by
    pa_paged_attention_decode leave them, and the rows of the other
    sequences agree at the bar."""
    lengths = [40, 17, 65, 33]
    B, Hkv, G, D, bs = 4, 2, 4, 128, 16
    case = custom_case(lengths, Hkv * G, Hkv, D, bs, torch.bfloat16, seed=97, extra_blocks=10, table_width=8)
    bt, lens, max_len = case.block_tables.clone(), case.lengths.clone(), case.max_len
    bad = {"length_over_max": 2, "length_over_max_unmapped": 2, "bad_last_block": 1, "negative_last_block": 1,
           "negative_length": 3, "bad_middle_block": 0}[fault]
    if fault == "length_over_max":
        max_len = 50  # sequence 2 (65 tokens) is longer; its token 64 still has a table entry
    elif fault == "length_over_max_unmapped":
        max_len = 50
        bt[2, 4] = -1  # ... and here it has none
    elif fault == "bad_last_block":
        bt[1, 1] = case.num_blocks + 5  # the block of sequence 1's new token is outside the pool
    elif fault == "negative_last_block":
        bt[1, 1] = -3
    elif fault == "negative_length":
        lens[3] = -5
    else:
        bt[0, 1] = case.num_blocks + 2  # a block attention reads, not the written one
    g = torch.Generator().manual_seed(98)
    key = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16).cuda()
    val = torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16).cuda()
    q, gbt, glens = case.q.cuda(), bt.cuda(), lens.cuda()
    pa.pa_read_error_flag()

    # two calls
    k2, v2 = case.k_pool.cuda(), case.v_pool.cuda()
    s2 = torch.full((B,), 7, dtype=torch.int64, device="cuda")
    o2 = torch.zeros(B, Hkv * G, D, device="cuda")
    pa.pa_reshape_and_cache_decode(key, val, k2, v2, gbt, glens, s2)
    pa.pa_paged_attention_decode(q, k2, v2, gbt, glens, max_len, case.scale, o2)
    flag2 = pa.pa_read_error_flag()
    # one launch
    k1, v1 = case.k_pool.cuda(), case.v_pool.cuda()
    s1 = torch.full((B,), 7, dtype=torch.int64, device="cuda")
    o1 = torch.zeros(B, Hkv * G, D, device="cuda")
    pa.pa_paged_attention_decode_append(q, key, val, k1, v1, gbt, glens, max_len, case.scale, o1, slot_mapping=s1)
    flag1 = pa.pa_read_error_flag()

    assert flag2 == flag1 == 5, (flag2, flag1)
    assert torch.equal(s1, s2), (s1.tolist(), s2.tolist())
    assert torch.equal(k1.view(torch.int16), k2.view(torch.int16))
    assert torch.equal(v1.view(torch.int16), v2.view(torch.int16))
    keep = [b for b in range(B) if b != bad]
    assert_matches_oracle(o1[keep], o2[keep].double().cpu().numpy(), True, f"{fault}: other sequences")


def test_single_token_returns_value_bit_exactly(pa):
    case = custom_case([1, 1, 1], 8, 4, 128, 16, torch.float32, seed=11)
    out = run_gpu(pa, case)
    for b in range(3):
        blk = int(case.block_tables[b, 0])
        for h in range(8):
            assert torch.equal(out[b, h].cpu(), case.v_pool[blk, h // 2, 0]), (b, h)


def test_bf16_output(pa):
    case = custom_case([5, 70, 300, 1], 16, 4, 128, 16, torch.bfloat16, seed=4)
    out = run_gpu(pa, case, 64, out_dtype=torch.bfloat16)
    assert out.dtype == torch.bfloat16
    assert_matches_oracle(out, run_oracle(case), True, "bf16 out")


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("partition", [0, 64])
def test_physical_permutation_is_bit_identical(pa, partition):
    case = custom_case([3, 40, 129, 300, 17], 8, 2, 128, 16, torch.bfloat16, seed=21, extra_blocks=20)
    base = run_gpu(pa, case, partition)
    g = torch.Generator().manual_seed(22)
    perm = torch.randperm(case.num_blocks, generator=g)
    kp = torch.empty_like(case.k_pool)
    vp = torch.empty_like(case.v_pool)
    kp[perm] = case.k_pool
    vp[perm] = case.v_pool
    bt = torch.where(case.block_tables >= 0, perm[case.block_tables.clamp(min=0).long()].to(torch.int32),
                     case.block_tables)
    again = run_gpu(pa, case, partition, k_pool=kp, v_pool=vp, block_tables=bt)
    assert torch.equal(base, again)


def test_block_size_changes_nothing_beyond_rounding(pa):
    lengths = [7, 64, 100, 333]
    outs = []
    for bs in (8, 16, 32):
        # the same logical K/V (drawn per token) placed with three block sizes
        g = torch.Generator().manual_seed(31)
        logical_k = [torch.randn(L, 2, 128, generator=g).to(torch.bfloat16) for L in lengths]
        logical_v = [torch.randn(L, 2, 128, generator=g).to(torch.bfloat16) for L in lengths]
        case = custom_case(lengths, 8, 2, 128, bs, torch.bfloat16, seed=32)
        for b, L in enumerate(lengths):
            for t in range(L):
                blk = int(case.block_tables[b, t // bs])
                case.k_pool[blk, :, t % bs] = logical_k[b][t]
                case.v_pool[blk, :, t % bs] = logical_v[b][t]
        case.q = torch.randn(len(lengths), 8, 128, generator=torch.Generator().manual_seed(33)).to(torch.bfloat16)
        out = run_gpu(pa, case)
        assert_matches_oracle(out, run_oracle(case), True, f"bs{bs}")
        outs.append(out)
    # stages always hold 32 logical tokens, so the arithmetic is the same
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_shared_prefix_equals_private_copies(pa):
    # four samples of one prompt: shared prompt blocks vs private copies of them
    case = custom_case([200, 200, 200, 200], 8, 2, 128, 16, torch.bfloat16, seed=41, extra_blocks=40)
    bt = case.block_tables.clone()
    # private: every sample gets its own copy of sample 0's first 10 blocks
    kp, vp = case.k_pool.clone(), case.v_pool.clone()
    for s in range(1, 4):
        for i in range(10):
            kp[bt[s, i]] = kp[bt[0, i]]
            vp[bt[s, i]] = vp[bt[0, i]]
    private = run_gpu(pa, case, k_pool=kp, v_pool=vp)
    shared_bt = bt.clone()
    shared_bt[1:, :10] = bt[0, :10]
    shared = run_gpu(pa, case, k_pool=kp, v_pool=vp, block_tables=shared_bt)
    assert torch.equal(private, shared)


def test_copy_on_write_leaves_other_sharers_unchanged(pa):
    # 3 sequences share a 2-block prefix whose second block is partial (20 tokens)
    case = custom_case([20, 20, 20], 8, 2, 128, 16, torch.bfloat16, seed=51, extra_blocks=8, table_width=3)
    bt = case.block_tables.clone()
    bt[1, :2] = bt[0, :2]
    bt[2, :2] = bt[0, :2]
    gk, gv, gbt = case.k_pool.cuda(), case.v_pool.cuda(), bt.cuda()
    lens = case.lengths.cuda()
    q = case.q.cuda()
    before = torch.empty(3, 8, 128, device="cuda")
    pa.pa_paged_attention_decode(q, gk, gv, gbt, lens, 21, case.scale, before)
    snapshot_k, snapshot_v = gk.clone(), gv.clone()
    # sequence 2 appends token 20: CoW its partial block into a free block first
    free = int(case.block_tables[1, 0])  # sequence 1's own blocks are now unused
    pa.pa_copy_blocks(gk, gv, torch.tensor([[int(bt[0, 1]), free]], dtype=torch.int64, device="cuda"))
    gbt[2, 1] = free
    slots = torch.empty(1, dtype=torch.int64, device="cuda")
    pa.pa_slot_mapping(gbt, torch.tensor([2], dtype=torch.int32, device="cuda"),
                       torch.tensor([20], dtype=torch.int32, device="cuda"), 16, slots)
    new_k = torch.full((1, 2, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    pa.pa_reshape_and_cache(new_k, -new_k, gk, gv, slots)
    lens2 = torch.tensor([20, 20, 21], dtype=torch.int32, device="cuda")
    after = torch.empty(3, 8, 128, device="cuda")
    pa.pa_paged_attention_decode(q, gk, gv, gbt, lens2, 21, case.scale, after)
    torch.cuda.synchronize()
    assert slots.item() == free * 16 + 4
    for blk in (int(bt[0, 0]), int(bt[0, 1])):
        assert torch.equal(gk[blk], snapshot_k[blk]) and torch.equal(gv[blk], snapshot_v[blk])
    assert torch.equal(after[:2], before[:2])
    assert not torch.equal(after[2], before[2])
    ref = oracle.paged_decode(np_of(case.q), np_of(gk), np_of(gv), np_of(gbt), np_of(lens2), case.scale, 16)
    assert_matches_oracle(after, ref, True, "after CoW")
    assert pa.pa_read_error_flag() == 0


@pytest.mark.parametrize("partition", [0, 64])
def test_nan_poison_outside_the_sequences_is_never_read(pa, partition):
    case = custom_case([5, 33, 100, 250], 16, 4, 128, 16, torch.bfloat16, seed=61, extra_blocks=10,
                       table_width=20)
    clean = run_gpu(pa, case, partition)
    kp, vp = case.k_pool.clone(), case.v_pool.clone()
    used = torch.zeros(case.num_blocks, 16, dtype=torch.bool)
    for b, L in enumerate(case.lengths.tolist()):
        for t in range(L):
            used[case.block_tables[b, t // 16], t % 16] = True
    kp.permute(0, 2, 1, 3)[~used] = float("nan")  # [NB, bs, Hkv, D] view, mask over (NB, bs)
    vp.permute(0, 2, 1, 3)[~used] = float("nan")
    bt = case.block_tables.clone()
    bt[bt < 0] = case.num_blocks + 1000  # table entries past each sequence: out of range, never read
    out = run_gpu(pa, case, partition, k_pool=kp, v_pool=vp, block_tables=bt)
    assert torch.equal(out, clean)
    assert pa.pa_read_error_flag() == 0


def test_bad_block_id_is_flagged_not_dereferenced(pa):
    case = custom_case([40, 40], 8, 2, 128, 16, torch.bfloat16, seed=71)
    bt = case.block_tables.clone()
    bt[1, 1] = case.num_blocks + 7
    run_gpu(pa, case, block_tables=bt)
    assert pa.pa_read_error_flag() == 5
    run_gpu(pa, case)
    assert pa.pa_read_error_flag() == 0


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("partition", [0, 32])
def test_misaligned_output_is_bit_identical(pa, out_dtype, partition):
    """An output buffer that starts one element past an alignment boundary
    (rows no longer 16-byte aligned) gets the same values, element by
    element, as an aligned one."""
    case = custom_case([1, 17, 300, 64, 129], 8, 2, 128, 16, torch.bfloat16, seed=77)
    a = run_gpu(pa, case, partition=partition, out_dtype=out_dtype)
    b = run_gpu(pa, case, partition=partition, out_dtype=out_dtype, out_offset=1)
    assert torch.equal(a, b)
    assert pa.pa_read_error_flag() == 0


def test_repeat_runs_are_bit_identical(pa):
    case = custom_case([1000, 3000, 17, 4096], 32, 8, 128, 16, torch.bfloat16, seed=81)
    a = run_gpu(pa, case, 256)
    b = run_gpu(pa, case, 256)
    assert torch.equal(a, b)


# ---------------------------------------------------------------------------
# contiguous-cache variant (the baseline of the paging-overhead measurement)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("partition", [0, 64])
def test_contiguous_variant(pa, dtype, partition):
    case = custom_case([1, 17, 64, 200, 333], 16, 4, 128, 16, DT[dtype], seed=91)
    B, L_pad = 5, 352
    k_c = torch.full((B, 4, L_pad, 128), float("nan"), dtype=DT[dtype])
    v_c = torch.full((B, 4, L_pad, 128), float("nan"), dtype=DT[dtype])
    for b, L in enumerate(case.lengths.tolist()):
        for t in range(L):
            blk = int(case.block_tables[b, t // 16])
            k_c[b, :, t] = case.k_pool[blk, :, t % 16]
            v_c[b, :, t] = case.v_pool[blk, :, t % 16]
    out = torch.empty(B, 16, 128, device="cuda")
    pa.pa_paged_attention_decode_contiguous(case.q.cuda(), k_c.cuda(), v_c.cuda(), case.lengths.cuda(),
                                            case.max_len, case.scale, out, block_size=16,
                                            partition_size=partition)
    torch.cuda.synchronize()
    ref = oracle.contiguous_decode(np_of(case.q), np_of(k_c), np_of(v_c), np_of(case.lengths), case.scale)
    assert_matches_oracle(out, ref, dtype == "bf16", "contiguous")
    # same kernel, same stages, same order: identical bits to the paged call
    assert torch.equal(out, run_gpu(pa, case, partition))
