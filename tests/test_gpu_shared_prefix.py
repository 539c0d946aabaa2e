"""GPU parity of pa_paged_attention_decode_shared_prefix: groups of sequences
that share their prompt blocks, attended with one read of each shared block
per group, against the fp64 oracle (which knows nothing of the sharing: it
walks every sequence's own table), over head sizes, block sizes, group sizes
(several row chunks per group included), prefix and suffix splits, members
whose whole context is the prefix, and broken group descriptions."""
from __future__ import annotations

import pytest
import torch

import oracle
from tests.helpers import assert_matches_oracle, np_of, shared_prefix_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_355_b200 as pa

    assert torch.cuda.is_available()
    pa.pa_read_error_flag()
    return pa


def _groups(bs):
    r = lambda x: x - x % bs
    return [
        (r(64), [r(64) + 7, r(64) + 1, r(64) + 90]),
        (0, [5]),
        (bs, [bs, bs + 1]),  # the first member's whole context is the prefix
        (r(640), [r(640) + k for k in (0, 1, 13, 31, 32, 33, 200, 7, 64)]),
        (r(1000), [r(1000) + 3, r(1000) + 517]),
    ]


def run_shared(pa, case, starts, plens, partition=0, max_prefix=None, max_group=None, bt=None, kp=None, vp=None,
               out_dtype=torch.float32, out_offset=0):
    B, Hq, D = case.q.shape
    buf = torch.full((B * Hq * D + out_offset,), float("nan"), dtype=out_dtype, device="cuda")
    out = buf[out_offset:].view(B, Hq, D)
    gs = torch.tensor(starts, dtype=torch.int32, device="cuda")
    gl = torch.tensor(plens, dtype=torch.int32, device="cuda")
    mp = max(plens) if max_prefix is None else max_prefix
    mg = max(b - a for a, b in zip(starts[:-1], starts[1:])) if max_group is None else max_group
    pa.pa_paged_attention_decode_shared_prefix(
        case.q.cuda(), (case.k_pool if kp is None else kp).cuda(), (case.v_pool if vp is None else vp).cuda(),
        (case.block_tables if bt is None else bt).cuda(), case.lengths.cuda(), case.max_len, case.scale, out, gs, gl,
        mp, mg, partition_size=partition)
    torch.cuda.synchronize()
    return out


def run_oracle(case, bt=None, kp=None, vp=None):
    return oracle.paged_decode(np_of(case.q), np_of(case.k_pool if kp is None else kp),
                               np_of(case.v_pool if vp is None else vp),
                               np_of(case.block_tables if bt is None else bt), np_of(case.lengths), case.scale,
                               case.workload.block_size)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("partition", [0, 64])
def test_shared_prefix_sweep(pa, D, bs, G, partition):
    Hkv = 2
    case, starts, plens = shared_prefix_case(_groups(bs), Hkv * G, Hkv, D, bs, torch.bfloat16, seed=D + bs + G)
    out = run_shared(pa, case, starts, plens, partition)
    assert_matches_oracle(out, run_oracle(case), True, f"shared prefix D{D} bs{bs} G{G} P{partition}")
    assert pa.pa_read_error_flag() == 0


def test_bf16_output(pa):
    case, starts, plens = shared_prefix_case(_groups(16), 32, 8, 128, 16, torch.bfloat16, seed=5)
    out = run_shared(pa, case, starts, plens, out_dtype=torch.bfloat16)
    assert_matches_oracle(out, run_oracle(case), True, "shared prefix, bf16 out")


def test_no_prefix_is_bit_identical_to_plain_decode(pa):
    """With every prefix 0 the call is pass 1 and the merge of the plain
    decode, with the same splits: the same bits."""
    groups = [(0, [70, 5]), (0, [300]), (0, [1, 2, 1000])]
    case, starts, plens = shared_prefix_case(groups, 16, 4, 128, 16, torch.bfloat16, seed=9)
    for part in (0, 64):
        out = run_shared(pa, case, starts, plens, part)
        ref = torch.full_like(out, float("nan"))
        pa.pa_paged_attention_decode(case.q.cuda(), case.k_pool.cuda(), case.v_pool.cuda(),
                                     case.block_tables.cuda(), case.lengths.cuda(), case.max_len, case.scale, ref,
                                     partition_size=part)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)


def test_prefix_last_with_no_shared_tokens_is_bit_identical_to_plain_decode(pa):
    """A prefix bound above 0 but every group's prefix 0, own tokens in one
    split (4096-token partition), head_dim 128: the prefix pass is launched
    after pass 1 and none of its CTAs has work (its last CTA still waits for
    pass 1 before the grid ends).  Pass 1 alone writes every row: the plain
    decode's bits, and the next call sees a finished result."""
    groups = [(0, [70, 5]), (0, [300]), (0, [1, 2, 1000])]
    case, starts, plens = shared_prefix_case(groups, 16, 4, 128, 16, torch.bfloat16, seed=19)
    ref = torch.full((case.q.shape[0], 16, 128), float("nan"), device="cuda")
    pa.pa_paged_attention_decode(case.q.cuda(), case.k_pool.cuda(), case.v_pool.cuda(), case.block_tables.cuda(),
                                 case.lengths.cuda(), case.max_len, case.scale, ref, partition_size=4096)
    for _ in range(3):
        out = run_shared(pa, case, starts, plens, partition=4096, max_prefix=64)
        assert torch.equal(out, ref)
    assert pa.pa_read_error_flag() == 0


def test_repeat_runs_and_physical_permutation_are_bit_identical(pa):
    case, starts, plens = shared_prefix_case(_groups(16), 32, 8, 128, 16, torch.bfloat16, seed=13, extra_blocks=30)
    a = run_shared(pa, case, starts, plens)
    assert torch.equal(a, run_shared(pa, case, starts, plens))
    perm = torch.randperm(case.num_blocks, generator=torch.Generator().manual_seed(14))
    kp, vp = torch.empty_like(case.k_pool), torch.empty_like(case.v_pool)
    kp[perm] = case.k_pool
    vp[perm] = case.v_pool
    bt = torch.where(case.block_tables >= 0, perm[case.block_tables.clamp(min=0).long()].to(torch.int32),
                     case.block_tables)
    assert torch.equal(a, run_shared(pa, case, starts, plens, bt=bt, kp=kp, vp=vp))


def test_nan_poison_outside_the_sequences_is_never_read(pa):
    case, starts, plens = shared_prefix_case(_groups(16), 16, 4, 128, 16, torch.bfloat16, seed=17, extra_blocks=12)
    clean = run_shared(pa, case, starts, plens)
    kp, vp = case.k_pool.clone(), case.v_pool.clone()
    used = torch.zeros(case.num_blocks, 16, dtype=torch.bool)
    for b, L in enumerate(case.lengths.tolist()):
        for t in range(L):
            used[case.block_tables[b, t // 16], t % 16] = True
    kp.permute(0, 2, 1, 3)[~used] = float("nan")
    vp.permute(0, 2, 1, 3)[~used] = float("nan")
    bt = case.block_tables.clone()
    bt[bt < 0] = case.num_blocks + 1000
    assert torch.equal(clean, run_shared(pa, case, starts, plens, bt=bt, kp=kp, vp=vp))
    assert pa.pa_read_error_flag() == 0


@pytest.mark.parametrize("fault", ["not_whole_blocks", "longer_than_a_member", "above_max_prefix",
                                   "group_above_max_size", "starts_out_of_order"])
def test_broken_group_description_is_flagged_and_attended_without_sharing(pa, fault):
    """A group whose description breaks the rules records
    PA_ERR_BAD_BLOCK_ID and is attended as if nothing were shared, so the
    output still matches the oracle."""
    case, starts, plens = shared_prefix_case(_groups(16), 16, 4, 128, 16, torch.bfloat16, seed=23)
    starts, plens = list(starts), list(plens)
    kw = {}
    if fault == "not_whole_blocks":
        plens[0] = 56                     # not a multiple of 16
    elif fault == "longer_than_a_member":
        plens[2] = 32                     # the first member of group 2 has 16 tokens
    elif fault == "above_max_prefix":
        kw["max_prefix"] = 512            # group 3 declares 640
    elif fault == "group_above_max_size":
        kw["max_group"] = 3               # group 3 has 9 members
    else:
        starts[1], starts[2] = starts[2], starts[1]  # group 1 ends before it starts
    pa.pa_read_error_flag()
    out = run_shared(pa, case, starts, plens, **kw)
    assert pa.pa_read_error_flag() == 5
    if fault == "starts_out_of_order":
        # groups 0 and 1 now overlap / are empty; only the untouched groups are specified
        keep = list(range(starts[3], case.workload.batch))
        assert_matches_oracle(out[keep], run_oracle(case)[keep], True, fault)
    else:
        assert_matches_oracle(out, run_oracle(case), True, fault)


def test_groups_that_do_not_cover_the_batch_are_flagged(pa):
    case, starts, plens = shared_prefix_case(_groups(16), 16, 4, 128, 16, torch.bfloat16, seed=29)
    pa.pa_read_error_flag()
    short = starts[:-1]
    out = run_shared(pa, case, short, plens[:-1])  # the last group's sequences belong to no group
    assert pa.pa_read_error_flag() == 5
    covered = list(range(short[-1]))
    assert_matches_oracle(out[covered], run_oracle(case)[covered], True, "covered sequences")


def test_block_manager_groups_drive_the_shared_prefix_call(pa):
    """Prompts forked into samples by the native block manager, each sample
    then writing its own tokens (copy-on-write of the partial prompt block):
    the manager's group description drives the shared-prefix call, which
    matches the oracle walking every sample's own table."""
    import numpy as np

    from paged_kv_cache_355_b200.block_manager import BlockManager
    from paged_kv_cache_355_b200.workloads import Workload, build_case

    bs, Hkv, G, D = 16, 2, 4, 128
    bm = BlockManager(900, bs)
    rng = np.random.default_rng(5)
    order = []
    for p in range(5):
        root = 100 * p
        bm.add_sequence(root)
        for _ in range(int(rng.integers(20, 400))):
            bm.append_token(root)
        order.append(root)
        for s in range(1, int(rng.integers(1, 10))):
            bm.fork(root, root + s)
            order.append(root + s)
    for s in order:
        for _ in range(int(rng.integers(1, 60))):
            bm.append_token(s)
    starts, plens, mg, mp = bm.shared_prefix_groups(order)
    assert mp > 0 and mg > 1
    tables = [bm.block_table(s) for s in order]
    lengths = [bm.length(s) for s in order]
    w = Workload("bm", len(order), Hkv * G, Hkv, D, bs, torch.bfloat16, "fixed")
    case = build_case(w, lengths, tables, 900, [], [], None, 77)
    out = run_shared(pa, case, starts.tolist(), plens.tolist(), max_prefix=mp, max_group=mg)
    assert_matches_oracle(out, run_oracle(case), True, "block-manager groups")
    assert pa.pa_read_error_flag() == 0


# ---- many groups (the GPU-filling case), head_dim 128 ---------------------
# 16 copies of the five groups above with 2 kv heads: 80 groups x 2 kv heads x
# the row chunks >= 160 prefix CTAs, so every group's prefix is one split (the
# tensor-core pass's widest tiling).  With the automatic partition (512
# tokens here) the own tokens take up to 3 splits: the prefix pass runs first,
# pass 1 folds the prefix into one-split rows and the merge pass finishes the
# others.  With a 4096-token partition the own tokens are one split: a set-up
# kernel, pass 1, then the prefix pass, which finishes every shared row.
MANY_COPIES = 16
ORDERS = pytest.mark.parametrize("partition", [0, 4096], ids=["prefix_first", "prefix_last"])


def _many_case(bs, G, seed, extra=(), extra_blocks=4):
    groups = _groups(bs) * MANY_COPIES + list(extra)
    return shared_prefix_case(groups, 2 * G, 2, 128, bs, torch.bfloat16, seed=seed, extra_blocks=extra_blocks)


@ORDERS
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_many_groups_sweep(pa, bs, G, partition):
    """Own parts of 0..517 tokens, members whose context is the prefix, a
    group without a prefix; several row chunks per group for G >= 4."""
    case, starts, plens = _many_case(bs, G, seed=100 + bs + G)
    out = run_shared(pa, case, starts, plens, partition=partition)
    assert_matches_oracle(out, run_oracle(case), True, f"many groups bs{bs} G{G} partition {partition}")
    assert pa.pa_read_error_flag() == 0


@ORDERS
def test_many_groups_bf16_output_and_empty_sequences(pa, partition):
    """bf16 rows; groups without a prefix whose members are empty (rows of
    zeros) or mixed with a non-empty one."""
    case, starts, plens = _many_case(16, 4, seed=131, extra=[(0, [0, 0]), (0, [0, 9])])
    out = run_shared(pa, case, starts, plens, partition=partition, out_dtype=torch.bfloat16)
    ref = run_oracle(case)
    assert_matches_oracle(out, ref, True, "many groups, bf16 out")
    empty = [b for b, L in enumerate(case.lengths.tolist()) if L == 0]
    assert len(empty) == 3 and torch.all(out[empty] == 0)
    assert pa.pa_read_error_flag() == 0


@ORDERS
def test_many_groups_are_deterministic_and_placement_free(pa, partition):
    case, starts, plens = _many_case(16, 4, seed=137, extra_blocks=40)
    a = run_shared(pa, case, starts, plens, partition=partition)
    assert torch.equal(a, run_shared(pa, case, starts, plens, partition=partition))
    perm = torch.randperm(case.num_blocks, generator=torch.Generator().manual_seed(138))
    kp, vp = torch.empty_like(case.k_pool), torch.empty_like(case.v_pool)
    kp[perm] = case.k_pool
    vp[perm] = case.v_pool
    bt = torch.where(case.block_tables >= 0, perm[case.block_tables.clamp(min=0).long()].to(torch.int32),
                     case.block_tables)
    assert torch.equal(a, run_shared(pa, case, starts, plens, partition=partition, bt=bt, kp=kp, vp=vp))


@ORDERS
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_many_groups_misaligned_output_is_bit_identical(pa, partition, out_dtype):
    """An output buffer one element past an alignment boundary gets the same
    values as an aligned one."""
    case, starts, plens = _many_case(16, 4, seed=141)
    a = run_shared(pa, case, starts, plens, partition=partition, out_dtype=out_dtype)
    b = run_shared(pa, case, starts, plens, partition=partition, out_dtype=out_dtype, out_offset=1)
    assert torch.equal(a, b)
    assert pa.pa_read_error_flag() == 0


@ORDERS
def test_many_groups_never_read_outside_the_sequences(pa, partition):
    """NaN in every pool slot no sequence uses (the rest of each partly used
    block included) and junk block ids past each table's used entries."""
    case, starts, plens = _many_case(16, 2, seed=139, extra_blocks=24)
    clean = run_shared(pa, case, starts, plens, partition=partition)
    kp, vp = case.k_pool.clone(), case.v_pool.clone()
    used = torch.zeros(case.num_blocks, 16, dtype=torch.bool)
    for b, L in enumerate(case.lengths.tolist()):
        for t in range(L):
            used[case.block_tables[b, t // 16], t % 16] = True
    kp.permute(0, 2, 1, 3)[~used] = float("nan")
    vp.permute(0, 2, 1, 3)[~used] = float("nan")
    bt = case.block_tables.clone()
    bt[bt < 0] = case.num_blocks + 1000
    assert torch.equal(clean, run_shared(pa, case, starts, plens, partition=partition, bt=bt, kp=kp, vp=vp))
    assert pa.pa_read_error_flag() == 0


@ORDERS
@pytest.mark.parametrize("fault", ["longer_than_a_member", "above_max_prefix", "not_whole_blocks"])
def test_many_groups_broken_group_is_flagged_and_attended_without_sharing(pa, fault, partition):
    case, starts, plens = _many_case(16, 4, seed=149)
    starts, plens = list(starts), list(plens)
    kw = {}
    if fault == "longer_than_a_member":
        plens[7] = 32                     # a copy of group 2: its first member has 16 tokens
    elif fault == "above_max_prefix":
        kw["max_prefix"] = 512            # the copies of group 3 declare 640
    else:
        plens[5] = 56                     # not a multiple of 16
    pa.pa_read_error_flag()
    out = run_shared(pa, case, starts, plens, partition=partition, **kw)
    assert pa.pa_read_error_flag() == 5
    assert_matches_oracle(out, run_oracle(case), True, f"many groups, {fault}, partition {partition}")


@ORDERS
@pytest.mark.parametrize("bad", [-3, 1 << 20])
def test_many_groups_bad_shared_block_id_is_flagged_not_dereferenced(pa, partition, bad):
    """A shared prompt block id out of range (in every member's table, as
    the sharing requires) is flagged and never loaded; the other groups'
    rows are unaffected, and the next call with a clean table is clean."""
    case, starts, plens = _many_case(16, 4, seed=171)
    s, e = starts[3], starts[4]  # the first copy of the 640-token prefix group
    bt = case.block_tables.clone()
    bt[s:e, 5] = bad
    pa.pa_read_error_flag()
    out = run_shared(pa, case, starts, plens, partition=partition, bt=bt)
    assert pa.pa_read_error_flag() == 5
    ref = run_oracle(case)
    others = [b for b in range(case.q.shape[0]) if not s <= b < e]
    assert_matches_oracle(out[others], ref[others], True, f"bad shared block {bad}, partition {partition}")
    clean = run_shared(pa, case, starts, plens, partition=partition)
    assert pa.pa_read_error_flag() == 0
    assert_matches_oracle(clean, ref, True, f"clean after a bad shared block, partition {partition}")


@ORDERS
def test_many_groups_flag_lengths_above_max_context(pa, partition):
    """A length above max_context_len is clamped to it and flagged, as the
    plain decode does."""
    case, starts, plens = _many_case(16, 4, seed=151)
    lens = case.lengths.clone()
    b = int(torch.argmax(lens))
    L = int(lens[b])
    lens[b] = L + 5  # the call is told max_context_len = L
    pa.pa_read_error_flag()
    out = torch.full_like(case.q, float("nan"), dtype=torch.float32, device="cuda")
    gs = torch.tensor(starts, dtype=torch.int32, device="cuda")
    gl = torch.tensor(plens, dtype=torch.int32, device="cuda")
    mg = max(e - s for s, e in zip(starts[:-1], starts[1:]))
    pa.pa_paged_attention_decode_shared_prefix(case.q.cuda(), case.k_pool.cuda(), case.v_pool.cuda(),
                                               case.block_tables.cuda(), lens.cuda(), L, case.scale, out, gs, gl,
                                               max(plens), mg, partition_size=partition)
    torch.cuda.synchronize()
    assert pa.pa_read_error_flag() == 5
    assert_matches_oracle(out, run_oracle(case), True, "many groups, clamped length")
