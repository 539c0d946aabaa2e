"""The decode entry point that allocates nothing.

pa_paged_attention_decode_static_scratch serves callers that cannot allocate
device memory where they run attention (inside a graph capture, a serving
loop kept out of the allocator, or a host framework that owns all device
memory): its split-KV scratch is a fixed array inside libpa.  It must give
the same bits as pa_paged_attention_decode with a caller-provided workspace,
call after call.  The array keeps the previous call's contents, so the calls
here alternate between cases with different split counts and shapes: a
leftover partial result of one call reaching the next call's merge would
show as a difference.  It must also refuse sizes whose scratch would not fit.

This file is collected last so that a run stopping at the first failure has
run every other test first; it also passes alone in a fresh process.
"""
from __future__ import annotations

import pytest
import torch

import oracle
from paged_kv_cache_355_b200.workloads import custom_case
from tests.helpers import assert_matches_oracle, np_of

pytestmark = pytest.mark.gpu

# (lengths, Hq, Hkv, head_dim, partition): the first case has more splits per
# row and more rows than the second, so the second call leaves stale partials
# of the first in the array wherever it does not write
CASES = [
    ([1, 40, 200, 333, 64, 129, 777], 16, 4, 128, 64),
    ([35, 90, 3], 8, 2, 64, 32),
]


def _inputs(lengths, hq, hkv, d, dtype, seed):
    case = custom_case(lengths, hq, hkv, d, 16, dtype, seed=seed)
    return case, case.q.cuda(), case.k_pool.cuda(), case.v_pool.cuda(), case.block_tables.cuda(), case.lengths.cuda()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_scratch_matches_the_workspace_entry_point(dtype):
    import paged_kv_cache_355_b200 as pa

    pa.pa_read_error_flag()
    for call, (lengths, hq, hkv, d, part) in enumerate(CASES + CASES[:1]):
        case, q, kp, vp, bt, lens = _inputs(lengths, hq, hkv, d, dtype, seed=123 + 10 * (call % 2))
        B = len(lengths)
        need = pa.pa_paged_attention_workspace_size(B, hq, hkv, d, case.max_len, 16, part)
        assert 0 < need <= pa.STATIC_SCRATCH_BYTES
        ref = torch.full((B, hq, d), float("nan"), device="cuda")
        pa.pa_paged_attention_decode(q, kp, vp, bt, lens, case.max_len, case.scale, ref, partition_size=part,
                                     workspace=torch.empty(need, dtype=torch.uint8, device="cuda"))
        out = torch.full((B, hq, d), float("nan"), device="cuda")
        pa.pa_paged_attention_decode_static_scratch(q, kp, vp, bt, lens, case.max_len, case.scale, out,
                                                    partition_size=part)
        torch.cuda.synchronize()
        # same kernels, same plan: the same bits as the workspace call
        assert torch.equal(out, ref), f"static scratch call {call} differs from the workspace entry point"
        want = oracle.paged_decode(np_of(case.q), np_of(case.k_pool), np_of(case.v_pool),
                                   np_of(case.block_tables), np_of(case.lengths), case.scale, 16)
        assert_matches_oracle(out, want, dtype == torch.bfloat16, f"static scratch call {call}")
    assert pa.pa_read_error_flag() == 0


def test_static_scratch_rejects_sizes_beyond_its_maximum():
    import paged_kv_cache_355_b200 as pa

    # batch 64 x 64 query heads x 128 splits of 32 tokens needs far more than the array holds
    B, Hq, Hkv, D, L = 64, 64, 8, 128, 4096
    assert pa.pa_paged_attention_workspace_size(B, Hq, Hkv, D, L, 16, 32) > pa.STATIC_SCRATCH_BYTES
    q = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros(1, Hkv, 16, D, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(B, L // 16, dtype=torch.int32, device="cuda")
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    out = torch.empty(B, Hq, D, device="cuda")
    with pytest.raises(pa.PAError, match="PA_ERR_WORKSPACE"):
        pa.pa_paged_attention_decode_static_scratch(q, pool, pool, bt, lens, L, 0.1, out, partition_size=32)
