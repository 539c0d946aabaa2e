"""The decode entry point that allocates nothing.

pa_paged_attention_decode_static_scratch serves callers that cannot allocate
device memory where they run attention (inside a graph capture, a serving
loop kept out of the allocator, or a host framework that owns all device
memory): its split-KV scratch is a fixed array inside libpa.  It must give the
same results as pa_paged_attention_decode with a caller-provided workspace,
call after call (the array keeps the previous call's contents), and refuse
sizes whose scratch would not fit.

This file is collected last so that a run stopping at the first failure has
run every other test first; it also passes alone in a fresh process.
"""
from __future__ import annotations

import pytest
import torch

from paged_kv_cache_355_b200.workloads import custom_case
from tests.helpers import assert_matches_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_scratch_matches_the_workspace_entry_point(dtype):
    import paged_kv_cache_355_b200 as pa

    # long enough for several 64-token splits, so the scratch is really used
    case = custom_case([1, 40, 200, 333, 64, 129], 16, 4, 128, 16, dtype, seed=123)
    q, kp, vp = case.q.cuda(), case.k_pool.cuda(), case.v_pool.cuda()
    bt, lens = case.block_tables.cuda(), case.lengths.cuda()
    part = 64
    need = pa.pa_paged_attention_workspace_size(6, 16, 4, 128, case.max_len, 16, part)
    assert 0 < need <= pa.STATIC_SCRATCH_BYTES
    ref = torch.empty(6, 16, 128, device="cuda")
    pa.pa_paged_attention_decode(q, kp, vp, bt, lens, case.max_len, case.scale, ref, partition_size=part,
                                 workspace=torch.empty(need, dtype=torch.uint8, device="cuda"))
    for call in range(2):
        out = torch.full((6, 16, 128), float("nan"), device="cuda")
        pa.pa_paged_attention_decode_static_scratch(q, kp, vp, bt, lens, case.max_len, case.scale, out,
                                                    partition_size=part)
        torch.cuda.synchronize()
        assert_matches_oracle(out, ref.double().cpu().numpy(), dtype == torch.bfloat16, f"static scratch call {call}")
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
