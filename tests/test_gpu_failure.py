"""Failure detection without a GPU fault: a bounded wait that runs out is
reported through the device error word, the kernel returns normally, and the
context stays usable for the next call."""
from __future__ import annotations

import time

import pytest
import torch

from paged_kv_cache_355_b200.workloads import custom_case
from tests.helpers import assert_matches_oracle, np_of

import oracle

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout_and_context_survives():
    import paged_kv_cache_355_b200 as pa

    assert torch.cuda.is_available()
    pa.pa_read_error_flag()  # clear
    t0 = time.perf_counter()
    pa.pa_selftest_wait_timeout(100_000)  # 100 ms
    assert pa.pa_read_error_flag() == 6  # PA_ERR_TIMEOUT
    assert time.perf_counter() - t0 >= 0.09
    assert pa.pa_read_error_flag() == 0  # read and cleared
    # the context still runs the decode kernels correctly
    case = custom_case([5, 77, 300], 8, 2, 128, 16, torch.bfloat16, seed=31)
    out = torch.empty(tuple(case.q.shape), dtype=torch.float32, device="cuda")
    pa.pa_paged_attention_decode(case.q.cuda(), case.k_pool.cuda(), case.v_pool.cuda(), case.block_tables.cuda(),
                                 case.lengths.cuda(), case.max_len, case.scale, out)
    torch.cuda.synchronize()
    want = oracle.paged_decode(np_of(case.q), np_of(case.k_pool), np_of(case.v_pool), np_of(case.block_tables),
                               np_of(case.lengths), case.scale, 16)
    assert_matches_oracle(out, want, True, "decode after a timed-out wait")
    assert pa.pa_read_error_flag() == 0


def test_read_probe_streams_a_buffer_without_errors():
    import paged_kv_cache_355_b200 as pa

    pa.pa_read_error_flag()
    for nbytes in (16, 16384 + 48, 64 << 20):
        buf = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
        pa.pa_hbm_read_probe(buf)
        assert pa.pa_read_error_flag() == 0
