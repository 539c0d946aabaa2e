"""The timeline build (libpa_timeline.so: the decode kernels with per-CTA
globaltimer stamps) on the GPU.  One shared-prefix call in the prefix-last
order gives the same bits as libpa.so, and its stamps are consistent: every
CTA that ran left its entry and exit, and each CTA's events come in the
order the kernel passes them."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from tests.helpers import shared_prefix_case

pytestmark = pytest.mark.gpu

TL_CTAS, TL_SLOTS = 65536, 16
TT_CTAS, TT_TILES, TT_EVENTS = 512, 16, 8


def _call(b, case, starts, plens, out):
    gs = torch.tensor(starts, dtype=torch.int32, device="cuda")
    gl = torch.tensor(plens, dtype=torch.int32, device="cuda")
    mg = max(e - s for s, e in zip(starts[:-1], starts[1:]))
    b.pa_paged_attention_decode_shared_prefix(case.q.cuda(), case.k_pool.cuda(), case.v_pool.cuda(),
                                              case.block_tables.cuda(), case.lengths.cuda(), case.max_len,
                                              case.scale, out, gs, gl, max(plens), mg, partition_size=4096)
    torch.cuda.synchronize()


def test_timeline_build_gives_the_same_bits_and_ordered_stamps():
    import paged_kv_cache_355_b200._binding as b
    from paged_kv_cache_355_b200.build import TIMELINE_LIB
    from paged_kv_cache_355_b200.timeline import _load

    # prefixes of at most 256 tokens: with 4 groups x 8 kv heads the prefix
    # partition stays 256 tokens, so the prefix is one split (prefix-last order)
    groups = [(256, [300, 257, 900, 256]), (128, [200, 129]), (0, [9]), (128, [130] * 3)]
    case, starts, plens = shared_prefix_case(groups, 32, 8, 128, 16, torch.bfloat16, seed=181)
    ref = torch.full((case.q.shape[0], 32, 128), float("nan"), device="cuda")
    _call(b, case, starts, plens, ref)
    assert b.pa_read_error_flag() == 0

    tl = _load(TIMELINE_LIB)
    saved = b._lib
    b._lib = tl
    try:
        assert tl.pa_timeline_clear() == 0
        out = torch.full_like(ref, float("nan"))
        _call(b, case, starts, plens, out)
        assert b.pa_read_error_flag() == 0
        ev = np.zeros(3 * TL_CTAS * TL_SLOTS, np.uint64)
        tt = np.zeros(TT_CTAS * TT_TILES * TT_EVENTS, np.uint64)
        assert tl.pa_timeline_read(0, ev.ctypes.data, ev.nbytes) == 0
        assert tl.pa_timeline_read(1, tt.ctypes.data, tt.nbytes) == 0
        assert tl.pa_timeline_read(2, ev.ctypes.data, 8) != 0
    finally:
        b._lib = saved
    assert torch.equal(out, ref)

    ev = ev.reshape(3, TL_CTAS, TL_SLOTS).astype(np.int64)
    B, Hkv = case.q.shape[0], 8
    # set-up kernel: one CTA, entry <= wait done <= exit
    s = ev[0, 0]
    assert 0 < s[0] <= s[1] <= s[2] and (ev[0, 1:, 0] == 0).all()
    # pass 1: one CTA per (sequence, kv head), all ran to the end
    p1 = ev[2, :B * Hkv]
    assert (p1[:, 0] > 0).all() and (p1[:, 2] >= p1[:, 0]).all() and (ev[2, B * Hkv:, 0] == 0).all()
    streamed = p1[:, 3] > 0  # CTAs whose own tokens filled at least one stage
    assert streamed.sum() == B * Hkv - Hkv  # the member whose whole context is the prefix streams nothing
    q = p1[streamed]
    assert (q[:, 0] <= q[:, 1]).all() and (q[:, 1] <= q[:, 3]).all() and (q[:, 3] <= q[:, 4]).all()
    assert (q[:, 4] <= q[:, 2]).all()
    # prefix pass: CTAs of groups with a prefix ran through; the others left at once
    pre = ev[1][ev[1][:, 0] > 0]
    done = pre[pre[:, 2] > 0]
    assert len(done) == 3 * Hkv  # three groups share a prefix, one CTA per (group, kv head) here
    assert (done[:, 0] <= done[:, 1]).all() and (done[:, 1] <= done[:, 3]).all()
    assert (done[:, 3] <= done[:, 4]).all() and (done[:, 4] <= done[:, 2]).all()
    # the prefix pass runs after pass 1 in this order: it finishes after every pass-1 CTA has started
    assert done[:, 2].max() >= p1[:, 0].max()
    # per-tile events of the first tile of every prefix CTA with work: K request <= S issue <= scores <= P <= P.V
    t = tt.reshape(TT_CTAS, TT_TILES, TT_EVENTS).astype(np.int64)[:, 0]
    t = t[t[:, 0] > 0]
    assert len(t) == 3 * Hkv
    assert (t[:, 5] <= t[:, 4]).all() and (t[:, 4] <= t[:, 0]).all() and (t[:, 0] <= t[:, 1]).all()
    assert (t[:, 1] <= t[:, 3]).all()


def test_prefill_timeline_gives_the_same_bits_and_ordered_stamps():
    """The prefill kernel of the timeline build: bit-identical output, and
    for every CTA with query rows entry <= ready <= first S <= tile 0's last
    P.V <= exit (tile 1's last P.V before the exit when it has rows)."""
    import paged_kv_cache_355_b200._binding as b
    from paged_kv_cache_355_b200.build import TIMELINE_LIB
    from paged_kv_cache_355_b200.timeline import PF_CTAS, PF_SLOTS, _load
    from paged_kv_cache_355_b200.workloads import custom_case

    lengths, news = [700, 300, 129, 64], [700, 170, 1, 64]
    case = custom_case(lengths, 32, 8, 128, 16, torch.bfloat16, seed=191)
    qs = torch.tensor(np.concatenate([[0], np.cumsum(news)]), dtype=torch.int32, device="cuda")
    g = torch.Generator().manual_seed(192)
    q = torch.randn(int(sum(news)), 32, 128, generator=g).to(torch.bfloat16).cuda()
    args = (q, case.k_pool.cuda(), case.v_pool.cuda(), case.block_tables.cuda(), case.lengths.cuda(), qs, max(news),
            case.scale)
    ref = torch.full((q.shape[0], 32, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    b.pa_paged_attention_prefill(*args, ref)
    torch.cuda.synchronize()
    tl = _load(TIMELINE_LIB)
    saved = b._lib
    b._lib = tl
    try:
        assert tl.pa_timeline_clear_prefill() == 0
        out = torch.full_like(ref, float("nan"))
        b.pa_paged_attention_prefill(*args, out)
        torch.cuda.synchronize()
        assert b.pa_read_error_flag() == 0
        ev = np.zeros(PF_CTAS * PF_SLOTS, np.uint64)
        assert tl.pa_timeline_read_prefill(ev.ctypes.data, ev.nbytes) == 0
        assert tl.pa_timeline_read_prefill(ev.ctypes.data, ev.nbytes + 8) != 0
    finally:
        b._lib = saved
    assert torch.equal(out, ref)
    e = ev.reshape(PF_CTAS, PF_SLOTS).astype(np.int64)
    e = e[e[:, 0] > 0]
    # CTAs with rows: pairs of 32-token tiles (G = 4) per (sequence, kv head)
    assert len(e) == 8 * sum(-(-n // 64) for n in news)
    assert (e[:, 0] <= e[:, 1]).all() and (e[:, 1] <= e[:, 2]).all() and (e[:, 2] <= e[:, 3]).all()
    assert (e[:, 3] <= e[:, 5]).all()
    two = e[:, 4] > 0
    assert (e[two, 4] <= e[two, 5]).all() and two.any() and (~two).any()
    assert (e[:, PF_SLOTS - 1] < torch.cuda.get_device_properties(0).multi_processor_count).all()
