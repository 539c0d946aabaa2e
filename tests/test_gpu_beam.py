"""Beam / tree search forking on the paged cache: repeated fork and free with
copy-on-write at arbitrary depth ("How does vLLM PagedAttention manage
Virtual Memory Pages ...", "Key Technical Innovations" item 3; "PagedAttention
and KV memory management", "In practice" item 4).

Each step every surviving beam picks a parent, children fork from their
parents (sharing all blocks), the beams not chosen are freed, and each child
appends one token.  The native block manager (libpa) decides slots and
copy-on-write pairs; the GPU runs copy_blocks, reshape_and_cache and decode
attention.  The oracle side replays the same decisions with the oracle's
block manager and CPU ops: slots, pairs and pools must match bit for bit and
the attention within the bf16 tolerance."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle.block_manager import BlockManager as RefManager
from tests.helpers import assert_matches_oracle, np_of

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bs,width,children", [(16, 4, None), (8, 6, None), (16, 3, (1, 3))])
def test_beam_search_forking_matches_oracle(bs, width, children):
    from paged_kv_cache_355_b200 import _binding as pa
    from paged_kv_cache_355_b200.block_manager import BlockManager

    rng = np.random.default_rng(bs * 10 + width)
    g = torch.Generator().manual_seed(bs + width)
    NB, Hq, Hkv, D, prompt, steps = 512, 16, 4, 128, 37, 9
    scale = float(np.float32(1.0 / np.sqrt(D)))
    k_pool = torch.randn(NB, Hkv, bs, D, generator=g).to(torch.bfloat16)
    v_pool = torch.randn(NB, Hkv, bs, D, generator=g).to(torch.bfloat16)
    gk, gv = k_pool.cuda(), v_pool.cuda()
    hk, hv = np_of(k_pool).copy(), np_of(v_pool).copy()
    nat, ref = BlockManager(NB, bs), RefManager(NB, bs)

    def append(seqs, key, val):
        slots, pairs = nat.append_tokens(seqs)
        ref_slots, ref_pairs = [], []
        for s in seqs:
            slot, ps = ref.append_token(s)
            ref_slots.append(slot)
            ref_pairs += ps
        assert slots.tolist() == ref_slots and [tuple(p) for p in pairs.tolist()] == ref_pairs
        if len(pairs):
            pa.pa_copy_blocks(gk, gv, torch.from_numpy(pairs).cuda())
            oracle.copy_blocks(hk, hv, pairs)
        pa.pa_reshape_and_cache(key.cuda(), val.cuda(), gk, gv, torch.from_numpy(slots).cuda())
        oracle.reshape_and_cache(np_of(key), np_of(val), hk, hv, slots)
        return len(pairs)

    # the prompt, written in one go for beam 0
    append([0] * prompt, torch.randn(prompt, Hkv, D, generator=g).to(torch.bfloat16),
           torch.randn(prompt, Hkv, D, generator=g).to(torch.bfloat16))
    beams, next_id, copies = [0], 1, 0
    for step in range(steps):
        parents = []
        for _ in range(width):
            parents.append(int(rng.choice(beams)))
        if children:  # tree search: some parents spawn several children, others none
            parents = [int(b) for b in rng.choice(beams, size=int(rng.integers(*children)) * len(beams))][:width] or beams
        new = []
        for p in parents:
            nat.fork(p, next_id)
            ref.fork(p, next_id)
            new.append(next_id)
            next_id += 1
        for b in beams:
            nat.free_sequence(b)
            ref.free_sequence(b)
        beams = new
        key = torch.randn(len(beams), Hkv, D, generator=g).to(torch.bfloat16)
        val = torch.randn(len(beams), Hkv, D, generator=g).to(torch.bfloat16)
        copies += append(beams, key, val)
        assert nat.free_list() == list(ref.free)
        # decode attention for every beam over its (partly shared) blocks
        width_tbl = max(len(ref.block_table(b)) for b in beams)
        tables, lens = nat.block_tables(beams, width_tbl)
        ref_tables = np.full((len(beams), width_tbl), -1, np.int32)
        for i, b in enumerate(beams):
            ref_tables[i, : len(ref.block_table(b))] = ref.block_table(b)
        assert np.array_equal(tables, ref_tables)
        q = torch.randn(len(beams), Hq, D, generator=g).to(torch.bfloat16)
        out = torch.empty(len(beams), Hq, D, device="cuda")
        pa.pa_paged_attention_decode(q.cuda(), gk, gv, torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                                     int(lens.max()), scale, out, partition_size=32)
        torch.cuda.synchronize()
        want = oracle.paged_decode(np_of(q), hk, hv, tables, lens, scale, bs)
        assert_matches_oracle(out, want, True, f"beam step {step}")
        assert np_of(gk).tobytes() == hk.tobytes() and np_of(gv).tobytes() == hv.tobytes()
    assert copies > 0  # forks into partial blocks really exercised copy-on-write
    assert pa.pa_read_error_flag() == 0
