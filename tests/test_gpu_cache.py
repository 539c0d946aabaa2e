"""GPU parity of the cache kernels: slot mapping, reshape_and_cache and
copy_blocks must match the oracle bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import np_of

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_355_b200 as pa

    assert torch.cuda.is_available()
    pa.pa_read_error_flag()  # clear
    return pa


def test_slot_mapping_bit_exact(pa):
    g = torch.Generator().manual_seed(5)
    for bs in (8, 16, 32):
        B, MBS = 37, 9
        bt = torch.randperm(B * MBS + 11, generator=g)[: B * MBS].reshape(B, MBS).to(torch.int32)
        T = 500
        sid = torch.randint(0, B, (T,), generator=g, dtype=torch.int32)
        pos = torch.randint(0, MBS * bs, (T,), generator=g, dtype=torch.int32)
        want = oracle.slot_mapping(np_of(bt), np_of(sid), np_of(pos), bs)
        got = torch.empty(T, dtype=torch.int64, device="cuda")
        pa.pa_slot_mapping(bt.cuda(), sid.cuda(), pos.cuda(), bs, got)
        assert np.array_equal(np_of(got), want)
        # decode form: the last token of each sequence
        lens = torch.randint(1, MBS * bs + 1, (B,), generator=g, dtype=torch.int32)
        want = oracle.slot_mapping(np_of(bt), np.arange(B, dtype=np.int32), np_of(lens) - 1, bs)
        got = torch.empty(B, dtype=torch.int64, device="cuda")
        pa.pa_decode_slot_mapping(bt.cuda(), lens.cuda(), bs, got)
        assert np.array_equal(np_of(got), want)
    assert pa.pa_read_error_flag() == 0


def test_slot_mapping_flags_unmapped_tokens(pa):
    bt = torch.tensor([[4, -1], [7, 2]], dtype=torch.int32, device="cuda")
    sid = torch.tensor([0, 0, 1, 3], dtype=torch.int32, device="cuda")
    pos = torch.tensor([3, 20, 20, 0], dtype=torch.int32, device="cuda")
    got = torch.empty(4, dtype=torch.int64, device="cuda")
    pa.pa_slot_mapping(bt, sid, pos, 16, got)
    assert got.tolist() == [4 * 16 + 3, -1, 2 * 16 + 4, -1]
    assert pa.pa_read_error_flag() == 5
    lens = torch.tensor([0, 17], dtype=torch.int32, device="cuda")
    got = torch.empty(2, dtype=torch.int64, device="cuda")
    pa.pa_decode_slot_mapping(bt, lens, 16, got)
    assert got.tolist() == [-1, 2 * 16 + 0]
    assert pa.pa_read_error_flag() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_reshape_and_cache_bit_exact(pa, dtype, D, bs):
    g = torch.Generator().manual_seed(D + bs)
    NB, Hkv, T = 40, 4, 150
    k_pool = torch.randn(NB, Hkv, bs, D, generator=g).to(DT[dtype])
    v_pool = torch.randn(NB, Hkv, bs, D, generator=g).to(DT[dtype])
    key = torch.randn(T, Hkv, D, generator=g).to(DT[dtype])
    val = torch.randn(T, Hkv, D, generator=g).to(DT[dtype])
    slots = torch.randperm(NB * bs, generator=g)[:T].to(torch.int64)
    slots[::7] = -1
    kp, vp = np_of(k_pool).copy(), np_of(v_pool).copy()
    oracle.reshape_and_cache(np_of(key), np_of(val), kp, vp, np_of(slots))
    gk, gv = k_pool.cuda(), v_pool.cuda()
    pa.pa_reshape_and_cache(key.cuda(), val.cuda(), gk, gv, slots.cuda())
    assert np_of(gk).tobytes() == kp.tobytes()
    assert np_of(gv).tobytes() == vp.tobytes()
    assert pa.pa_read_error_flag() == 0


def test_reshape_and_cache_flags_slot_outside_pool(pa):
    k_pool = torch.zeros(2, 1, 8, 64, device="cuda")
    v_pool = torch.zeros_like(k_pool)
    key = torch.ones(2, 1, 64, device="cuda")
    slots = torch.tensor([3, 16], dtype=torch.int64, device="cuda")
    pa.pa_reshape_and_cache(key, key, k_pool, v_pool, slots)
    assert pa.pa_read_error_flag() == 5
    assert k_pool[0, 0, 3].eq(1).all() and k_pool.sum().item() == 64


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_fused_decode_write_matches_two_step_oracle(pa, dtype, D, bs):
    """pa_reshape_and_cache_decode = decode slot mapping + cache write, bit for bit,
    with a length-0 sequence in the batch (no write, slot -1)."""
    g = torch.Generator().manual_seed(3 * D + bs)
    B, MBS, Hkv = 45, 7, 4
    NB = B * MBS + 5
    bt = torch.randperm(NB, generator=g)[: B * MBS].reshape(B, MBS).to(torch.int32)
    lens = torch.randint(1, MBS * bs + 1, (B,), generator=g, dtype=torch.int32)
    lens[3] = 0
    lens[4] = MBS * bs  # last slot of the last block
    k_pool = torch.randn(NB, Hkv, bs, D, generator=g).to(DT[dtype])
    v_pool = torch.randn(NB, Hkv, bs, D, generator=g).to(DT[dtype])
    key = torch.randn(B, Hkv, D, generator=g).to(DT[dtype])
    val = torch.randn(B, Hkv, D, generator=g).to(DT[dtype])
    pos = np_of(lens) - 1
    pos[3] = 0  # the empty sequence writes nothing: its slot is -1 below
    want_slots = oracle.slot_mapping(np_of(bt), np.arange(B, dtype=np.int32), pos, bs)
    want_slots[3] = -1
    kp, vp = np_of(k_pool).copy(), np_of(v_pool).copy()
    oracle.reshape_and_cache(np_of(key), np_of(val), kp, vp, want_slots)
    gk, gv = k_pool.cuda(), v_pool.cuda()
    got = torch.full((B,), 7, dtype=torch.int64, device="cuda")
    pa.pa_reshape_and_cache_decode(key.cuda(), val.cuda(), gk, gv, bt.cuda(), lens.cuda(), got)
    assert np.array_equal(np_of(got), want_slots)
    assert np_of(gk).tobytes() == kp.tobytes()
    assert np_of(gv).tobytes() == vp.tobytes()
    # without the slot output the pools come out the same
    gk2, gv2 = k_pool.cuda(), v_pool.cuda()
    pa.pa_reshape_and_cache_decode(key.cuda(), val.cuda(), gk2, gv2, bt.cuda(), lens.cuda())
    assert torch.equal(gk2, gk) and torch.equal(gv2, gv)
    assert pa.pa_read_error_flag() == 0


def test_fused_decode_write_flags_bad_entries(pa):
    k_pool = torch.zeros(2, 1, 8, 64, device="cuda")
    v_pool = torch.zeros_like(k_pool)
    key = torch.ones(4, 1, 64, device="cuda")
    bt = torch.tensor([[1, -1], [1, 0], [5, 0], [0, 1]], dtype=torch.int32, device="cuda")
    # seq 0: unmapped block; seq 1: slot 0*8+0; seq 2: block 5 outside a 2-block pool; seq 3: length 0
    lens = torch.tensor([9, 9, 3, 0], dtype=torch.int32, device="cuda")
    got = torch.empty(4, dtype=torch.int64, device="cuda")
    pa.pa_reshape_and_cache_decode(key, 2 * key, k_pool, v_pool, bt, lens, got)
    assert got.tolist() == [-1, 0, 5 * 8 + 2, -1]
    assert pa.pa_read_error_flag() == 5
    assert k_pool[0, 0, 0].eq(1).all() and k_pool.sum().item() == 64
    assert v_pool[0, 0, 0].eq(2).all() and v_pool.sum().item() == 128


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_copy_blocks_bit_exact(pa, dtype, bs):
    g = torch.Generator().manual_seed(bs)
    NB, Hkv, D = 64, 8, 128
    k_pool = torch.randn(NB, Hkv, bs, D, generator=g).to(DT[dtype])
    v_pool = torch.randn(NB, Hkv, bs, D, generator=g).to(DT[dtype])
    perm = torch.randperm(NB, generator=g)
    pairs = torch.stack([perm[:20], perm[20:40]], 1).to(torch.int64)  # distinct dsts, no dst is a src
    kp, vp = np_of(k_pool).copy(), np_of(v_pool).copy()
    oracle.copy_blocks(kp, vp, np_of(pairs))
    gk, gv = k_pool.cuda(), v_pool.cuda()
    pa.pa_copy_blocks(gk, gv, pairs.cuda())
    assert np_of(gk).tobytes() == kp.tobytes()
    assert np_of(gv).tobytes() == vp.tobytes()
    assert pa.pa_read_error_flag() == 0


def test_copy_blocks_flags_bad_pair(pa):
    k_pool = torch.arange(4 * 64, dtype=torch.float32, device="cuda").reshape(4, 1, 1, 64).expand(4, 1, 8, 64)
    k_pool = k_pool.contiguous()
    v_pool = k_pool.clone()
    before = k_pool.clone()
    pa.pa_copy_blocks(k_pool, v_pool, torch.tensor([[0, 9], [1, 2]], dtype=torch.int64, device="cuda"))
    assert pa.pa_read_error_flag() == 5
    assert torch.equal(k_pool[2], before[1]) and torch.equal(k_pool[0], before[0])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_swap_out_and_in_through_pinned_host_memory(pa, dtype):
    """Blocks swapped to a pinned host pool and back are bit-identical, and the
    host pool holds exactly the swapped blocks (oracle: a numpy copy)."""
    g = torch.Generator().manual_seed(7)
    NB, HNB, Hkv, bs, D = 64, 24, 8, 16, 128
    k = torch.randn(NB, Hkv, bs, D, generator=g).to(DT[dtype]).cuda()
    v = torch.randn(NB, Hkv, bs, D, generator=g).to(DT[dtype]).cuda()
    hk = torch.zeros(HNB, Hkv, bs, D, dtype=DT[dtype]).pin_memory()
    hv = torch.zeros(HNB, Hkv, bs, D, dtype=DT[dtype]).pin_memory()
    src = torch.randperm(NB, generator=g)[:20]
    dst = torch.randperm(HNB, generator=g)[:20]
    out_map = torch.stack([src, dst], 1).to(torch.int64)
    k0, v0 = k.clone(), v.clone()
    pa.pa_swap_blocks(k, v, hk, hv, out_map.cuda())  # swap out: device -> host
    torch.cuda.synchronize()
    want_k, want_v = np.zeros_like(np_of(hk)), np.zeros_like(np_of(hv))
    want_k[np_of(dst)] = np_of(k0)[np_of(src)]
    want_v[np_of(dst)] = np_of(v0)[np_of(src)]
    assert np_of(hk).tobytes() == want_k.tobytes() and np_of(hv).tobytes() == want_v.tobytes()
    k[src] = 0  # the device blocks are reused by someone else meanwhile
    v[src] = 0
    new_home = torch.randperm(NB, generator=g)[:20]
    in_map = torch.stack([dst, new_home], 1).to(torch.int64).pin_memory()  # mapping read from host memory too
    pa.pa_swap_blocks(hk, hv, k, v, in_map)  # swap in: host -> device, to new block ids
    torch.cuda.synchronize()
    assert torch.equal(k[new_home].cpu(), k0[src].cpu()) and torch.equal(v[new_home].cpu(), v0[src].cpu())
    assert pa.pa_read_error_flag() == 0


def test_swap_bandwidth_is_reported(pa):
    """Swap 2048 blocks (256 MiB of K+V at 8 heads, bs 16, D 128, bf16) each
    way and print the achieved host-link bandwidth (no bound asserted)."""
    NB, Hkv, bs, D = 2048, 8, 16, 128
    k = torch.empty(NB, Hkv, bs, D, dtype=torch.bfloat16, device="cuda").normal_()
    v = torch.empty_like(k).normal_()
    hk = torch.empty(NB, Hkv, bs, D, dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    m = torch.stack([torch.arange(NB), torch.randperm(NB)], 1).to(torch.int64).cuda()
    nbytes = 2 * k.numel() * k.element_size()
    for name, args in (("device->host", (k, v, hk, hv)), ("host->device", (hk, hv, k, v))):
        pa.pa_swap_blocks(*args, m)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        pa.pa_swap_blocks(*args, m)
        e1.record()
        torch.cuda.synchronize()
        print(f"swap {name}: {nbytes / e0.elapsed_time(e1) / 1e6:.1f} GB/s")
    assert pa.pa_read_error_flag() == 0
