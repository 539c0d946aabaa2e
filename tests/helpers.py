"""Test-side helpers: lay logical token data out in a block pool, dtype views.

The pool layout is [num_blocks, Hkv, block_size, D]; token t of a sequence
whose block table is ``table`` lives at pool[table[t // bs], :, t % bs, :].
This is the layout definition written as a scatter, independently of the
oracle's gather.
"""
from __future__ import annotations

import numpy as np


def place_logical(logical_k, logical_v, tables, num_blocks, block_size, fill=0.0):
    """logical_k[b]: array [L_b, Hkv, D] -> (k_pool, v_pool) float32 arrays.

    tables[b] lists the physical blocks of sequence b in logical order.
    Slots that hold no token are set to ``fill``.
    """
    Hkv, D = None, None
    for lk in logical_k:
        if len(lk):
            Hkv, D = lk.shape[1], lk.shape[2]
            break
    assert Hkv is not None
    k_pool = np.full((num_blocks, Hkv, block_size, D), fill, np.float32)
    v_pool = np.full((num_blocks, Hkv, block_size, D), fill, np.float32)
    for b, (lk, lv) in enumerate(zip(logical_k, logical_v)):
        for t in range(len(lk)):
            phys = tables[b][t // block_size]
            off = t % block_size
            for h in range(Hkv):
                k_pool[phys, h, off, :] = lk[t, h, :]
                v_pool[phys, h, off, :] = lv[t, h, :]
    return k_pool, v_pool


def pad_tables(tables, width, pad=-1):
    """List of per-sequence block lists -> int32 [B, width], padded with ``pad``."""
    out = np.full((len(tables), max(width, 1)), pad, np.int32)
    for b, row in enumerate(tables):
        out[b, : len(row)] = row
    return out


def random_tables(rng, lengths, block_size, num_blocks):
    """Scatter every sequence's logical blocks over distinct random physical ids."""
    need = [-(-L // block_size) for L in lengths]
    assert sum(need) <= num_blocks
    ids = rng.permutation(num_blocks)
    tables, at = [], 0
    for n in need:
        tables.append([int(x) for x in ids[at: at + n]])
        at += n
    return tables


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 bits via torch (round to nearest even)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def to_logical_lists(arr_list):
    """[array [L, Hkv, D]] -> nested python lists for the brute force."""
    return [[[list(map(float, arr[t, h])) for h in range(arr.shape[1])] for t in range(arr.shape[0])]
            for arr in arr_list]


# ---------------------------------------------------------------------------
# GPU-test helpers: hand tensors to the oracle, compare against it
# ---------------------------------------------------------------------------
def np_of(t):
    """torch tensor (any device) -> numpy array in the oracle's conventions
    (fp32 as float32, bf16 as its raw uint16 bits, integers as they are)."""
    import torch

    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


# Tolerances of paged decode attention against the fp64 oracle:
# fp32 inputs: max |delta| <= 1e-5; bf16 inputs (fp32 accumulation):
# max |delta| <= 2e-3 and every |delta| <= 2e-3 + 1e-2 * |oracle|.
F32_ATOL = 1e-5
BF16_ATOL, BF16_RTOL = 2e-3, 1e-2


def assert_matches_oracle(got, ref, kv_is_bf16: bool, what: str = ""):
    import torch

    if got.dtype == torch.bfloat16:
        return assert_bf16_output_matches_oracle(got, ref, what)
    g = got.detach().float().cpu().double().numpy()
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    if kv_is_bf16:
        bad = err > BF16_ATOL + BF16_RTOL * np.abs(ref)
        assert err.max() <= BF16_ATOL and not bad.any(), (
            f"{what}: max|d|={err.max():.3e}, {int(bad.sum())} elements outside allclose(2e-3, 1e-2)")
    else:
        assert err.max() <= F32_ATOL, f"{what}: max|d|={err.max():.3e} > {F32_ATOL}"
    return float(err.max())


def assert_bf16_output_matches_oracle(got, ref, what: str = ""):
    """bf16 OUTPUT: the max-abs bound does not apply (one bf16 rounding of a
    value near 2 is already 4e-3); every element must satisfy
    allclose(2e-3, 1e-2) and lie within one bf16 step of the oracle rounded
    once to bf16, or within 1e-5 of the oracle."""
    import oracle
    import torch

    ref = np.asarray(ref, np.float64)
    bits = got.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    g = oracle.bf16_bits_to_f64(bits)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    bad = err > BF16_ATOL + BF16_RTOL * np.abs(ref)
    assert not bad.any(), f"{what}: {int(bad.sum())} elements outside allclose(2e-3, 1e-2)"
    ref_bits = oracle.round_bf16(ref).astype(np.int32)
    # ordered integer view of bf16 bit patterns: adjacent values differ by 1
    def ordered(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    steps = np.abs(ordered(bits) - ordered(ref_bits))
    # near zero a bf16 step is far below the fp32 accumulation error (which
    # scales with |V|, not with the output), so 1e-5 absolute also passes
    far = (steps > 1) & (err > F32_ATOL)
    assert not far.any(), f"{what}: {int(far.sum())} elements more than one bf16 step (and 1e-5) from the oracle"
    return float(err.max())


def shared_prefix_case(groups, num_q_heads, num_kv_heads, head_dim, block_size, dtype, seed=0, extra_blocks=4):
    """A decode case whose sequences come in groups sharing a prompt.

    groups: list of (prefix_len, [member lengths]); prefix_len is a multiple
    of block_size and at most every member's length.  Each group's first
    prefix_len / block_size blocks are the same physical ids in every
    member's table; every other block is private.  Blocks are scattered over
    the pool.  Returns (case, group_starts, group_prefix_lens) with the two
    lists as the shared-prefix call takes them."""
    import torch

    from paged_kv_cache_355_b200.workloads import Workload, build_case

    bs = block_size
    need = 0
    for P, members in groups:
        assert P % bs == 0 and all(L >= P for L in members)
        need += P // bs + sum(-(-L // bs) - P // bs for L in members)
    nb = need + extra_blocks
    ids = iter(torch.randperm(nb, generator=torch.Generator().manual_seed(seed + 1)).tolist())
    tables, lengths, starts, plens = [], [], [0], []
    for P, members in groups:
        shared = [next(ids) for _ in range(P // bs)]
        for L in members:
            t = list(shared)
            while len(t) < -(-L // bs):
                t.append(next(ids))
            tables.append(t)
            lengths.append(L)
        starts.append(len(lengths))
        plens.append(P)
    w = Workload("shared", len(lengths), num_q_heads, num_kv_heads, head_dim, bs, dtype, "fixed")
    sid = [b for b, L in enumerate(lengths) if L > 0]
    case = build_case(w, lengths, tables, nb, sid, [lengths[b] - 1 for b in sid], None, seed + 2)
    return case, starts, plens
