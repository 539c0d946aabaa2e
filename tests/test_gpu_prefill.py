"""GPU parity of causal multi-query paged attention (tcgen05 kernel) against
the fp64 oracle: chunks that are whole sequences or their tails, every group
size and block size, ragged lengths across tile boundaries, NaN-poisoned
slots past each sequence, and the single-token case against decode."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_355_b200.workloads import custom_case
from tests.helpers import assert_matches_oracle, np_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    import paged_kv_cache_355_b200 as pa

    assert torch.cuda.is_available()
    pa.pa_read_error_flag()
    return pa


def _run(pa, case, news, out_dtype=torch.float32, k_pool=None, v_pool=None):
    """Prefill with news[b] query tokens at the end of each sequence."""
    Hq, D = case.q.shape[1], case.q.shape[2]
    qs = np.concatenate([[0], np.cumsum(news)]).astype(np.int32)
    T = int(qs[-1])
    g = torch.Generator().manual_seed(T + Hq)
    q = torch.randn(T, Hq, D, generator=g).to(torch.bfloat16)
    kp = case.k_pool if k_pool is None else k_pool
    vp = case.v_pool if v_pool is None else v_pool
    out = torch.full((T, Hq, D), float("nan"), dtype=out_dtype, device="cuda")
    pa.pa_paged_attention_prefill(q.cuda(), kp.cuda(), vp.cuda(), case.block_tables.cuda(), case.lengths.cuda(),
                                  torch.from_numpy(qs).cuda(), int(max(news)), case.scale, out)
    torch.cuda.synchronize()
    ref = oracle.paged_prefill(np_of(q), np_of(kp), np_of(vp), np_of(case.block_tables), np_of(case.lengths), qs,
                               case.scale, case.workload.block_size)
    return out, ref


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_prefill_sweep(pa, D, bs, G):
    Hkv = 2
    lengths = [1, 63, 64, 65, 200, 300]
    news = [1, 63, 10, 65, 130, 1]
    case = custom_case(lengths, Hkv * G, Hkv, D, bs, torch.bfloat16, seed=D + bs + G)
    out, ref = _run(pa, case, news)
    assert_matches_oracle(out, ref, True, f"prefill D{D} bs{bs} G{G}")
    assert pa.pa_read_error_flag() == 0


def test_prefill_long_chunk_and_bf16_out(pa):
    case = custom_case([1500, 700, 2048], 32, 8, 128, 16, torch.bfloat16, seed=5)
    out, ref = _run(pa, case, [1500, 256, 129], out_dtype=torch.bfloat16)
    assert_matches_oracle(out, ref, True, "prefill long")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_prefill_bf16_out_every_shape(pa, D, G):
    """bf16 output, whose whole query tiles leave through shared memory by
    tiled TMA stores (box: 64 dims x G heads x 128 / G tokens) while partial
    tiles store rows directly: chunks of whole tiles, whole tiles plus a
    ragged tail, and a sequence's first tokens, for every head_dim and group
    size."""
    TQ = 128 // G
    lengths = [4 * TQ + 37, 6 * TQ, 2 * TQ + 1, 300]
    news = [4 * TQ, 6 * TQ, 2 * TQ + 1, 5]
    case = custom_case(lengths, 2 * G, 2, D, 16, torch.bfloat16, seed=70 + D + G)
    out, ref = _run(pa, case, news, out_dtype=torch.bfloat16)
    assert_matches_oracle(out, ref, True, f"prefill bf16 out D{D} G{G}")
    assert pa.pa_read_error_flag() == 0


def test_prefill_single_token_equals_decode(pa):
    case = custom_case([5, 77, 300, 1], 16, 4, 128, 16, torch.bfloat16, seed=6)
    out, ref = _run(pa, case, [1, 1, 1, 1])
    dec = torch.empty_like(out)
    qs = np.arange(5, dtype=np.int32)
    g = torch.Generator().manual_seed(4 + 16)
    q = torch.randn(4, 16, 128, generator=g).to(torch.bfloat16)
    pa.pa_paged_attention_decode(q.cuda(), case.k_pool.cuda(), case.v_pool.cuda(), case.block_tables.cuda(),
                                 case.lengths.cuda(), case.max_len, case.scale, dec)
    torch.cuda.synchronize()
    assert_matches_oracle(out, ref, True, "prefill n=1")
    assert_matches_oracle(dec, ref, True, "decode vs prefill oracle")


@pytest.mark.parametrize("scale", [-0.0883883461356163, 0.0])
def test_prefill_nonpositive_scale(pa, scale):
    """A negative or zero scale takes the kernel's scale-first path (a positive
    one folds the scale into the exponent); scale 0 is the plain average of
    the visible V rows."""
    case = custom_case([90, 300], 8, 2, 128, 16, torch.bfloat16, seed=11)
    case.scale = float(np.float32(scale))
    out, ref = _run(pa, case, [90, 170])
    assert_matches_oracle(out, ref, True, f"prefill scale {scale}")
    assert pa.pa_read_error_flag() == 0


def test_prefill_empty_chunks_and_empty_sequence(pa):
    """Sequences with no new tokens (one of them empty) take no query rows and
    leave their neighbours' rows exact; max_query_len above the longest chunk
    only adds CTAs that exit at once."""
    case = custom_case([0, 50, 300, 7, 129], 16, 4, 64, 16, torch.bfloat16, seed=12)
    Hq, D = 16, 64
    news = [0, 0, 130, 7, 0]
    qs = np.concatenate([[0], np.cumsum(news)]).astype(np.int32)
    T = int(qs[-1])
    g = torch.Generator().manual_seed(13)
    q = torch.randn(T, Hq, D, generator=g).to(torch.bfloat16)
    out = torch.full((T, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    pa.pa_paged_attention_prefill(q.cuda(), case.k_pool.cuda(), case.v_pool.cuda(), case.block_tables.cuda(),
                                  case.lengths.cuda(), torch.from_numpy(qs).cuda(), 512, case.scale, out)
    torch.cuda.synchronize()
    ref = oracle.paged_prefill(np_of(q), np_of(case.k_pool), np_of(case.v_pool), np_of(case.block_tables),
                               np_of(case.lengths), qs, case.scale, 16)
    assert_matches_oracle(out, ref, True, "empty chunks")
    assert pa.pa_read_error_flag() == 0


@pytest.mark.parametrize("seed", range(6))
def test_prefill_random_shapes(pa, seed):
    """Seeded random head_dim, block size, group size, batch, lengths and
    chunk sizes (zero-length chunks included), four cases per seed."""
    rng = np.random.default_rng(100 + seed)
    for it in range(4):
        D = int(rng.choice([64, 128]))
        bs = int(rng.choice([8, 16, 32]))
        G = int(rng.choice([1, 2, 4, 8, 16]))
        Hkv = int(rng.integers(1, 3))
        lengths = [int(x) for x in rng.integers(1, 700, int(rng.integers(1, 5)))]
        news = [int(rng.integers(0, L + 1)) for L in lengths]
        if sum(news) == 0:
            news[0] = lengths[0]
        case = custom_case(lengths, Hkv * G, Hkv, D, bs, torch.bfloat16, seed=1000 * seed + it)
        out, ref = _run(pa, case, news)
        assert_matches_oracle(out, ref, True, f"random prefill seed {seed}.{it} D{D} bs{bs} G{G} {lengths} {news}")
    assert pa.pa_read_error_flag() == 0


def test_prefill_never_reads_past_the_sequence(pa):
    lengths = [40, 129, 17]
    case = custom_case(lengths, 8, 2, 128, 16, torch.bfloat16, seed=7, extra_blocks=6)
    kp, vp = case.k_pool.clone(), case.v_pool.clone()
    used = torch.zeros(case.num_blocks, 16, dtype=torch.bool)
    for b, L in enumerate(lengths):
        for t in range(L):
            used[case.block_tables[b, t // 16], t % 16] = True
    kp.permute(0, 2, 1, 3)[~used] = float("nan")
    vp.permute(0, 2, 1, 3)[~used] = float("nan")
    out, ref = _run(pa, case, [40, 70, 3], k_pool=kp, v_pool=vp)
    assert_matches_oracle(out, ref, True, "poisoned slots")
    assert pa.pa_read_error_flag() == 0


def test_prefill_rejects_fp32(pa):
    case = custom_case([8], 4, 4, 64, 16, torch.float32, seed=8)
    q = torch.zeros(8, 4, 64, device="cuda")
    with pytest.raises(pa.PAError, match="UNSUPPORTED"):
        pa.pa_paged_attention_prefill(q, case.k_pool.cuda(), case.v_pool.cuda(), case.block_tables.cuda(),
                                      case.lengths.cuda(), torch.tensor([0, 8], dtype=torch.int32, device="cuda"), 8,
                                      case.scale, torch.empty(8, 4, 64, device="cuda"))


@pytest.mark.parametrize("G", [4, 16])
def test_prefill_many_items_per_cta(pa, G):
    """Far more work items (pairs of query tiles per sequence and kv head)
    than SMs, of mixed shapes: chunks of random length (zero, odd tile counts,
    whole sequences), so that every CTA of the kernel takes many items,
    among them empty ones and ones where the second tile has no rows."""
    rng = np.random.default_rng(41 + G)
    B, Hkv = 48, 8 if G == 4 else 2
    lengths = [int(x) for x in rng.integers(1, 400, B)]
    news = [int(rng.integers(0, L + 1)) if i % 5 else L for i, L in enumerate(lengths)]
    news[3] = 0
    case = custom_case(lengths, Hkv * G, Hkv, 128, 16, torch.bfloat16, seed=43 + G)
    out, ref = _run(pa, case, news)
    assert_matches_oracle(out, ref, True, f"many items G{G}")
    assert pa.pa_read_error_flag() == 0


# The chunked-prefill workload the benchmark times: batch 8, 32 q / 8 kv heads,
# head_dim 128, bs 16, context 4096 of which the last 2048 tokens are new.
FULL = (8, 32, 8, 128, 16, 4096, 2048)
SAMPLED_TOKENS = [0, 1, 31, 32, 63, 64, 127, 128, 1023, 1024, 2015, 2046, 2047]


@pytest.mark.parametrize("q_scale", [1.0, 4.0], ids=["as_benchmarked", "peaked"])
def test_prefill_full_size_sampled_rows(pa, q_scale):
    """The full chunked-prefill workload, built and launched as the benchmark
    does (same seeds, bf16 output, the whole grid), with sampled query tokens
    of every sequence (all 32 heads: tile edges, both ends of the chunk, plus
    seeded random ones) against the oracle.  A query at position p attends
    keys 0..p, so its row is decode attention over a sequence of length p + 1
    with the same block table.  q scaled by 4 makes the softmax peaked, the
    case where a bf16 P without its residual part leaves the bar."""
    B, Hq, Hkv, D, bs, L, n = FULL
    dev = torch.device("cuda", 0)
    case = custom_case([L] * B, Hq, Hkv, D, bs, torch.bfloat16, seed=2001, device=dev)
    qs = torch.arange(0, (B + 1) * n, n, dtype=torch.int32, device=dev)
    g = torch.Generator(device=dev).manual_seed(2002)
    q = (torch.randn(B * n, Hq, D, generator=g, device=dev) * q_scale).to(torch.bfloat16)
    out = torch.full((B * n, Hq, D), float("nan"), dtype=torch.bfloat16, device=dev)
    bt, lens = case.block_tables.to(dev), case.lengths.to(dev)
    pa.pa_paged_attention_prefill(q, case.k_pool, case.v_pool, bt, lens, qs, n, case.scale, out)
    torch.cuda.synchronize()
    assert pa.pa_read_error_flag() == 0
    rng = np.random.default_rng(2003)
    rows = []  # (sequence, query token)
    for b in range(B):
        toks = sorted(set(SAMPLED_TOKENS) | set(int(x) for x in rng.integers(0, n, 3)))
        rows += [(b, i) for i in toks]
    sel = torch.tensor([b * n + i for b, i in rows], dtype=torch.long)
    q_rows = q.cpu()[sel]
    bt_rows = np_of(case.block_tables)[[b for b, _ in rows]]
    len_rows = np.array([L - n + i + 1 for _, i in rows], np.int32)
    ref = oracle.paged_decode(np_of(q_rows), np_of(case.k_pool), np_of(case.v_pool), bt_rows, len_rows,
                              case.scale, bs)
    got = out.cpu()[sel]
    assert_matches_oracle(got, ref, True, f"full-size prefill, q x {q_scale}")
