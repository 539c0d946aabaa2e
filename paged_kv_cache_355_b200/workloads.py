"""Seeded synthetic decode workloads.

This module only draws inputs: lengths, block placements and N(0, 1) values.
It holds none of the attention, slot or copy arithmetic, and is shared by the
tests, the benchmark and the oracle-side checks so that both sides see the
same bytes.

Workloads (sizes as named; "length" is the context length INCLUDING the token
written in this decode step, which sits at position length - 1):

  tiny      4 sequences of 1, 7, 16, 33 tokens that each append one token
            (lengths 2, 8, 17, 34), 4 query = 4 kv heads, head_dim 64,
            block_size 16, fp32, a 64-block pool handed out in the order of
            a seeded random permutation, scale 1/sqrt(64).
  llama7b   batch 64, 32 = 32 heads, head_dim 128, block_size 16, bf16,
            lengths uniform in [128, 2048], blocks drawn without replacement
            from a pool of 1.25x the blocks needed.
  gqa       batch 256, 32 query / 8 kv heads, head_dim 128, block_size 16,
            bf16, lengths lognormal (median 1000, sigma 0.8) rounded and
            clipped to [16, 4096], blocks scattered over a 1.25x pool.
  cow       32 prompts x 8 samples, 32 / 8 heads, head_dim 128, block_size
            16, bf16: a 1000-token prompt in 62 full blocks shared by all 8
            samples plus a partial block of 8 tokens that sample 0 keeps and
            samples 1..7 receive as copies (copy_blocks pairs), then 0..512
            generated tokens per sample (uniform) written into private
            blocks.
  long16 /  batch 16, 64 / 8 heads, head_dim 128, bf16, lengths uniform in
  long32    [32768, 131072], block_size 16 / 32, pool of 1.1x need.

Values: q, the new token's K and V, and every pool slot are N(0, 1) drawn in
fp32 and rounded to the workload's element type (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: torch.dtype
    lengths: str               # "fixed" | "uniform" | "lognormal" | "cow"
    len_lo: int = 0
    len_hi: int = 0
    median: float = 0.0
    sigma: float = 0.0
    pool_factor: float = 1.25
    fixed: tuple = ()
    prompts: int = 0
    samples: int = 0
    prompt_len: int = 0
    gen_hi: int = 0
    pool_blocks: int = 0       # explicit pool size (tiny)


WORKLOADS = {
    "tiny": Workload("tiny", 4, 4, 4, 64, 16, torch.float32, "fixed", fixed=(1, 7, 16, 33), pool_blocks=64),
    "llama7b": Workload("llama7b", 64, 32, 32, 128, 16, torch.bfloat16, "uniform", len_lo=128, len_hi=2048),
    "gqa": Workload("gqa", 256, 32, 8, 128, 16, torch.bfloat16, "lognormal", len_lo=16, len_hi=4096,
                    median=1000.0, sigma=0.8),
    "cow": Workload("cow", 256, 32, 8, 128, 16, torch.bfloat16, "cow", prompts=32, samples=8, prompt_len=1000,
                    gen_hi=512, pool_factor=1.05),
    "long16": Workload("long16", 16, 64, 8, 128, 16, torch.bfloat16, "uniform", len_lo=32768, len_hi=131072,
                       pool_factor=1.1),
    "long32": Workload("long32", 16, 64, 8, 128, 32, torch.bfloat16, "uniform", len_lo=32768, len_hi=131072,
                       pool_factor=1.1),
}

SEEDS = {"tiny": 1000, "llama7b": 1001, "gqa": 1002, "cow": 1003, "long16": 1004, "long32": 1005}


@dataclass
class DecodeCase:
    """One decode step's inputs.  Metadata lives on the host (int32/int64
    CPU tensors); value tensors live on `device`."""
    workload: Workload
    scale: float
    lengths: torch.Tensor            # int32 [B], including the appended token
    block_tables: torch.Tensor       # int32 [B, MBS], -1 past each sequence's blocks
    num_blocks: int
    q: torch.Tensor                  # [B, Hq, D]
    k_new: torch.Tensor              # [T_new, Hkv, D]  (T_new = B for plain decode)
    v_new: torch.Tensor
    new_seq_ids: torch.Tensor        # int32 [T_new]
    new_positions: torch.Tensor      # int32 [T_new]
    k_pool: torch.Tensor             # [NB, Hkv, bs, D]
    v_pool: torch.Tensor
    cow_pairs: torch.Tensor = field(default_factory=lambda: torch.zeros((0, 2), dtype=torch.int64))
    # sequences [starts[g], starts[g + 1]) share their first prefix_len[g]
    # tokens in the same physical blocks (None: no sharing)
    prefix_groups: tuple | None = None

    @property
    def max_len(self) -> int:
        return int(self.lengths.max()) if self.lengths.numel() else 0

    def kv_bytes(self) -> int:
        """K and V bytes of the tokens attention reads (tokens < length)."""
        w = self.workload
        return int(self.lengths.sum()) * w.num_kv_heads * w.head_dim * self.k_pool.element_size() * 2


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_into(t: torch.Tensor, gen: torch.Generator, chunk: int = 1 << 26) -> torch.Tensor:
    """Fill t with N(0, 1) drawn in fp32 and rounded to t's dtype, in chunks."""
    flat = t.view(-1)
    for s in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - s)
        flat[s: s + n] = torch.randn(n, generator=gen, device=t.device, dtype=torch.float32).to(t.dtype)
    return t


def draw_lengths(w: Workload, gen: torch.Generator) -> list[int]:
    if w.lengths == "fixed":
        return [L + 1 for L in w.fixed]
    if w.lengths == "uniform":
        return torch.randint(w.len_lo, w.len_hi + 1, (w.batch,), generator=gen).tolist()
    if w.lengths == "lognormal":
        z = torch.randn(w.batch, generator=gen, dtype=torch.float64)
        vals = torch.exp(math.log(w.median) + w.sigma * z).round().clamp(w.len_lo, w.len_hi)
        return [int(x) for x in vals.tolist()]
    raise ValueError(w.lengths)


def _blocks_for(n_tokens: int, bs: int) -> int:
    return -(-n_tokens // bs)


def make_case(name: str, device="cpu", seed: int | None = None, batch: int | None = None,
              block_size: int | None = None, dtype: torch.dtype | None = None) -> DecodeCase:
    """Draw the inputs of workload `name` (optionally with a smaller batch, a
    different block size or element type for reduced-size tests)."""
    w = WORKLOADS[name]
    if batch is not None:
        w = replace(w, batch=batch, prompts=(batch // w.samples if w.lengths == "cow" else w.prompts))
    if block_size is not None:
        w = replace(w, block_size=block_size)
    if dtype is not None:
        w = replace(w, dtype=dtype)
    seed = SEEDS[name] if seed is None else seed
    host = _gen(seed, "cpu")
    place = _gen(seed + 1, "cpu")
    bs = w.block_size

    cow_pairs = torch.zeros((0, 2), dtype=torch.int64)
    groups = None
    if w.lengths == "cow":
        tables, lengths, new_sid, new_pos, cow_pairs, nb = _cow_layout(w, host, place)
        # the samples of a prompt are consecutive and share its full blocks
        groups = ([p * w.samples for p in range(w.prompts + 1)], [(w.prompt_len // bs) * bs] * w.prompts)
    else:
        lengths = draw_lengths(w, host)
        need = [_blocks_for(L, bs) for L in lengths]
        if w.lengths == "fixed":
            nb = w.pool_blocks
            ids = torch.randperm(nb, generator=place).tolist()
            # each sequence first takes the blocks of its tokens before the
            # append, then the appended tokens take further blocks if needed
            before = [_blocks_for(L - 1, bs) for L in lengths]
            tables, at = [], 0
            for n in before:
                tables.append(ids[at: at + n])
                at += n
            for b, n in enumerate(need):
                while len(tables[b]) < n:
                    tables[b].append(ids[at])
                    at += 1
        else:
            nb = int(math.ceil(w.pool_factor * sum(need)))
            ids = torch.randperm(nb, generator=place).tolist()
            tables, at = [], 0
            for n in need:
                tables.append(ids[at: at + n])
                at += n
        new_sid = list(range(w.batch))
        new_pos = [L - 1 for L in lengths]

    case = build_case(w, lengths, tables, nb, new_sid, new_pos, cow_pairs, seed + 2, device)
    case.prefix_groups = groups
    return case


def shared_prefix_groups(case: DecodeCase):
    """(group_starts, prefix_len) lists of a case whose consecutive sequences
    share their leading blocks, as its layout made them; None if none do."""
    return case.prefix_groups


def build_case(w: Workload, lengths, tables, num_blocks: int, new_sid, new_pos, cow_pairs=None, value_seed: int = 0,
               device="cpu", table_width: int | None = None) -> DecodeCase:
    """Pack block tables and draw every value tensor of a case."""
    mbs = max(1, max(len(t) for t in tables)) if table_width is None else table_width
    bt = torch.full((len(tables), mbs), -1, dtype=torch.int32)
    for b, t in enumerate(tables):
        if t:
            bt[b, : len(t)] = torch.tensor(t, dtype=torch.int32)
    vals = _gen(value_seed, device)
    D, Hkv, Hq, bs = w.head_dim, w.num_kv_heads, w.num_q_heads, w.block_size
    T_new = len(new_sid)
    q = randn_into(torch.empty((len(tables), Hq, D), dtype=w.dtype, device=device), vals)
    k_new = randn_into(torch.empty((T_new, Hkv, D), dtype=w.dtype, device=device), vals)
    v_new = randn_into(torch.empty((T_new, Hkv, D), dtype=w.dtype, device=device), vals)
    k_pool = randn_into(torch.empty((num_blocks, Hkv, bs, D), dtype=w.dtype, device=device), vals)
    v_pool = randn_into(torch.empty((num_blocks, Hkv, bs, D), dtype=w.dtype, device=device), vals)
    scale = float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))
    if cow_pairs is None:
        cow_pairs = torch.zeros((0, 2), dtype=torch.int64)
    return DecodeCase(w, scale, torch.tensor(list(lengths), dtype=torch.int32), bt, num_blocks, q, k_new, v_new,
                      torch.tensor(list(new_sid), dtype=torch.int32), torch.tensor(list(new_pos), dtype=torch.int32),
                      k_pool, v_pool, cow_pairs)


def custom_case(lengths, num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int, dtype: torch.dtype,
                seed: int = 0, device="cpu", extra_blocks: int = 3, table_width: int | None = None) -> DecodeCase:
    """A decode case with the given lengths (each including its appended
    token), every sequence's blocks scattered over a pool with a few spare
    blocks, one new token per non-empty sequence."""
    w = Workload("custom", len(lengths), num_q_heads, num_kv_heads, head_dim, block_size, dtype, "fixed")
    place = _gen(seed + 1, "cpu")
    need = [_blocks_for(L, block_size) for L in lengths]
    nb = sum(need) + extra_blocks
    ids = torch.randperm(nb, generator=place).tolist()
    tables, at = [], 0
    for n in need:
        tables.append(ids[at: at + n])
        at += n
    sid = [b for b, L in enumerate(lengths) if L > 0]
    pos = [lengths[b] - 1 for b in sid]
    return build_case(w, lengths, tables, nb, sid, pos, None, seed + 2, device, table_width)


def _cow_layout(w: Workload, host: torch.Generator, place: torch.Generator):
    """Block tables of `prompts` x `samples` sequences sharing a prompt.

    Per prompt: full prompt blocks shared by every sample, one partial block
    kept by sample 0 and copied for samples 1..samples-1, then private blocks
    for each sample's generated tokens."""
    bs = w.block_size
    full = w.prompt_len // bs
    partial = 1 if w.prompt_len % bs else 0
    gens = torch.randint(0, w.gen_hi + 1, (w.prompts * w.samples,), generator=host).tolist()
    lengths = [w.prompt_len + g for g in gens]
    need = w.prompts * (full + partial * w.samples)
    need += sum(_blocks_for(L, bs) - full - partial for L in lengths)
    nb = int(math.ceil(w.pool_factor * need))
    ids = iter(torch.randperm(nb, generator=place).tolist())
    tables, pairs, new_sid, new_pos = [], [], [], []
    for p in range(w.prompts):
        shared = [next(ids) for _ in range(full)]
        orig = next(ids) if partial else None
        for s in range(w.samples):
            b = p * w.samples + s
            t = list(shared)
            if partial:
                if s == 0:
                    t.append(orig)
                else:
                    dst = next(ids)
                    pairs.append((orig, dst))
                    t.append(dst)
            while len(t) < _blocks_for(lengths[b], bs):
                t.append(next(ids))
            tables.append(t)
            for pos in range(w.prompt_len, lengths[b]):
                new_sid.append(b)
                new_pos.append(pos)
    cow = torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2)
    return tables, lengths, new_sid, new_pos, cow, nb
