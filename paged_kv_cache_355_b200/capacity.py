"""Capacity and waste of paged vs contiguous KV allocation, on libpa's native
block manager.

What the pages claim, and what this measures on synthetic request lengths:
  * contiguous max-length reservation wastes most of the KV memory
    ("PagedAttention and KV memory management", "Key takeaways"; "How does
    vLLM PagedAttention manage Virtual Memory Pages ...", "Short answer":
    ~60-80 % down to under 4 %);
  * paging wastes about one partly filled block per sequence (the first
    page's introduction);
  * so 2-4x more sequences fit ("The kernel side"; "Interview tips");
  * n = 8 parallel samples without sharing store the prompt 8 times
    ("Myths and failure modes").

Admission model (the pages give none; the plainest reading): requests arrive
in order and are admitted while their KV fits.  Contiguous: each admitted
request reserves max_model_len tokens.  Paged: each admitted request takes
blocks for its actual length from the block manager.

    python -m paged_kv_cache_355_b200.capacity
"""
from __future__ import annotations

import math
import time

import numpy as np

from .block_manager import BlockManager, OutOfBlocks


def contiguous(lengths, pool_tokens: int, max_model_len: int) -> dict:
    """Admit in order, each request reserving max_model_len tokens."""
    admitted = min(len(lengths), pool_tokens // max_model_len)
    used = int(sum(lengths[:admitted]))
    reserved = admitted * max_model_len
    return {"admitted": admitted, "used_tokens": used, "reserved_tokens": reserved,
            "waste": 1.0 - used / reserved if reserved else 0.0}


def paged(lengths, pool_tokens: int, block_size: int) -> dict:
    """Admit in order through the native block manager until a request no
    longer fits (that request's blocks are given back)."""
    bm = BlockManager(pool_tokens // block_size, block_size)
    admitted, used = 0, 0
    t0 = time.perf_counter()
    appends = 0
    for i, L in enumerate(lengths):
        need = -(-int(L) // block_size)
        if need > bm.num_free():
            break
        try:
            bm.append_tokens(np.full(int(L), i, np.int64))
        except OutOfBlocks:
            bm.free_sequence(i)
            break
        appends += int(L)
        admitted += 1
        used += int(L)
    secs = time.perf_counter() - t0
    reserved = (bm.num_blocks - bm.num_free()) * block_size
    return {"admitted": admitted, "used_tokens": used, "reserved_tokens": reserved,
            "waste": 1.0 - used / reserved if reserved else 0.0,
            "appends_per_s": appends / secs if secs > 0 else float("inf")}


def parallel_sampling_blocks(prompt_len: int, n: int, block_size: int, share: bool) -> int:
    """Blocks holding the prompt of n samples, with or without prefix sharing."""
    bm = BlockManager(n * (prompt_len // block_size + 2), block_size)
    bm.append_tokens(np.zeros(prompt_len, np.int64))
    for s in range(1, n):
        if share:
            bm.fork(0, s)
        else:
            bm.append_tokens(np.full(prompt_len, s, np.int64))
    return bm.num_blocks - bm.num_free()


def lognormal_lengths(n: int, median: float, sigma: float, lo: int, hi: int, seed: int = 7) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.clip(np.rint(np.exp(math.log(median) + sigma * rng.standard_normal(n))), lo, hi).astype(np.int64)


def report(pool_tokens: int = 1 << 20, block_size: int = 16, max_model_len: int = 4096, seed: int = 7) -> dict:
    """The pages' capacity figures on one synthetic length mix (lognormal,
    median 1000, sigma 0.8, clipped to [16, max_model_len])."""
    lengths = lognormal_lengths(20000, 1000.0, 0.8, 16, max_model_len, seed)
    c = contiguous(lengths, pool_tokens, max_model_len)
    p = paged(lengths, pool_tokens, block_size)
    one = contiguous([100], 4096, 4096)
    return {
        "pool_tokens": pool_tokens, "block_size": block_size, "max_model_len": max_model_len,
        "contiguous": c, "paged": p, "batch_gain": p["admitted"] / max(c["admitted"], 1),
        "single_request_100_of_4096_waste": one["waste"],
        "prompt_blocks_n8_shared": parallel_sampling_blocks(1000, 8, block_size, True),
        "prompt_blocks_n8_private": parallel_sampling_blocks(1000, 8, block_size, False),
    }


if __name__ == "__main__":
    import json

    print(json.dumps(report(), indent=1))
