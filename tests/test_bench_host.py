"""bench.py's host-side helpers on CPU: the code hash that keys the committed
DRAM-traffic record, the distinct-slot byte count, and the traffic lookup."""
from __future__ import annotations

import importlib.util
import json
import os

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_host", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_code_hash_ignores_comments_and_blank_lines(bench, tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text("int f(int x) {\n    return x + 1;\n}\n")
    b.write_text("// a comment\nint f(int x) {  // trailing\n\n    return x + 1;   \n}\n")
    c.write_text("int f(int x) {\n    return x + 2;\n}\n")
    assert bench.code_sha256(str(a)) == bench.code_sha256(str(b))
    assert bench.code_sha256(str(a)) != bench.code_sha256(str(c))


def test_traffic_record_matches_the_current_decode_code(bench):
    """The committed record was taken on the current pass-1 code: the lookup
    returns its bytes for each recorded workload, and nothing otherwise."""
    rec = json.load(open(os.path.join(ROOT, "profiles", "decode_traffic.json")))
    for name, entry in rec.items():
        if name.startswith("_"):
            continue
        assert bench.dram_traffic(name) == entry["dram_bytes_per_launch"]
    assert bench.dram_traffic("tiny") is None


def test_traffic_record_matches_the_current_prefill_code(bench):
    """The same for the prefill kernel's record."""
    rec = json.load(open(os.path.join(ROOT, "profiles", "prefill_traffic.json")))
    entry = rec["prefill"]
    assert bench.dram_traffic("prefill", "prefill_traffic.json", "pa_prefill.cu") == entry["dram_bytes_per_launch"]
    assert entry["dram_bytes_per_launch"] == entry["read_bytes"] + entry["write_bytes"]


class _W:
    def __init__(self, bs, hkv, d):
        self.block_size, self.num_kv_heads, self.head_dim = bs, hkv, d


class _Case:
    def __init__(self, lengths, tables, bs, hkv=2, d=64):
        self.workload = _W(bs, hkv, d)
        self.lengths = torch.tensor(lengths, dtype=torch.int32)
        self.block_tables = torch.tensor(tables, dtype=torch.int32)
        self.k_pool = torch.zeros(1, dtype=torch.bfloat16)


def test_unique_bytes_count_shared_slots_once(bench):
    # two sequences share block 3 fully (16 tokens) and then diverge
    case = _Case([20, 18], [[3, 5], [3, 7]], bs=16)
    per_token = 2 * 64 * 2 * 2  # Hkv * D * elt * (K and V)
    assert bench.unique_kv_bytes(case) == (16 + 4 + 2) * per_token
    # no sharing: the logical bytes
    case = _Case([20, 18], [[3, 5], [4, 7]], bs=16)
    assert bench.unique_kv_bytes(case) == (20 + 18) * per_token
    # a partial block shared by both: only its filled slots count, once
    case = _Case([5, 9], [[2, -1], [2, -1]], bs=16)
    assert bench.unique_kv_bytes(case) == 9 * per_token


def test_prefill_useful_flops_counts_the_visible_pairs(bench):
    """The prefill metric's FLOP count against a brute-force count of the
    (query, key) pairs the causal mask leaves visible."""
    lengths, news = [1, 7, 64, 65, 300, 0], [1, 3, 64, 1, 130, 0]
    pairs = 0
    for L, n in zip(lengths, news):
        for i in range(n):
            pos = L - n + i
            pairs += sum(1 for t in range(L) if t <= pos)
    assert bench.prefill_useful_flops(lengths, news, 32, 128) == 4.0 * 128 * 32 * pairs
    # the benchmark's workload: batch 8, context 4096, the last 2048 tokens new
    assert bench.prefill_useful_flops([4096] * 8, [2048] * 8, 32, 128) == 4.0 * 128 * 32 * 8 * (
        2048 * 2048 + 2048 * 2049 // 2)
