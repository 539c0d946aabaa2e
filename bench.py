"""Benchmark of the paged decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one decode step of one attention layer over one batch: the new
token's slot and its K/V write, and paged decode attention over every
sequence, in one call (pa_paged_attention_decode_append: for bf16 one pass-1
launch that also writes the new token, plus the split-KV merge when a
sequence is split).  The workloads that append several tokens per sequence
run pa_slot_mapping and pa_reshape_and_cache, copy-on-write copies when the
workload has them (pa_copy_blocks), and pa_paged_attention_decode.  Inputs are seeded synthetic tensors shaped like the named workload,
resident in HBM before timing.

Timing: W untimed warm-up steps, then the step is captured into a CUDA graph
and K replays are timed, each bracketed by CUDA events on the launching
stream; then the decode call alone, captured into its own graph, is timed the
same way for the roofline.  Between replays (outside the events) 256 MiB are
written and another 256 MiB read, which leaves the 126 MB L2 holding none of
the step's data and no dirty lines.  The region is bracketed by a barrier and
torch.cuda.synchronize(); the reported time is the max over ranks.  The
end-to-end figure goes through the plain Python API instead.

value  = K/V bytes attention reads (tokens < length, K and V) / step time,
         summed over ranks (each rank runs its own batch: weak scaling, no
         data-path collective).
e2e    = the same metric through the public API with the step's inputs in
         pinned host memory: one H2D copy of q, new K/V, block tables and
         lengths packed together, the step (direct calls on views of the
         device copy), and D2H of the output, timed by the host clock from
         the first issue to a synchronize after the read-back (what a
         caller without graphs waits).  device_ms_per_step times the same
         calls by CUDA events with a device spin ahead of each step.
roofline = the decode call alone (pass 1 + merge; at least 100 timed replays,
         mean, median, p10 and p90 reported) against the measured HBM copy
         bandwidth, and against the read ceiling that pa_hbm_read_probe (a
         plain bulk read stream of 2 GiB) reaches in the same run.  Its
         algorithmic bytes are the distinct K/V bytes the call must read:
         every sequence's K/V, except that on the shared-prefix workload a
         prompt block shared by a group counts once.
other_workloads = (default run only) the decode calls of the GQA,
         long-context and shared-prefix workloads, timed the same way, with
         their paging overheads; the shared-prefix workload also by the
         distinct (unique) K/V bytes it reads.

--impl reference times the CPU oracle (fp64, OpenMP) on the host cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Paged decode attn: achieved HBM GB/s vs peak; decode tokens/s per batch"
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 256 << 20
# ~4 ms at 1.965 GHz.  With a 1 ms spin the step's first H2D copy measured
# 0.126 ms instead of 0.038 ms on the B200 (the same copy with no spin, or
# after a 4 ms one, takes 0.038-0.040 ms), which inflated the e2e time.
SPIN_CYCLES = 8_000_000

DESCRIPTIONS = {
    "tiny": "tiny: batch 4, lengths 1,7,16,33 (+1 appended), 4/4 heads, head_dim 64, block_size 16, fp32",
    "llama7b": "Llama-7B-shaped decode: batch 64, 32 q = 32 kv heads, head_dim 128, block_size 16, bf16, "
               "lengths U[128, 2048], blocks drawn without replacement from a 1.25x pool",
    "gqa": "GQA decode: batch 256, 32 q / 8 kv heads, head_dim 128, block_size 16, bf16, lengths lognormal "
           "(median 1000, sigma 0.8) clipped to [16, 4096], blocks scattered",
    "cow": "shared-prefix parallel sampling: 32 prompts x 8 samples, 32/8 heads, head_dim 128, bf16, block_size 16, "
           "1000-token prompt shared (refcount 8), partial block copied by copy_blocks, 0-512 generated tokens",
    "long16": "long-context split-KV decode: batch 16, 64 q / 8 kv heads, head_dim 128, bf16, block_size 16, "
              "lengths U[32768, 131072], pool 1.1x",
    "long32": "long-context split-KV decode: batch 16, 64 q / 8 kv heads, head_dim 128, bf16, block_size 32, "
              "lengths U[32768, 131072], pool 1.1x",
}


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="llama7b", choices=sorted(DESCRIPTIONS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--partition", type=int, default=0, help="tokens per KV split (0 = automatic)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiler captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the GQA, long-context and shared-prefix decode calls that the default "
                         "Llama-7B-shaped run also times")
    ap.add_argument("--op", default="decode", choices=["decode", "prefill", "blocks"],
                    help="decode: the decode step (default); prefill: causal multi-query paged attention "
                         "on a chunked-prefill workload, in TFLOP/s; blocks: copy_blocks inside the device "
                         "pool and swap_blocks to and from a pinned host pool, in GB/s")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def code_sha256(path: str) -> str:
    """sha256 of a source file's code: // comments and blank lines removed,
    so that a comment edit does not void a measurement of the same kernel."""
    lines = []
    for line in open(path, encoding="utf-8"):
        code = line.split("//", 1)[0].rstrip()
        if code:
            lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def dram_traffic(workload: str, record: str = "decode_traffic.json", source: str = "pa_decode.cu"):
    """Per-launch DRAM bytes of a kernel from a committed ncu summary
    (profiles/<record>), if it was taken on the current code of its source
    file (csrc/<source>); else None."""
    path = os.path.join(ROOT, "profiles", record)
    src = os.path.join(ROOT, "paged_kv_cache_355_b200", "csrc", source)
    try:
        rec = json.load(open(path))
        sha = code_sha256(src)
        entry = rec.get(workload)
        if entry and entry.get("kernel_code_sha256") == sha:
            return int(entry["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples (SM clock, throttle reasons) while the region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for _, _, flags in rows:
            for n, f in zip(names, flags[1:]):
                if f.lower() == "active":
                    reasons.add(n)
        loaded = [r[0] for r in rows if r[0] > 0.5 * r[1]] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


def unique_kv_bytes(case) -> int:
    """K and V bytes of the distinct pool slots the step's attention reads:
    less than the logical K/V bytes when sequences share blocks."""
    w = case.workload
    bs = w.block_size
    slots = []
    for b, L in enumerate(case.lengths.tolist()):
        if L > 0:
            t = torch.arange(L, dtype=torch.int64)
            slots.append(case.block_tables[b, t // bs].to(torch.int64) * bs + t % bs)
    n = int(torch.unique(torch.cat(slots)).numel()) if slots else 0
    return n * w.num_kv_heads * w.head_dim * case.k_pool.element_size() * 2


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank time over all ranks (the job is as slow as its slowest GPU)."""
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------
def oracle_sample(case, max_seqs: int):
    """Host arrays of the first `max_seqs` sequences of a case (a bounded
    sample of the same workload) for the oracle."""
    import numpy as np

    def bits(t):
        t = t.detach().cpu().contiguous()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    n = min(max_seqs, case.workload.batch)
    sel = (case.new_seq_ids < n).numpy()
    return dict(q=bits(case.q[:n]), k_new=bits(case.k_new)[sel], v_new=bits(case.v_new)[sel],
                sid=case.new_seq_ids.numpy()[sel], pos=case.new_positions.numpy()[sel],
                bt=case.block_tables[:n].numpy(), lens=case.lengths[:n].numpy(),
                k_pool=bits(case.k_pool).copy(), v_pool=bits(case.v_pool).copy(),
                pairs=case.cow_pairs.numpy(), bytes=int(case.lengths[:n].sum()) * case.workload.num_kv_heads
                * case.workload.head_dim * case.k_pool.element_size() * 2, seqs=n)


def oracle_step(s, scale, bs):
    import oracle

    if len(s["pairs"]):
        oracle.copy_blocks(s["k_pool"], s["v_pool"], s["pairs"])
    slots = oracle.slot_mapping(s["bt"], s["sid"], s["pos"], bs)
    oracle.reshape_and_cache(s["k_new"], s["v_new"], s["k_pool"], s["v_pool"], slots)
    return oracle.paged_decode(s["q"], s["k_pool"], s["v_pool"], s["bt"], s["lens"], scale, bs)


def time_oracle(case, min_seconds=10.0, max_reps=1000, max_seqs=None):
    """The oracle on the host cores: whole decode steps of the workload,
    repeated until about min_seconds of CPU work have run."""
    import oracle

    n = max_seqs or case.workload.batch
    s = oracle_sample(case, n)
    reps, t_total = 0, 0.0
    while reps < max_reps and (reps == 0 or t_total < min_seconds):
        t0 = time.perf_counter()
        oracle_step(s, case.scale, case.workload.block_size)
        t_total += time.perf_counter() - t0
        reps += 1
    sec = t_total / reps
    return {"value": s["bytes"] / sec / 1e9, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{s['seqs']} of {case.workload.batch} sequences of the same workload, one full decode step "
                      f"(slot mapping, cache write, attention) per repetition, {reps} repetition(s), "
                      f"{sec:.3f} s each, {t_total:.1f} s in all", "seconds_per_step": sec}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from paged_kv_cache_355_b200.workloads import make_case

    import oracle

    if args.op == "prefill":
        run_reference_prefill(args, world)
        return
    case = make_case(args.workload, device="cpu")
    w = case.workload
    # each step: the oracle over a bounded sample of the workload's sequences
    seqs = {"tiny": 4, "llama7b": 8, "gqa": 16, "cow": 16, "long16": 1, "long32": 1}[args.workload]
    s = oracle_sample(case, seqs)
    for _ in range(args.warmup):
        oracle_step(s, case.scale, w.block_size)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(s, case.scale, w.block_size)
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = s["bytes"] / sec / 1e9
    sample = (f"{s['seqs']} of {w.batch} sequences of the workload per step (slot mapping, cache write, attention), "
              f"fp64 oracle")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": DESCRIPTIONS[args.workload], "sample_sequences": s["seqs"]},
            "tokens_per_s": s["seqs"] / sec,
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_prefill(args, world):
    """Reference arm of --op prefill: the oracle's causal multi-query attention
    on the host cores; each step is the first 64 queries of the workload's
    first sequence (all heads)."""
    import numpy as np

    import oracle
    from paged_kv_cache_355_b200.workloads import custom_case

    B, Hq, Hkv, D, bs, L, n = PREFILL_SHAPE
    case = custom_case([L] * B, Hq, Hkv, D, bs, torch.bfloat16, seed=2001, device="cpu")
    g = torch.Generator().manual_seed(2002)
    q = torch.randn(n, Hq, D, generator=g).to(torch.bfloat16)
    u16 = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    m = 64  # the sample: the first m of the n new queries, so context L - n + m
    kp, vp, qm = u16(case.k_pool), u16(case.v_pool), u16(q[:m])
    bt, lens = case.block_tables[:1].numpy(), np.array([L - n + m], dtype=np.int32)
    qs = np.array([0, m], dtype=np.int32)
    flops = 4.0 * D * Hq * (m * (L - n) + m * (m + 1) // 2)
    for _ in range(args.warmup):
        oracle.paged_prefill(qm, kp, vp, bt, lens, qs, case.scale, bs)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.paged_prefill(qm, kp, vp, bt, lens, qs, case.scale, bs)
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = flops / sec / 1e12
    sample = f"the first {m} of {n} new queries of 1 of {B} sequences, all {Hq} heads, fp64 oracle"
    print(json.dumps({
        "impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "dtype": "f64", "data": "synthetic", "config": {"workload": PREFILL_WORKLOAD},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
        flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
ROOFLINE_MIN_ITERS = 100  # timed replays of the decode call alone (at least)
PROBE_BYTES = 2 << 30     # read-ceiling probe buffer: 2 GiB, 16x the L2
OTHER_WORKLOADS = ("gqa", "long16", "cow")


def time_stats(ms):
    """mean, median, p10 and p90 (nearest rank) of a list of times in ms."""
    s = sorted(ms)
    at = lambda f: s[min(len(s) - 1, max(0, int(round(f * (len(s) - 1)))))]
    return {"mean": sum(s) / len(s), "median": statistics.median(s), "p10": at(0.1), "p90": at(0.9), "n": len(s)}


def timed_replays(run, n, flush_l2, stream, warmup=0):
    """CUDA-event times (ms) of n calls of run(), each preceded by an L2
    flush outside the events."""
    evs = []
    for i in range(warmup + n):
        flush_l2()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        if i >= warmup:
            evs.append((e0, e1))
    torch.cuda.synchronize()
    return [a.elapsed_time(b_) for a, b_ in evs]


def capture(fn):
    """fn captured into a CUDA graph (returns the graph and its replay), or
    (None, fn) when capture is unavailable."""
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        return g, g.replay
    except Exception as exc:
        print(f"bench: CUDA graph capture failed ({exc}); timing direct calls", file=sys.stderr)
        return None, fn


def make_decode_call(pa, case, bt, lens, out, part, ws, groups=None):
    """The decode-attention call the step makes for a case: the shared-prefix
    form when the case's sequences share prompt blocks, else the plain one."""
    if groups is not None:
        gs, gl, max_prefix, max_group = groups
        return lambda: pa.pa_paged_attention_decode_shared_prefix(
            case.q, case.k_pool, case.v_pool, bt, lens, case.max_len, case.scale, out, gs, gl, max_prefix,
            max_group, partition_size=part, workspace=ws)
    return lambda: pa.pa_paged_attention_decode(case.q, case.k_pool, case.v_pool, bt, lens, case.max_len, case.scale,
                                                out, partition_size=part, workspace=ws)


def prefix_groups(pa, case, dev):
    """(group_starts, group_prefix_len, max_prefix_len, max_group_size) of a
    case whose consecutive sequences share leading blocks, as device tensors;
    None when no two sequences share a block."""
    from paged_kv_cache_355_b200.workloads import shared_prefix_groups

    groups = shared_prefix_groups(case)
    if groups is None:
        return None
    starts, plen = groups
    return (torch.tensor(starts, dtype=torch.int32, device=dev), torch.tensor(plen, dtype=torch.int32, device=dev),
            max(plen), max(b - a for a, b in zip(starts[:-1], starts[1:])))


def workspace_for(pa, case, part, groups):
    w = case.workload
    B, Hq, Hkv, D, bs = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size
    if groups is not None:
        return pa.pa_paged_attention_shared_prefix_workspace_size(B, Hq, Hkv, D, case.max_len, bs,
                                                                  groups[1].numel(), groups[3], groups[2], part)
    return pa.pa_paged_attention_workspace_size(B, Hq, Hkv, D, case.max_len, bs, part)


def measure_other_workload(pa, name, dev, flush_l2, stream, iters, peak):
    """The decode-attention call of another named workload, timed like the
    headline's roofline loop (graph replays, L2 flushed between them), with
    its paging overhead against the contiguous-cache kernel."""
    from paged_kv_cache_355_b200.workloads import make_case

    case = make_case(name, device=dev)
    w = case.workload
    B, Hq, Hkv, D, bs = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size
    bt, lens = case.block_tables.to(dev), case.lengths.to(dev)
    part = pa.pa_paged_attention_partition_size(B, Hq, Hkv, D, case.max_len, bs)
    groups = prefix_groups(pa, case, dev)
    ws = torch.empty(max(workspace_for(pa, case, part, groups), 16), dtype=torch.uint8, device=dev)
    out = torch.empty(B, Hq, D, dtype=torch.float32, device=dev)
    call = make_decode_call(pa, case, bt, lens, out, part, ws, groups)
    call()
    g, run = capture(call)
    ms = timed_replays(run, iters, flush_l2, stream, warmup=3)
    del g
    kv = case.kv_bytes()
    st = time_stats(ms)
    res = {"workload": DESCRIPTIONS[name], "decode_call": "pa_paged_attention_decode_shared_prefix"
           if groups is not None else "pa_paged_attention_decode", "partition_tokens": part,
           "kv_bytes": kv, "decode_ms": st, "gbs": kv / (st["median"] * 1e-3) / 1e9}
    res["frac"] = res["gbs"] / peak
    ub = unique_kv_bytes(case)
    if ub != kv:
        res["unique_kv"] = {"bytes": ub, "gbs": ub / (st["median"] * 1e-3) / 1e9,
                            "frac": ub / (st["median"] * 1e-3) / 1e9 / peak}
    # the same kernel on a contiguous cache with the same lengths
    L_pad = -(-case.max_len // 32) * 32
    k_c = torch.empty(B, Hkv, L_pad, D, dtype=w.dtype, device=dev).normal_()
    v_c = torch.empty_like(k_c).normal_()
    out_c = torch.empty_like(out)
    ws_c = torch.empty(max(pa.pa_paged_attention_workspace_size(B, Hq, Hkv, D, case.max_len, bs, part), 16),
                       dtype=torch.uint8, device=dev)
    contig = lambda: pa.pa_paged_attention_decode_contiguous(case.q, k_c, v_c, lens, case.max_len, case.scale, out_c,
                                                             block_size=bs, partition_size=part, workspace=ws_c)
    contig()
    g, run = capture(contig)
    ms_c = timed_replays(run, iters, flush_l2, stream, warmup=3)
    del g
    res["paging_overhead"] = st["median"] / statistics.median(ms_c) - 1.0
    assert pa.pa_read_error_flag() == 0, f"device error during the {name} measurement"
    del case, k_c, v_c, out_c, ws, ws_c
    torch.cuda.empty_cache()
    return res
def run_ours(args):
    world, rank, local = dist_setup(args.gpus)
    import paged_kv_cache_355_b200 as pa
    from paged_kv_cache_355_b200.workloads import SEEDS, WORKLOADS, make_case

    dev = torch.device("cuda", local)
    case = make_case(args.workload, device=dev, seed=SEEDS[args.workload] + 101 * rank, batch=args.batch)
    w = case.workload
    B, Hq, Hkv, D, bs = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size
    stream = torch.cuda.current_stream()
    bt = case.block_tables.to(dev)
    lens = case.lengths.to(dev)
    max_len = case.max_len
    kv_bytes = case.kv_bytes()
    unique_bytes = unique_kv_bytes(case)
    out = torch.empty(B, Hq, D, dtype=torch.float32, device=dev)
    slots = torch.empty(case.new_seq_ids.numel(), dtype=torch.int64, device=dev)
    sid, pos = case.new_seq_ids.to(dev), case.new_positions.to(dev)
    pairs = case.cow_pairs.to(dev)
    part = args.partition or pa.pa_paged_attention_partition_size(B, Hq, Hkv, D, max_len, bs)
    groups = prefix_groups(pa, case, dev)
    ws_bytes = workspace_for(pa, case, part, groups)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    plain_decode = pairs.numel() == 0 and case.new_seq_ids.numel() == B
    peak, peak_kind = measured_hbm_peak()

    def cache_part():
        if pairs.numel():
            pa.pa_copy_blocks(case.k_pool, case.v_pool, pairs)
        if plain_decode:
            # slot mapping and cache write of the step's one token per sequence, one launch
            pa.pa_reshape_and_cache_decode(case.k_new, case.v_new, case.k_pool, case.v_pool, bt, lens, slots)
        else:
            pa.pa_slot_mapping(bt, sid, pos, bs, slots)
            pa.pa_reshape_and_cache(case.k_new, case.v_new, case.k_pool, case.v_pool, slots)

    decode_part = make_decode_call(pa, case, bt, lens, out, part, ws, groups)

    def step():
        if plain_decode and w.dtype == torch.bfloat16:
            # the new token's slot and cache write folded into the attention launch
            pa.pa_paged_attention_decode_append(case.q, case.k_new, case.v_new, case.k_pool, case.v_pool, bt, lens,
                                                max_len, case.scale, out, partition_size=part, workspace=ws,
                                                slot_mapping=slots)
        else:
            cache_part()
            decode_part()

    def flush_l2():
        # write a buffer twice the L2, then read another one, so that the
        # step starts with the L2 holding none of its inputs and no dirty
        # lines whose write-back it would pay for
        flush.zero_()
        clean.sum()

    max_splits = -(-max(max_len, 1) // part)
    cache_launches = (1 if pairs.numel() else 0) + (1 if plain_decode else 2)
    # shared prefixes: the prefix pass, pass 1 (which finishes rows whose own
    # tokens are one split) and the merge pass only when a suffix can split
    decode_launches = (1 if groups is not None else 0) + 1 + (1 if max_splits > 1 else 0)
    step_launches = decode_launches + (0 if plain_decode and w.dtype == torch.bfloat16 else cache_launches)

    # ---- device-resident timed region
    # The step is captured once into a CUDA graph and replayed, as a serving
    # engine runs its decode step: Python's launch overhead stays out of the
    # device timeline and the kernels' programmatic launches overlap each
    # kernel's start with the previous one's drain.  The decode call alone is
    # captured into a second graph and timed the same way (at least 100
    # replays), for the roofline; then the read-ceiling probe.
    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    g_step, run_step = capture(step)
    g_decode, run_decode = capture(decode_part)
    graphs = g_step is not None and g_decode is not None
    for _ in range(2):
        run_step()
        run_decode()
    n_dec = max(args.steps, ROOFLINE_MIN_ITERS)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    ev_dec = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_dec)]
    probe_buf = torch.zeros(PROBE_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(3):
        pa.pa_hbm_read_probe(probe_buf)
    torch.cuda.synchronize()
    barrier(world)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        torch.cuda.synchronize()
        barrier(world)
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush_l2()
            ev[i][0].record(stream)
            run_step()
            ev[i][1].record(stream)
        for i in range(n_dec):
            flush_l2()
            ev_dec[i][0].record(stream)
            run_decode()
            ev_dec[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        t_wall = time.perf_counter() - t_wall
        probe_ms = timed_replays(lambda: pa.pa_hbm_read_probe(probe_buf), 20, flush_l2, stream)
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    dec_ms = [e[0].elapsed_time(e[1]) for e in ev_dec]
    ms_step = max_over_ranks(sum(step_ms) / len(step_ms), world)
    ms_dec = max_over_ranks(sum(dec_ms) / len(dec_ms), world)
    assert pa.pa_read_error_flag() == 0, "device error during the timed steps"
    del probe_buf
    read_ceiling = PROBE_BYTES / (statistics.median(probe_ms) * 1e-3) / 1e9

    # ---- the step's cache kernels alone (slot mapping, cache write, copy-on-write
    # copies), captured and timed the same way; their algorithmic bytes: each new
    # token's K and V rows read and written, each copied block's K and V read and
    # written, and the slots
    elt = case.k_pool.element_size()
    n_new = case.new_seq_ids.numel()
    cache_bytes = (n_new * Hkv * D * elt * 2 * 2 + pairs.shape[0] * Hkv * bs * D * elt * 2 * 2
                   + n_new * 8 * (1 if plain_decode else 2))
    g_cache, run_cache_only = capture(cache_part)
    cache_ms = timed_replays(run_cache_only, min(args.steps, 200), flush_l2, stream, warmup=args.warmup)
    ms_cache = max_over_ranks(sum(cache_ms) / len(cache_ms), world)
    del g_cache

    # ---- contiguous-cache variant of the same kernel on the same lengths (paging overhead),
    # timed the same way (graph replay)
    L_pad = -(-max_len // 32) * 32
    k_c = torch.empty(B, Hkv, L_pad, D, dtype=w.dtype, device=dev).normal_()
    v_c = torch.empty_like(k_c).normal_()
    out_c = torch.empty_like(out)
    ws_c = torch.empty(max(pa.pa_paged_attention_workspace_size(B, Hq, Hkv, D, max_len, bs, part), 16),
                       dtype=torch.uint8, device=dev)
    contig = lambda: pa.pa_paged_attention_decode_contiguous(case.q, k_c, v_c, lens, max_len, case.scale, out_c,
                                                             block_size=bs, partition_size=part, workspace=ws_c)
    contig()
    torch.cuda.synchronize()
    g_contig, run_contig = capture(contig)
    contig_ms = timed_replays(run_contig, min(n_dec, 200), flush_l2, stream, warmup=args.warmup)
    ms_contig = max_over_ranks(sum(contig_ms) / len(contig_ms), world)
    paged_med = statistics.median(dec_ms)
    contig_med = statistics.median(contig_ms)
    del k_c, v_c, run_contig, g_contig

    # ---- end to end through the public API with host buffers
    # The step's inputs (q, new K/V, block tables, lengths) sit in one pinned
    # host buffer and cross to the device in one copy; the API gets tensor
    # views of the device copy.
    srcs = [case.q, case.k_new, case.v_new, case.block_tables, case.lengths]
    if not plain_decode:  # the new tokens' sequences and positions, and the copy-on-write pairs
        srcs += [case.new_seq_ids, case.new_positions, case.cow_pairs]
    offs, total = [], 0
    for t in srcs:
        offs.append(total)
        total += -(-t.numel() * t.element_size() // 256) * 256
    h_pack = torch.empty(total, dtype=torch.uint8).pin_memory()
    d_pack = torch.empty(total, dtype=torch.uint8, device=dev)

    def view(buf, i):
        t = srcs[i]
        n = t.numel() * t.element_size()
        return buf[offs[i]: offs[i] + n].view(t.dtype).view(t.shape)

    for i, t in enumerate(srcs):
        view(h_pack, i).copy_(t.detach().cpu())
    d_q, d_kn, d_vn, d_bt, d_lens = (view(d_pack, i) for i in range(5))
    d_sid, d_pos, d_pairs = (view(d_pack, i) for i in range(5, 8)) if not plain_decode else (None, None, None)
    h_out = torch.empty(B, Hq, D, dtype=torch.float32).pin_memory()
    h2d = total
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step():
        d_pack.copy_(h_pack, non_blocking=True)
        if plain_decode:
            pa.decode_step(d_q, d_kn, d_vn, case.k_pool, case.v_pool, d_bt, d_lens, max_len, case.scale, out, slots,
                           workspace=ws, partition_size=part)
        else:
            if d_pairs.numel():
                pa.pa_copy_blocks(case.k_pool, case.v_pool, d_pairs)
            pa.pa_slot_mapping(d_bt, d_sid, d_pos, bs, slots)
            pa.pa_reshape_and_cache(d_kn, d_vn, case.k_pool, case.v_pool, slots)
            if groups is not None:
                pa.pa_paged_attention_decode_shared_prefix(d_q, case.k_pool, case.v_pool, d_bt, d_lens, max_len,
                                                           case.scale, out, groups[0], groups[1], groups[2],
                                                           groups[3], partition_size=part, workspace=ws)
            else:
                pa.pa_paged_attention_decode(d_q, case.k_pool, case.v_pool, d_bt, d_lens, max_len, case.scale, out,
                                             partition_size=part, workspace=ws)
        h_out.copy_(out, non_blocking=True)

    e2e_ev = []
    for i in range(args.warmup + args.steps):
        flush_l2()
        # a 4 ms spin on the device before the start event: the host enqueues
        # the whole step (copies, API calls, read-back) while it runs, so the
        # events time the step's device work, not Python's issue rate
        torch.cuda._sleep(SPIN_CYCLES)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_step()
        e1.record(stream)
        if i >= args.warmup:
            e2e_ev.append((e0, e1))
    torch.cuda.synchronize()
    e2e_ms = [a.elapsed_time(b_) for a, b_ in e2e_ev]
    ms_e2e = max_over_ranks(sum(e2e_ms) / len(e2e_ms), world)
    # the same step as a caller without graphs or a device spin sees it: host
    # wall time from the first copy's issue to the read-back's completion
    host_ms = []
    for i in range(args.warmup + args.steps):
        flush_l2()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        e2e_step()
        torch.cuda.synchronize()
        if i >= args.warmup:
            host_ms.append((time.perf_counter() - t0) * 1e3)
    ms_host = max_over_ranks(sum(host_ms) / len(host_ms), world)
    assert pa.pa_read_error_flag() == 0, "device error during the end-to-end steps"

    # ---- the other decode workloads, each timed like the roofline loop above
    # (one GPU, default headline run only)
    others = None
    if world == 1 and not args.no_other_workloads and args.batch is None and args.workload == "llama7b":
        torch.cuda.empty_cache()
        others = {}
        with ClockSampler(torch.cuda.current_device()) as oclocks:
            for name in OTHER_WORKLOADS:
                others[name] = measure_other_workload(pa, name, dev, flush_l2, stream, ROOFLINE_MIN_ITERS, peak)
        others["clocks"] = oclocks.summary()

    # ---- CPU oracle on this machine's host cores (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle(case)

    if rank != 0:
        return
    # the decode call's algorithmic bytes: the distinct K/V slots it reads
    achieved = unique_bytes / (ms_dec * 1e-3) / 1e9
    value = world * kv_bytes / (ms_step * 1e-3) / 1e9
    # the committed ncu record covers the workloads at their own batch only
    traffic = dram_traffic(args.workload) if args.batch in (None, WORKLOADS[args.workload].batch) else None
    clk = clocks.summary()
    st_step, st_dec = time_stats(step_ms), time_stats(dec_ms)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": {"workload": DESCRIPTIONS[args.workload] + (f" (batch overridden to {B})" if args.batch else ""),
                   "batch_per_gpu": B, "partition_tokens": part,
                   "max_splits": max_splits, "kv_bytes_per_step": kv_bytes,
                   "l2": "flushed between steps outside the timed events (256 MiB written, then another "
                         "256 MiB read, so no dirty line is written back inside the step); K/V read per "
                         "step also exceeds the 126 MB L2",
                   "parallelism": f"{world} independent replicas (sequences sharded, no collective)"},
        "tokens_per_s": world * B / (ms_step * 1e-3),
        "step_ms": st_step,
        "decode_attention_ms": st_dec,
        "decode_gbs_median": kv_bytes / (st_dec["median"] * 1e-3) / 1e9,
        "unique_kv": ({"bytes_per_step": unique_bytes,
                       "step_gbs": world * unique_bytes / (ms_step * 1e-3) / 1e9,
                       "decode_gbs": unique_bytes / (ms_dec * 1e-3) / 1e9,
                       "note": "distinct pool slots read; shared prompt blocks counted once"}
                      if unique_bytes != kv_bytes else None),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "algorithmic_bytes": unique_bytes,
                     "kernel": ("pa_paged_attention_decode_shared_prefix (set-up kernel, pass 1 over each sample's "
                                "own tokens, then the tensor-core prefix pass over each group's shared blocks)"
                                if groups is not None else "pa_paged_attention_decode (pass 1 + split merge)"),
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)",
                     "read_ceiling_gbs": read_ceiling, "frac_of_read_ceiling": achieved / read_ceiling,
                     "read_ceiling_source": f"pa_hbm_read_probe: a {PROBE_BYTES >> 30} GiB buffer streamed through "
                                            "shared memory by bulk TMA copies, median of 20 launches, this run",
                     "timed_iterations": n_dec},
        "cache_part": {"kernels": (["pa_copy_blocks"] if pairs.numel() else [])
                       + (["pa_reshape_and_cache_decode"] if plain_decode
                          else ["pa_slot_mapping", "pa_reshape_and_cache"]),
                       "ms": ms_cache, "bytes": cache_bytes, "gbs": cache_bytes / (ms_cache * 1e-3) / 1e9,
                       "frac": cache_bytes / (ms_cache * 1e-3) / 1e9 / peak,
                       "note": "timed alone as one graph; small writes are launch-latency bound"
                               + ("; the bf16 decode step itself does this write inside its attention launch"
                                  if plain_decode and w.dtype == torch.bfloat16 else "")},
        "paging_overhead": {"paged_ms_median": paged_med, "contiguous_ms_median": contig_med,
                            "overhead": paged_med / contig_med - 1.0, "contiguous_ms_mean_max_ranks": ms_contig},
        "e2e": {"value": world * kv_bytes / (ms_host * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_host, "ms_stats": time_stats(host_ms),
                "device_ms_per_step": ms_e2e, "device_ms_stats": time_stats(e2e_ms),
                "device_gbs": world * kv_bytes / (ms_e2e * 1e-3) / 1e9,
                "timing": "host clock from the first issue (the H2D copies of the step's inputs from pinned "
                          "memory) to a synchronize after the D2H read-back of the result, direct API calls, no "
                          "graph, max over ranks: what a caller without graphs waits. device_*: the same calls "
                          "timed by CUDA events with a device spin ahead of each step (host issue latency "
                          "hidden); on some boxes the GPU idling through the spin slows the step after it, so "
                          "that figure can exceed the host's"},
        "other_workloads": others,
        "gpu_launches": step_launches * args.steps,
        "gpu_launches_decode_roofline_loop": decode_launches * n_dec,
        "timing": ("K replays of the step's CUDA graph (value), then max(K, 100) replays of the decode call's "
                   "graph (roofline), each bracketed by events" if graphs else "direct calls"),
        "clocks": clk,
        "wall_s_timed_region": t_wall,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


PREFILL_SHAPE = (8, 32, 8, 128, 16, 4096, 2048)  # batch, Hq, Hkv, head_dim, block_size, context, new tokens
PREFILL_METRIC = "Paged prefill attn (causal, multi-query): achieved TFLOP/s vs bf16 peak"
PREFILL_WORKLOAD = ("chunked prefill: batch 8, 32 q / 8 kv heads, head_dim 128, block_size 16, bf16, "
                    "context 4096 of which the last 2048 tokens are the new chunk, blocks scattered")


def prefill_useful_flops(lengths, news, num_q_heads: int, head_dim: int) -> float:
    """Useful FLOPs of causal multi-query attention: the last n of a
    sequence's L tokens are queries, query i (position L - n + i) sees
    L - n + i + 1 keys, and each visible (query, key) pair costs 2 * D for
    q.k and 2 * D for p.v in every query head."""
    pairs = sum(n * (L - n) + n * (n + 1) // 2 for L, n in zip(lengths, news))
    return 4.0 * head_dim * num_q_heads * pairs


def run_prefill(args):
    """Causal multi-query paged attention on one GPU: useful FLOPs (4 * D per
    (query, visible key, query head)) / CUDA-event time."""
    import paged_kv_cache_355_b200 as pa
    from paged_kv_cache_355_b200.workloads import custom_case

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, Hq, Hkv, D, bs, L, n = PREFILL_SHAPE
    case = custom_case([L] * B, Hq, Hkv, D, bs, torch.bfloat16, seed=2001, device=dev)
    qs = torch.arange(0, (B + 1) * n, n, dtype=torch.int32, device=dev)
    g = torch.Generator(device=dev).manual_seed(2002)
    q = torch.randn(B * n, Hq, D, generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty(B * n, Hq, D, dtype=torch.bfloat16, device=dev)
    bt, lens = case.block_tables.to(dev), case.lengths.to(dev)
    flops = prefill_useful_flops([L] * B, [n] * B, Hq, D)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    run = lambda: pa.pa_paged_attention_prefill(q, case.k_pool, case.v_pool, bt, lens, qs, n, case.scale, out)
    for _ in range(args.warmup):
        run()
    evs = []
    torch.cuda.synchronize()
    with ClockSampler(0) as clocks:
        for _ in range(args.steps):
            flush.zero_()  # L2 flush outside the events: write, then read another buffer
            clean.sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            run()
            e1.record()
            evs.append((e0, e1))
        torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b_) for a, b_ in evs) / len(evs)
    assert pa.pa_read_error_flag() == 0
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    peak = float(peaks.get("bf16_tflops", 1590.0))
    tflops = flops / (ms * 1e-3) / 1e12
    cpu = None if args.no_cpu_baseline else time_oracle_prefill(case, q, n, L, bs)
    print(json.dumps({
        "metric": PREFILL_METRIC, "value": tflops,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic", "config": {"workload": PREFILL_WORKLOAD},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                     "traffic": dram_traffic("prefill", "prefill_traffic.json", "pa_prefill.cu"),
                     "kernel": "prefill_tc_kernel (tcgen05)",
                     "peak_source": "measured (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)" if peaks
                     else "fallback"},
        "note": "useful FLOPs only; the kernel multiplies P by V twice (bf16 high part and residual), "
                "so the tensor pipe executes 1.5x these FLOPs",
        "clocks": clocks.summary(), "cpu_baseline": cpu}), flush=True)


def time_oracle_prefill(case, q, n, L, bs, min_seconds=10.0, max_reps=100):
    """The oracle's causal multi-query attention for the first sequence of the
    prefill workload (all its n queries and heads), on the host cores,
    repeated until about min_seconds of CPU work have run."""
    import numpy as np

    import oracle

    u16 = lambda t: t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    kp, vp, q0 = u16(case.k_pool), u16(case.v_pool), u16(q[:n])
    bt, lens = case.block_tables[:1].numpy(), case.lengths[:1].numpy()
    qs = np.array([0, n], dtype=np.int32)
    Hq, D = q.shape[1], q.shape[2]
    flops = 4.0 * D * Hq * (n * (L - n) + n * (n + 1) // 2)
    reps, t_total = 0, 0.0
    while reps < max_reps and (reps == 0 or t_total < min_seconds):
        t0 = time.perf_counter()
        oracle.paged_prefill(q0, kp, vp, bt, lens, qs, case.scale, bs)
        t_total += time.perf_counter() - t0
        reps += 1
    sec = t_total / reps
    return {"value": flops / sec / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"1 of 8 sequences of the same workload (its {n} new queries, all {Hq} heads), "
                      f"{reps} repetition(s), {sec:.2f} s each, {t_total:.1f} s in all", "seconds_per_step": sec}


def run_blocks(args):
    """Whole-block copies for 2048 scattered blocks (256 MiB of K+V at 8 kv
    heads, bs 16, head_dim 128, bf16): pa_copy_blocks inside the device pool
    (copy-on-write) against the measured HBM copy bandwidth, and
    pa_swap_blocks between the device pool and a pinned host pool, each way,
    against a plain contiguous copy of the same bytes over the same host link
    (torch copy_, one DMA transfer) measured in the same run."""
    import paged_kv_cache_355_b200 as pa

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    NB, Hkv, bs, D = 2048, 8, 16, 128
    g = torch.Generator(device=dev).manual_seed(3001)
    k = torch.randn(NB, Hkv, bs, D, generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn(NB, Hkv, bs, D, generator=g, device=dev).to(torch.bfloat16)
    hk = torch.empty(NB, Hkv, bs, D, dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    perm = torch.randperm(NB, generator=torch.Generator().manual_seed(3002))
    m = torch.stack([torch.arange(NB), perm], 1).to(torch.int64).to(dev)
    nbytes = 2 * k.numel() * k.element_size()

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        evs = []
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            evs.append((e0, e1))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b_) for a, b_ in evs) / len(evs)

    # copy-on-write inside a 4096-block device pool: blocks 0..2047 to 2048..4095, scattered
    pool_k = torch.empty(2 * NB, Hkv, bs, D, dtype=torch.bfloat16, device=dev).normal_()
    pool_v = torch.empty_like(pool_k).normal_()
    cp = torch.stack([perm, NB + torch.randperm(NB, generator=torch.Generator().manual_seed(3003))], 1)
    cp = cp.to(torch.int64).to(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    with ClockSampler(0) as clocks:
        evs = []
        for i in range(args.warmup + args.steps):
            flush.zero_()
            clean.sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            pa.pa_copy_blocks(pool_k, pool_v, cp)
            e1.record()
            if i >= args.warmup:
                evs.append((e0, e1))
        torch.cuda.synchronize()
        ms_copy = sum(a.elapsed_time(b_) for a, b_ in evs) / len(evs)
        ms_out = timed(lambda: pa.pa_swap_blocks(k, v, hk, hv, m))
        ms_in = timed(lambda: pa.pa_swap_blocks(hk, hv, k, v, m))
        ms_d2h = timed(lambda: (hk.copy_(k, non_blocking=True), hv.copy_(v, non_blocking=True)))
        ms_h2d = timed(lambda: (k.copy_(hk, non_blocking=True), v.copy_(hv, non_blocking=True)))
    assert pa.pa_read_error_flag() == 0
    gbs = lambda ms: nbytes / (ms * 1e-3) / 1e9
    out, inn, d2h, h2d = gbs(ms_out), gbs(ms_in), gbs(ms_d2h), gbs(ms_h2d)
    copy_gbs = 2 * nbytes / (ms_copy * 1e-3) / 1e9  # read and written
    peak, peak_kind = measured_hbm_peak()
    print(json.dumps({
        "metric": "pa_copy_blocks GB/s vs HBM peak; pa_swap_blocks host-link GB/s vs a plain copy",
        "value": copy_gbs, "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "2048 scattered blocks, 8 kv heads, block_size 16, head_dim 128, bf16 "
                               f"({nbytes} bytes of K and V per direction)",
                   "l2": "flushed before each copy_blocks launch (256 MiB written, 256 MiB read)"},
        "roofline": {"bound": "hbm", "achieved": copy_gbs, "peak": peak, "unit": "GB/s", "frac": copy_gbs / peak,
                     "traffic": None, "kernel": "pa_copy_blocks (read + written bytes)",
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)"},
        "copy_blocks": {"ms": ms_copy, "gbs": copy_gbs},
        "swap_out": {"ms": ms_out, "gbs": out, "frac_of_plain_copy": out / d2h},
        "swap_in": {"ms": ms_in, "gbs": inn, "frac_of_plain_copy": inn / h2d},
        "host_link": {"d2h_gbs": d2h, "h2d_gbs": h2d,
                      "source": "torch copy_ of the same bytes, contiguous, measured in this run"},
        "clocks": clocks.summary()}), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.op == "prefill":
        run_prefill(args)
        return
    if args.op == "blocks":
        run_blocks(args)
        return
    run_ours(args)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
