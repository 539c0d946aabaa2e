"""Per-CTA timelines of one decode-attention or prefill call, from
libpa_timeline.so (libpa with globaltimer stamps compiled into the decode and
prefill kernels; the events are listed in include/pa_timeline.h).

    python -m paged_kv_cache_355_b200.timeline [--workload cow] [--repeats 3] [--json out.json]

With --workload prefill the call is pa_paged_attention_prefill on the
chunked-prefill workload (batch 8, 32 q / 8 kv heads, head_dim 128, bs 16,
context 4096 of which the last 2048 tokens are new), launched directly after
an L2 flush; printed per repeat: the CTAs' lives, entry to the first S MMA,
last P.V to exit, exit to the next CTA's entry on the same SM, the CTAs per
SM, the share of SM time between each CTA's first S and last P.V, and when
each SM finished.

The workload's decode call (the shared-prefix call for the shared-prefix
workload, the plain call otherwise) is captured as a CUDA graph and replayed
with L2 flushed before each replay; the stamps are cleared and one more
replay is recorded.  Printed per repeat, in microseconds from the first CTA's
entry:
  * each kernel's CTA entries and exits (percentiles) and the end of the call;
  * resident CTAs of each kernel every 5 us;
  * pass 1's phases per CTA (prologue: entry to the block-table slice staged;
    first stage: to the first K/V stage landed; stream; epilogue), a
    least-squares fit of a CTA's life against the tokens it reads (its
    sequence found through the launch order: longest first, as the kernel
    ranks it, for the plain call on batches up to 2048, index order
    otherwise), and the CTAs' summed lives divided by the most that were
    resident at once;
  * the prefix pass's per-tile chain: medians over CTAs of the time from a
    tile's scores to its P, from P to its P.V issue, from the V request to the
    P.V issue, from the K request to the S issue, and the tile period.
A profiling aid: the stamps add a few stores per CTA to the kernels.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os

import numpy as np

KERNELS = ("set-up kernel", "prefix pass", "pass 1")
TL_CTAS, TL_SLOTS = 65536, 16
TT_CTAS, TT_TILES, TT_EVENTS = 512, 16, 8
PF_CTAS, PF_SLOTS = 65536, 8
# the chunked-prefill workload: batch, q heads, kv heads, head_dim, block
# size, context, new tokens (seeds 2001 for the cache, 2002 for q)
PREFILL_SHAPE = (8, 32, 8, 128, 16, 4096, 2048)


def _load(path: str):
    from . import _binding as b

    lib = ctypes.CDLL(path)
    for name, (argtypes, restype) in b._SIGS.items():
        f = getattr(lib, name)
        f.argtypes, f.restype = argtypes, restype
    lib.pa_timeline_clear.argtypes, lib.pa_timeline_clear.restype = [], ctypes.c_int
    lib.pa_timeline_read.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t]
    lib.pa_timeline_read.restype = ctypes.c_int
    lib.pa_timeline_clear_prefill.argtypes, lib.pa_timeline_clear_prefill.restype = [], ctypes.c_int
    lib.pa_timeline_read_prefill.argtypes = [ctypes.c_void_p, ctypes.c_size_t]
    lib.pa_timeline_read_prefill.restype = ctypes.c_int
    return lib


def _pct(a) -> list:
    a = np.asarray(a, float)
    a = a[~np.isnan(a)]
    return [round(float(x), 2) for x in np.percentile(a, [0, 10, 50, 90, 100])] if a.size else []


def _summary(ev: np.ndarray, tt: np.ndarray, own_tokens) -> dict:
    """ev: [3, TL_CTAS, TL_SLOTS] u64; tt: [TT_CTAS, TT_TILES, TT_EVENTS] u64."""
    used = [ev[k][ev[k][:, 0] > 0] for k in range(3)]
    t0 = min(int(u[:, 0].min()) for u in used if len(u))
    rel = [np.where(u[:, :TL_SLOTS - 1] > 0, (u[:, :TL_SLOTS - 1].astype(np.int64) - t0) / 1e3, np.nan) for u in used]
    out = {"ctas": [int(len(u)) for u in used], "kernels": {}}
    end = 0.0
    for k, name in enumerate(KERNELS):
        r = rel[k]
        if not len(r):
            continue
        out["kernels"][name] = {"entry_us": _pct(r[:, 0]), "exit_us": _pct(r[:, 2])}
        end = max(end, float(np.nanmax(r[:, 2])))
    out["call_end_us"] = round(end, 2)
    grid = np.arange(0.0, end + 5.0, 5.0)
    out["resident"] = {"t_us": grid.tolist()}
    for k, name in enumerate(KERNELS):
        r = rel[k]
        if len(r):
            out["resident"][name] = [int(((r[:, 0] <= x) & (r[:, 2] > x)).sum()) for x in grid]
    p1 = rel[2]
    if len(p1):
        phases = {"prologue": p1[:, 1] - p1[:, 0], "first stage": p1[:, 3] - p1[:, 1], "stream": p1[:, 4] - p1[:, 3],
                  "epilogue": p1[:, 2] - p1[:, 4], "life": p1[:, 2] - p1[:, 0]}
        out["pass1_phases_us"] = {n: _pct(v) for n, v in phases.items()}
        peak = max(out["resident"]["pass 1"]) if "pass 1" in out["resident"] else 0
        if peak:
            out["pass1_summed_life_per_slot_us"] = round(float(np.nansum(phases["life"])) / peak, 2)
        if own_tokens is not None:
            ids = np.nonzero(ev[2][:, 0] > 0)[0]
            tok = np.asarray(own_tokens(ids), float)
            ok = ~np.isnan(phases["life"])
            A = np.vstack([np.ones(ok.sum()), tok[ok]]).T
            c = np.linalg.lstsq(A, phases["life"][ok], rcond=None)[0]
            out["pass1_life_fit"] = {"fixed_us": round(float(c[0]), 2), "ns_per_token": round(float(c[1]) * 1e3, 2),
                                     "mean_tokens": round(float(tok[ok].mean()), 1)}
    if len(rel[1]) and (tt[:, :, 0] > 0).any():
        T = np.where(tt > 0, (tt.astype(np.int64) - t0) / 1e3, np.nan)
        med = lambda x: round(float(np.nanmedian(x)), 2)
        chain = []
        for j in range(1, min(TT_TILES, 8)):
            a, p = T[:, j], T[:, j - 1]
            if np.isnan(a[:, 0]).all():
                break
            chain.append({"tile": j, "period": med(a[:, 0] - p[:, 0]), "scores_to_P": med(a[:, 1] - a[:, 0]),
                          "P_to_PV": med(a[:, 3] - a[:, 1]), "Vreq_to_PV": med(a[:, 3] - a[:, 6]),
                          "Kreq_to_S": med(a[:, 4] - a[:, 5]), "S_to_scores": med(a[:, 0] - a[:, 4])})
        out["prefix_tiles_us"] = chain
    return out


def _prefill_summary(ev: np.ndarray) -> dict:
    """ev: [PF_CTAS, PF_SLOTS] u64 of one prefill launch (slots: 0 entry, 1
    ready, 2 first S, 3 and 4 the tiles' last P.V, 5 exit, 7 SM id)."""
    ev = ev.astype(np.int64)
    ran = ev[:, 0] > 0
    e = ev[ran]
    t0 = e[:, 0].min()
    us = lambda c: (e[:, c] - t0) / 1000.0
    entry, ready, first_s, exit_ = us(0), us(1), us(2), us(5)
    last_pv = np.maximum(us(3), np.where(e[:, 4] > 0, us(4), 0.0))
    sm = e[:, PF_SLOTS - 1]
    span = float(exit_.max())
    gaps, windows, per_sm, last_exit = [], 0.0, [], []
    for s in np.unique(sm):
        idx = np.where(sm == s)[0]
        o = idx[np.argsort(entry[idx])]
        gaps += list(entry[o[1:]] - exit_[o[:-1]])
        windows += float(np.sum(last_pv[o] - first_s[o]))
        per_sm.append(len(o))
        last_exit.append(float(exit_[o].max()))
    sms = len(per_sm)
    return {"ctas": int(ran.sum()), "sms": sms, "span_us": round(span, 2), "life_us": _pct(exit_ - entry),
            "entry_to_ready_us": _pct(ready - entry), "entry_to_first_S_us": _pct(first_s - entry),
            "last_PV_to_exit_us": _pct(exit_ - last_pv), "exit_to_next_entry_us": _pct(gaps),
            "ctas_per_sm": _pct(per_sm), "first_S_to_last_PV_share": round(windows / (sms * span), 4) if sms else 0.0,
            "sm_last_exit_us": _pct(last_exit)}


def run_prefill(repeats: int = 3) -> list:
    import torch

    from . import _binding as b
    from .build import TIMELINE_LIB
    from .workloads import custom_case

    if not os.path.exists(TIMELINE_LIB):
        raise RuntimeError("libpa_timeline.so is not built (python -m paged_kv_cache_355_b200.build)")
    lib = _load(TIMELINE_LIB)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, Hq, Hkv, D, bs, L, n = PREFILL_SHAPE
    case = custom_case([L] * B, Hq, Hkv, D, bs, torch.bfloat16, seed=2001, device=dev)
    qs = torch.arange(0, (B + 1) * n, n, dtype=torch.int32, device=dev)
    g = torch.Generator(device=dev).manual_seed(2002)
    q = torch.randn(B * n, Hq, D, generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty(B * n, Hq, D, dtype=torch.bfloat16, device=dev)
    bt, lens = case.block_tables.to(dev), case.lengths.to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    saved = b._lib
    b._lib = lib
    try:
        fn = lambda: b.pa_paged_attention_prefill(q, case.k_pool, case.v_pool, bt, lens, qs, n, case.scale, out)
        results = []
        for _ in range(repeats):
            for _ in range(3):
                flush.zero_()
                fn()
            torch.cuda.synchronize()
            if lib.pa_timeline_clear_prefill() != 0:
                raise RuntimeError("pa_timeline_clear_prefill failed")
            flush.zero_()
            torch.cuda.synchronize()
            fn()
            torch.cuda.synchronize()
            if b.pa_read_error_flag() != 0:
                raise RuntimeError("the prefill call flagged an error")
            ev = np.zeros(PF_CTAS * PF_SLOTS, np.uint64)
            if lib.pa_timeline_read_prefill(ev.ctypes.data, ev.nbytes):
                raise RuntimeError("pa_timeline_read_prefill failed")
            results.append(_prefill_summary(ev.reshape(PF_CTAS, PF_SLOTS)))
    finally:
        b._lib = saved
    return results


def launch_order(lengths: np.ndarray, max_len: int, max_batch: int = 2048) -> np.ndarray:
    """The sequence at each rank of plain decode's longest-first launch
    order: 64 length buckets (longest first), ties by index; index order for
    batches above max_batch, where the kernel does not rank."""
    n = len(lengths)
    if n > max_batch:
        return np.arange(n)
    L = np.clip(lengths.astype(np.int64), 0, max_len)
    key = 63 - np.minimum(63, (L * 64) // (max_len + 1))
    return np.array(sorted(range(n), key=lambda b: (key[b], b)))


def run(workload: str = "cow", repeats: int = 3) -> list:
    import torch

    from . import _binding as b
    from .build import TIMELINE_LIB
    from .workloads import make_case, shared_prefix_groups

    if not os.path.exists(TIMELINE_LIB):
        raise RuntimeError("libpa_timeline.so is not built (python -m paged_kv_cache_355_b200.build)")
    lib = _load(TIMELINE_LIB)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    case = make_case(workload, device=dev)
    w = case.workload
    bt, lens = case.block_tables.to(dev), case.lengths.to(dev)
    out = torch.empty(w.batch, w.num_q_heads, w.head_dim, device=dev)
    groups = shared_prefix_groups(case)
    saved = b._lib
    b._lib = lib
    try:
        part = b.pa_paged_attention_partition_size(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, case.max_len,
                                                   w.block_size)
        if groups is not None:
            gs = torch.tensor(groups[0], dtype=torch.int32, device=dev)
            gl = torch.tensor(groups[1], dtype=torch.int32, device=dev)
            mp, mg = max(groups[1]), max(e - s for s, e in zip(groups[0][:-1], groups[0][1:]))
            fn = lambda: b.pa_paged_attention_decode_shared_prefix(case.q, case.k_pool, case.v_pool, bt, lens,
                                                                   case.max_len, case.scale, out, gs, gl, mp, mg,
                                                                   partition_size=part)
            prefix = np.zeros(w.batch, np.int64)
            for g, P in enumerate(groups[1]):
                prefix[groups[0][g]:groups[0][g + 1]] = P
            order = np.arange(w.batch)  # the shared-prefix call keeps index order
        else:
            fn = lambda: b.pa_paged_attention_decode(case.q, case.k_pool, case.v_pool, bt, lens, case.max_len,
                                                     case.scale, out, partition_size=part)
            prefix = np.zeros(w.batch, np.int64)
            order = launch_order(case.lengths.numpy(), case.max_len)
        # pass 1's grid is (splits, kv heads, rank): a CTA reads the tokens of
        # its split of the sequence at its rank, after the sequence's prefix
        L = np.clip(case.lengths.numpy().astype(np.int64), 0, case.max_len)
        splits = -(-case.max_len // part)

        def own_tokens(ids):
            x, z = ids % splits, ids // (splits * w.num_kv_heads)
            seq = order[z]
            return np.clip(L[seq] - prefix[seq] - x * part, 0, part)
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        results = []
        for _ in range(repeats):
            for _ in range(3):
                flush.zero_()
                g.replay()
            torch.cuda.synchronize()
            if lib.pa_timeline_clear() != 0:
                raise RuntimeError("pa_timeline_clear failed")
            flush.zero_()
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            if b.pa_read_error_flag() != 0:
                raise RuntimeError("the decode call flagged an error")
            ev = np.zeros(3 * TL_CTAS * TL_SLOTS, np.uint64)
            tt = np.zeros(TT_CTAS * TT_TILES * TT_EVENTS, np.uint64)
            if lib.pa_timeline_read(0, ev.ctypes.data, ev.nbytes) or lib.pa_timeline_read(1, tt.ctypes.data, tt.nbytes):
                raise RuntimeError("pa_timeline_read failed")
            results.append(_summary(ev.reshape(3, TL_CTAS, TL_SLOTS), tt.reshape(TT_CTAS, TT_TILES, TT_EVENTS),
                                    own_tokens))
        del g
    finally:
        b._lib = saved
    return results


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--workload", default="cow")
    ap.add_argument("--repeats", type=int, default=3)
    ap.add_argument("--json", default=None, help="also write the summaries here")
    a = ap.parse_args()
    if a.workload == "prefill":
        res = run_prefill(a.repeats)
        for i, r in enumerate(res):
            print(f"== prefill, launch {i}: span {r['span_us']} us, {r['ctas']} CTAs on {r['sms']} SMs "
                  f"(p0 p10 p50 p90 p100, us)")
            for k in ("life_us", "entry_to_ready_us", "entry_to_first_S_us", "last_PV_to_exit_us",
                      "exit_to_next_entry_us", "ctas_per_sm", "sm_last_exit_us"):
                print(f"  {k:24s} {r[k]}")
            print(f"  first S to last P.V, share of SM time: {r['first_S_to_last_PV_share']}")
        if a.json:
            with open(a.json, "w") as f:
                json.dump(res, f, indent=1)
        return
    res = run(a.workload, a.repeats)
    for i, r in enumerate(res):
        print(f"== {a.workload}, replay {i}: call end {r['call_end_us']} us, CTAs {r['ctas']}")
        for name, k in r["kernels"].items():
            print(f"  {name:14s} entry {k['entry_us']}  exit {k['exit_us']}  (p0 p10 p50 p90 p100, us)")
        for name, v in r.get("pass1_phases_us", {}).items():
            print(f"  pass 1 {name:12s} {v}")
        if "pass1_life_fit" in r:
            f = r["pass1_life_fit"]
            print(f"  pass 1 life = {f['fixed_us']} us + {f['ns_per_token']} ns per token read "
                  f"(mean {f['mean_tokens']} tokens)")
        if "pass1_summed_life_per_slot_us" in r:
            print(f"  pass 1 summed CTA lives / peak resident CTAs: {r['pass1_summed_life_per_slot_us']} us")
        for c in r.get("prefix_tiles_us", []):
            print(f"  prefix tile {c['tile']}: period {c['period']}, scores->P {c['scores_to_P']}, "
                  f"P->P.V {c['P_to_PV']}, V req->P.V {c['Vreq_to_PV']}, K req->S {c['Kreq_to_S']}, "
                  f"S->scores {c['S_to_scores']}")
        t = r["resident"]
        print("  t (us)   " + " ".join(f"{x:5.0f}" for x in t["t_us"]))
        for name in KERNELS:
            if name in t:
                print(f"  {name[:8]:8s} " + " ".join(f"{x:5d}" for x in t[name]))
    if a.json:
        with open(a.json, "w") as f:
            json.dump(res, f, indent=1)


if __name__ == "__main__":
    main()
