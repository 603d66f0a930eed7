#!/usr/bin/env python
"""Benchmark of one gated block-sparse decode step on B200.

A step is the whole hot path on one batch: kpool refresh of the open block,
gate scores, block selection, split-KV sparse decode and the merge of the
split partials -- run as ONE cooperative launch (seer_decode_step). Inputs are
seeded synthetic tensors resident in HBM before timing starts. Consecutive
steps rotate over several independent input sets (caches, queries, weights,
pooled keys; the same lengths), so each step reads inputs that five other
steps' traffic -- more than the 126 MB L2, in normal-priority data alone --
has passed through since their last use: cold data, as for one layer of a
model whose other layers run in between, while the kernel's code stays
resident as it would in that loop. (--l2 flush instead writes a 256 MiB
buffer before each step on a single set, which also evicts the code; that
figure is reported as a secondary key.) A short device sleep before each step
lets the host enqueue it ahead of the GPU; neither is inside the timed
interval, a pair of CUDA events on the launching stream around the step.

The same step as the five separate C calls is timed afterwards (secondary
numbers, with the sparse decode kernel bracketed alone).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); the path has no exchange step, so
each rank runs an independent replica batch (weak scaling) and the step time
is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse decode attention µs/step and HBM GB/s vs ~8 TB/s at 90% sparsity"
UNIT = "us/step"
DEFAULT_WORKLOAD = "decode_b16"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "sparse_decode_traffic.json")
# the sources the fused step kernel is compiled from: a recorded traffic figure holds only while they are unchanged
DECODE_SRCS = [os.path.join(ROOT, "block_sparse_attention_seer_b200", "csrc", f)
               for f in ("sparse_decode.cu", "gate_core.cuh", "seer_device.cuh")]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--batch", type=int, default=0, help="override the workload's batch (small profiling cases)")
    p.add_argument("--e2e-steps", type=int, default=200)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    p.add_argument("--dense-steps", type=int, default=30, help="timed steps of the dense baseline (0: skip)")
    p.add_argument("--mass-steps", type=int, default=30, help="timed calls of the block-level ground truth (0: skip)")
    p.add_argument("--variant-steps", type=int, default=30, help="timed calls of each gate variant (0: skip)")
    p.add_argument("--prefill-steps", type=int, default=3, help="timed block-sparse prefills (0: skip)")
    p.add_argument("--prefill-batch", type=int, default=4, help="sequences of the prefill measurement")
    p.add_argument("--config-steps", type=int, default=100,
                   help="timed fused steps of each other decode workload (large block, ragged, sweep; 0: skip)")
    p.add_argument("--l2", default="rotate", choices=["rotate", "flush"],
                   help="cold inputs by rotating over independent input sets, or by a 256 MiB memset per step")
    p.add_argument("--sets", type=int, default=6, help="input sets of the rotation")
    p.add_argument("--flush-steps", type=int, default=300,
                   help="timed steps of the secondary memset-flush measurement of the headline (0: skip)")
    return p.parse_args()


# ---------------------------------------------------------------- shared helpers

def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def prefill_flops(lens, idx, nsel, blk, D, G):
    """Useful flops of the causal block-sparse prefill: 4 D per (query token, visible key token) per head."""
    B, Hkv, nbm, kmax = idx.shape
    L = np.asarray(lens, np.int64)[:, None, None, None]
    i = np.arange(nbm, dtype=np.int64)[None, None, :, None]
    j = idx.astype(np.int64)
    live = (np.arange(kmax)[None, None, None, :] < nsel[..., None]) & (j >= 0)
    nq = np.clip(L - i * blk, 0, blk)
    nk = np.clip(L - j * blk, 0, blk)
    pairs = np.where(j < i, nq * nk, np.where(j == i, nq * (nq + 1) // 2, 0))
    return int(4 * D * G * np.where(live, pairs, 0).sum())


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(wl, seq_lens, block_idx, num_selected):
    """Bytes the step must move: kept K+V tokens, the pooled-K scan, q and out.

    Returns (step_bytes, decode_kernel_bytes, kept_tokens, kept_blocks).
    """
    B, Hkv, D, dg, blk = wl.batch, wl.num_kv_heads, wl.head_dim, wl.gate_dim, wl.block_size
    toks = 0
    blocks = 0
    nb_total = 0
    for b in range(B):
        L = int(seq_lens[b])
        nb = -(-L // blk)
        nb_total += nb * Hkv
        for h in range(Hkv):
            n = int(num_selected[b, h])
            for j in block_idx[b, h, :n]:
                j = int(j)
                if 0 <= j < nb:
                    toks += min(blk, L - j * blk)
                    blocks += 1
    kv = toks * D * 2 * 2
    qo = 2 * B * wl.num_q_heads * D * 2
    kp = nb_total * dg * 4
    return kv + kp + qo, kv + qo // 2, toks, blocks


def kernel_sources_sha256():
    h = hashlib.sha256()
    for path in DECODE_SRCS:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload=None):
    """DRAM traffic per fused-step launch from the committed ncu summary: only for the workload it
    was recorded for (full batch) and only while the kernel's sources are unchanged."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        if workload is not None and d.get("workload") != workload:
            return None
        if d.get("sources_sha256") != kernel_sources_sha256():
            return None
        return d
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", str(self.index)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (every rank calls it, same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def smi_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


def oracle_sample_time(wl, host, target_s):
    """Time the fp64 oracle step (as it stands) on the first n batch entries; scale to the whole batch.

    Returns (us_per_full_step, threads, description).
    """
    from oracle import oracle as O
    O.build()

    def run(n):
        q, k, v = host["q"][:n], host["k"][:n], host["v"][:n]
        t0 = time.perf_counter()
        O.step(q, k, v, host["w_q"], host["w_k"], host["lens"][:n], wl.block_size, wl.budget_tokens)
        return time.perf_counter() - t0

    t1 = run(1)
    n = max(1, min(wl.batch, int(target_s / max(t1, 1e-3))))
    reps = 1
    t = run(n) if n > 1 else t1
    while t * (reps + 1) / reps < target_s and reps < 50 and t < target_s / 2:
        t += run(n)
        reps += 1
    per_call = t / reps
    us = per_call * wl.batch / n * 1e6
    desc = (f"oracle step (pool all blocks, gate, select, attend; fp64) on the first {n} of {wl.batch} batch "
            f"entries ({n * wl.num_kv_heads} of {wl.batch * wl.num_kv_heads} (b, kv-head) rows), {reps} run(s), "
            f"scaled by {wl.batch}/{n}")
    return us, O.num_threads(), desc


def host_inputs(inp):
    from block_sparse_attention_seer_b200 import workloads as W
    return dict(q=W.bf16_bits(inp["q"]), k=W.bf16_bits(inp["k_cache"]), v=W.bf16_bits(inp["v_cache"]),
                w_q=inp["w_q"].cpu().numpy(), w_k=inp["w_k"].cpu().numpy(),
                lens=np.asarray(inp["seq_lens_host"], np.int32))


# ---------------------------------------------------------------- reference arm: the oracle on host cores

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    from block_sparse_attention_seer_b200 import workloads as W
    from oracle import oracle as O
    O.build()
    wl = W.WORKLOADS[args.workload]
    if args.batch:
        wl = wl.with_(batch=args.batch, name=f"{wl.name}_batch{args.batch}")
    inp = W.make_inputs(wl, seed=args.seed, device="cpu")
    host = host_inputs(inp)
    total_budget = 150.0
    n_steps = args.steps + args.warmup
    per_step = total_budget / max(1, n_steps)
    # size the per-step sample (batch entries) to the per-step budget
    t0 = time.perf_counter()
    O.step(host["q"][:1], host["k"][:1], host["v"][:1], host["w_q"], host["w_k"], host["lens"][:1],
           wl.block_size, wl.budget_tokens)
    t1 = time.perf_counter() - t0
    n = max(1, min(wl.batch, int(per_step / max(t1, 1e-4))))
    times = []
    for i in range(n_steps):
        t0 = time.perf_counter()
        O.step(host["q"][:n], host["k"][:n], host["v"][:n], host["w_q"], host["w_k"], host["lens"][:n],
               wl.block_size, wl.budget_tokens)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    us = float(np.mean(times)) * wl.batch / n * 1e6
    desc = (f"oracle step on the first {n} of {wl.batch} batch entries per step, scaled by {wl.batch}/{n}")
    line = {"impl": "reference", "metric": METRIC, "value": us, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "description": wl.description},
            "cpu_baseline": {"value": us, "unit": UNIT, "cores": O.num_threads(), "kind": "oracle", "sample": desc},
            "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    del torch
    return 0


# ---------------------------------------------------------------- the other decode workloads

SWEEP = [f"sweep_b{b}_keep{k}" for b in (1, 4) for k in ("50", "30", "10", "05")]
OTHER_WORKLOADS = ["large_block", "ragged"] + SWEEP


def other_configs(args, dev, world, peak, flush, stream):
    """The fused step on every other decode workload of the benchmark (same timing method as the
    headline), each with its algorithmic bytes and roofline fraction; each sweep batch also gets this
    build's dense decode (sparse decode + combine over every block, after a memset flush) beside it."""
    import torch

    from block_sparse_attention_seer_b200 import api
    from block_sparse_attention_seer_b200 import workloads as W

    def timed(fns, n, rotate):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        for k in range(n + 5 * len(fns)):
            if not rotate:
                flush.zero_()
            torch.cuda._sleep(300_000)
            kk = k - 5 * len(fns)
            e = evs[kk] if kk >= 0 else None
            if e:
                e[0].record(stream)
            fns[k % len(fns)]()
            if e:
                e[1].record(stream)
        torch.cuda.synchronize()
        us = float(np.mean([a.elapsed_time(b) for a, b in evs])) * 1e3
        return max_over_ranks([us], dev)[0] if world > 1 else us

    out = {}
    rank = int(os.environ.get("RANK", "0"))
    for name in OTHER_WORKLOADS + ["sweep_b1_dense", "sweep_b4_dense"]:
        wl = W.WORKLOADS[name]
        inp = W.make_inputs(wl, seed=args.seed + rank, device=dev)
        lens = inp["seq_lens_host"]
        entry = {"kept_fraction_target": None}
        if not name.endswith("_dense"):
            rot = args.l2 == "rotate"
            group = []  # the rotation's input sets (the first is `inp`), the same lengths
            for k in range(max(1, args.sets) if rot else 1):
                ik = inp if k == 0 else W.make_inputs(wl, seed=args.seed + rank + 1000 * k, device=dev,
                                                      seq_lens=lens)
                sk = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens, device=dev)
                sk.build_pool(ik["k_cache"], ik["w_k"], ik["seq_lens"])
                group.append((ik, sk))
            fns = [lambda i=i, s_=s_: s_.fused_step(i["q"], i["k_cache"], i["v_cache"], i["w_q"], i["w_k"],
                                                    i["seq_lens"]) for i, s_ in group]
            us = timed(fns, args.config_steps, rot)
            st = group[0][1]
            step_bytes, _, toks, blocks = algorithmic_bytes(wl, lens, st.block_idx.cpu().numpy(),
                                                            st.num_selected.cpu().numpy())
            entry = {"us": round(us, 3), "bytes": step_bytes, "kept_blocks": blocks,
                     "sparsity": round(1 - toks / float(sum(int(x) for x in lens) * wl.num_kv_heads), 4),
                     "gbs": round(step_bytes / (us * 1e-6) / 1e9, 1),
                     "frac": round(step_bytes / (us * 1e-6) / 1e9 / peak, 4),
                     "frac_of_8tbs": round(step_bytes / (us * 1e-6) / 8e12, 4),
                     "kernel": "decode_step_kernel (the whole step)"}
            del st, group, fns
        else:  # this build's dense flash-decode at all blocks selected
            st = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens, device=dev)
            nbm = wl.nb_max
            idx_d, ns_d = W.identity_block_list(lens, wl.num_kv_heads, wl.block_size, nbm)
            idx_d = torch.from_numpy(idx_d).to(dev)
            ns_d = torch.from_numpy(ns_d).to(dev)
            us = timed([lambda: st.attend(inp["q"], inp["k_cache"], inp["v_cache"], inp["seq_lens"], idx_d, ns_d,
                                          nbm)], max(10, args.config_steps // 4), False)
            _, dense_bytes, toks, _ = algorithmic_bytes(wl, lens, idx_d.cpu().numpy(), ns_d.cpu().numpy())
            entry = {"us": round(us, 3), "bytes": dense_bytes, "gbs": round(dense_bytes / (us * 1e-6) / 1e9, 1),
                     "frac": round(dense_bytes / (us * 1e-6) / 1e9 / peak, 4),
                     "kernel": "sparse_decode + combine over every block (no gate)"}
            del st, idx_d, ns_d
        entry["description"] = wl.description
        out[name] = entry
        del inp
        torch.cuda.empty_cache()
    for b in (1, 4):  # each sweep point against the dense decode of its batch
        d = out.get(f"sweep_b{b}_dense")
        for k in ("50", "30", "10", "05"):
            e = out.get(f"sweep_b{b}_keep{k}")
            if d and e:
                e["speedup_vs_dense"] = round(d["us"] / e["us"], 3)
    return out


# ---------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    from block_sparse_attention_seer_b200 import api
    from block_sparse_attention_seer_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wl = W.WORKLOADS[args.workload]
    if args.batch:
        wl = wl.with_(batch=args.batch, name=f"{wl.name}_batch{args.batch}")
    # the input sets of the rotation: independent data, the same lengths (so the same bytes per step)
    R = max(1, args.sets) if args.l2 == "rotate" else 1
    sets = []
    for k in range(R):
        ik = W.make_inputs(wl, seed=args.seed + rank + 1000 * k, device=dev,
                           seq_lens=sets[0][0]["seq_lens_host"] if sets else None)
        sk = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens, device=dev)
        sk.build_pool(ik["k_cache"], ik["w_k"], ik["seq_lens"])
        sk.set_update_start(ik["seq_lens"])
        sets.append((ik, sk, sk.parts(sk.num_splits)))
    inp, st, _ = sets[0]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def run_fused(k):
        i, s_, _ = sets[k % R]
        s_.fused_step(i["q"], i["k_cache"], i["v_cache"], i["w_q"], i["w_k"], i["seq_lens"])

    def run_gate_calls(k):
        i, s_, _ = sets[k % R]
        api.seer_kpool_update(s_.dims, i["k_cache"], i["w_k"], i["seq_lens"], s_.upd_start, s_.kpool)
        api.seer_gate_scores(s_.dims, i["q"], i["w_q"], s_.kpool, i["seq_lens"], s_.scores)
        api.seer_select_blocks(s_.dims, s_.scores, i["seq_lens"], s_.budget_tokens, s_.block_idx,
                               s_.num_selected)

    def run_decode(k):
        i, s_, (o_part, lse_part) = sets[k % R]
        api.seer_sparse_decode(s_.dims, i["q"], i["k_cache"], i["v_cache"], i["seq_lens"], s_.block_idx,
                               s_.num_selected, s_.kmax, s_.num_splits, 0.0, o_part, lse_part)

    def run_combine(k):
        i, s_, (o_part, lse_part) = sets[k % R]
        api.seer_combine(s_.dims, o_part, lse_part, s_.num_splits, s_.out, s_.lse)

    def prepare_flush():
        flush.zero_()
        torch.cuda._sleep(300_000)  # ~0.15 ms: the host enqueues the step ahead of the GPU

    def prepare():  # before a step of the rotation (or, with --l2 flush, the memset)
        if args.l2 == "flush":
            flush.zero_()
        torch.cuda._sleep(300_000)

    def fused_once(k, evs=None, flushed=False):
        (prepare_flush if flushed else prepare)()
        if evs:
            evs[0].record(stream)
        run_fused(k)
        if evs:
            evs[1].record(stream)

    def separate_once(k, evs=None, brackets=True):
        # brackets: events between the calls too (they also end each call's overlap with the next)
        prepare()
        if evs:
            evs[0].record(stream)
        run_gate_calls(k)
        if evs and brackets:
            evs[1].record(stream)
        run_decode(k)
        if evs and brackets:
            evs[2].record(stream)
        run_combine(k)
        if evs:
            evs[3].record(stream)

    for _ in range(args.warmup):
        for k in range(R):
            fused_once(k)
            separate_once(k)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(smi_index(local))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for k in range(args.steps):
        fused_once(k, ev[k])
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = np.array([e[0].elapsed_time(e[1]) for e in ev])
    ms_step = float(step_ms.mean())

    # secondary: the headline step on one input set with a 256 MiB memset before each step
    flushed = None
    if args.flush_steps > 0 and args.l2 == "rotate":
        fev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.flush_steps)]
        for k in range(args.flush_steps + 3):
            fused_once(0, fev[k - 3] if k >= 3 else None, flushed=True)
        torch.cuda.synchronize()
        flush_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in fev]))
        if world > 1:
            (flush_ms,) = max_over_ranks([flush_ms], dev)
        flushed = {"us": round(flush_ms * 1e3, 3), "steps": args.flush_steps,
                   "method": "one input set, 256 MiB memset before every step (evicts the code too)"}

    # the same step as five separate calls: the whole step (events around it only), then
    # the per-kernel brackets (events between the calls)
    n_sep = min(args.steps, 300)
    wev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_sep)]
    for k in range(n_sep):
        separate_once(k, wev[k], brackets=False)
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_sep)]
    for k in range(n_sep):
        separate_once(k, sev[k])
    torch.cuda.synchronize()
    sep_step_ms = float(np.mean([e[0].elapsed_time(e[3]) for e in wev]))
    sep_br_ms = float(np.mean([e[0].elapsed_time(e[3]) for e in sev]))
    ms_dec = float(np.mean([e[1].elapsed_time(e[2]) for e in sev]))
    gate_ms = np.array([e[0].elapsed_time(e[1]) for e in sev])
    if world > 1:
        ms_step, ms_dec, sep_step_ms, sep_br_ms = max_over_ranks([ms_step, ms_dec, sep_step_ms, sep_br_ms], dev)

    lens = inp["seq_lens_host"]
    sets_bytes = sum(t.numel() * t.element_size() for i, _, _ in sets for t in i.values() if torch.is_tensor(t))
    bidx = st.block_idx.cpu().numpy()
    nsel = st.num_selected.cpu().numpy()
    step_bytes, dec_bytes, toks, blocks = algorithmic_bytes(wl, lens, bidx, nsel)
    peak, peak_kind = measured_peak()
    achieved = step_bytes / (ms_step * 1e-3) / 1e9
    traffic = recorded_traffic(wl.name)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_kind": peak_kind, "kernel": "decode_step_kernel",
                "traffic": (traffic["dram_bytes_per_launch"] if traffic else None),
                "algorithmic_bytes_per_launch": step_bytes}
    if flushed:
        flushed["gbs"] = round(step_bytes / (flushed["us"] * 1e-6) / 1e9, 1)
        flushed["frac"] = round(step_bytes / (flushed["us"] * 1e-6) / 1e9 / peak, 4)
    dec_achieved = dec_bytes / (ms_dec * 1e-3) / 1e9
    separate = {"step_us": round(sep_step_ms * 1e3, 3), "launches_per_step": 5,
                "bracketed_step_us": round(sep_br_ms * 1e3, 3),
                "gate_select_us": round(float(gate_ms.mean()) * 1e3, 3),
                "sparse_decode_us": round(ms_dec * 1e3, 3),
                "sparse_decode_bytes": dec_bytes,
                "sparse_decode_gbs": round(dec_achieved, 1),
                "sparse_decode_frac": round(dec_achieved / peak, 4)}

    # ---- dense baseline: the same decode kernels over every block of every row (a4 + a5)
    dense = None
    if args.dense_steps > 0:
        nbm = wl.nb_max
        idx_d, ns_d = W.identity_block_list(lens, wl.num_kv_heads, wl.block_size, nbm)
        idx_d = torch.from_numpy(idx_d).to(dev)
        ns_d = torch.from_numpy(ns_d).to(dev)
        d_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.dense_steps)]
        for k in range(args.dense_steps + 3):
            prepare_flush()
            evs = d_ev[k - 3] if k >= 3 else None
            if evs:
                evs[0].record(stream)
            st.attend(inp["q"], inp["k_cache"], inp["v_cache"], inp["seq_lens"], idx_d, ns_d, nbm)
            if evs:
                evs[1].record(stream)
        torch.cuda.synchronize()
        dense_us = float(np.mean([e[0].elapsed_time(e[1]) for e in d_ev])) * 1e3
        if world > 1:
            (dense_us,) = max_over_ranks([dense_us], dev)
        _, dense_bytes, dense_toks, _ = algorithmic_bytes(wl, lens, idx_d.cpu().numpy(), ns_d.cpu().numpy())
        dense = {"decode_us": round(dense_us, 3), "kernels": "sparse_decode + combine over every block",
                 "tokens": dense_toks, "bytes": dense_bytes,
                 "gbs": round(dense_bytes / (dense_us * 1e-6) / 1e9, 1),
                 "frac": round(dense_bytes / (dense_us * 1e-6) / 1e9 / peak, 4),
                 "speedup_of_sparse_step": round(dense_us / (ms_step * 1e3), 3),
                 "speedup_of_sparse_decode": round(dense_us / (sep_br_ms * 1e3 - float(gate_ms.mean()) * 1e3), 3)}

    # ---- block-level ground truth (seer_block_mass): each head's dense softmax mass per block
    block_mass = None
    if args.mass_steps > 0:
        mass_buf = torch.empty(wl.batch, wl.num_q_heads, wl.nb_max, dtype=torch.float32, device=dev)
        mlse_buf = torch.empty(wl.batch, wl.num_q_heads, dtype=torch.float32, device=dev)
        m_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.mass_steps)]
        for k in range(args.mass_steps + 3):
            prepare_flush()
            evs = m_ev[k - 3] if k >= 3 else None
            if evs:
                evs[0].record(stream)
            api.seer_block_mass(st.dims, inp["q"], inp["k_cache"], inp["seq_lens"], mass_buf, mlse_buf)
            if evs:
                evs[1].record(stream)
        torch.cuda.synchronize()
        mass_us = float(np.mean([e[0].elapsed_time(e[1]) for e in m_ev])) * 1e3
        if world > 1:
            (mass_us,) = max_over_ranks([mass_us], dev)
        k_bytes = int(sum(min(int(L), wl.max_seq_len) for L in lens)) * wl.num_kv_heads * wl.head_dim * 2
        mass_bytes = k_bytes + wl.batch * wl.num_q_heads * (wl.head_dim * 2 + wl.nb_max * 4 + 4)
        block_mass = {"us": round(mass_us, 3), "kernels": "block_lse + block_mass_finalize",
                      "bytes": mass_bytes, "gbs": round(mass_bytes / (mass_us * 1e-6) / 1e9, 1),
                      "frac": round(mass_bytes / (mass_us * 1e-6) / 1e9 / peak, 4)}

    # ---- gate variants: per-head aggregations of the block scores and threshold selection
    variants = None
    if args.variant_steps > 0:
        def timed(fn):
            v_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.variant_steps)]
            for k in range(args.variant_steps + 3):
                prepare_flush()
                evs = v_ev[k - 3] if k >= 3 else None
                if evs:
                    evs[0].record(stream)
                fn()
                if evs:
                    evs[1].record(stream)
            torch.cuda.synchronize()
            us = float(np.mean([e[0].elapsed_time(e[1]) for e in v_ev])) * 1e3
            return max_over_ranks([us], dev)[0] if world > 1 else us
        nb_rows = [-(-min(int(L), wl.max_seq_len) // wl.block_size) for L in lens]
        kp_bytes = sum(nb_rows) * wl.num_kv_heads * wl.gate_dim * 4  # one scan of every row's pooled keys
        vs = torch.empty_like(st.scores)
        variants = {"scan_bytes": kp_bytes}
        for name, agg in (("mean", api.AGG_MEAN), ("max", api.AGG_MAX), ("softmax_mean", api.AGG_SOFTMAX_MEAN)):
            us = timed(lambda: api.seer_gate_scores_agg(st.dims, inp["q"], inp["w_q"], st.kpool, inp["seq_lens"],
                                                        agg, vs))
            variants[f"agg_{name}_us"] = round(us, 3)
            variants[f"agg_{name}_frac"] = round(kp_bytes / (us * 1e-6) / 1e9 / peak, 4)
        thr_idx = torch.empty_like(st.block_idx)
        thr_ns = torch.empty_like(st.num_selected)
        variants["threshold_select_us"] = round(timed(lambda: api.seer_select_blocks_threshold(
            st.dims, vs, inp["seq_lens"], st.budget_tokens, 0.0, thr_idx, thr_ns)), 3)

    # ---- block-sparse prefill over the workload's own caches (the prompt = the cached tokens)
    prefill = None
    if args.prefill_steps > 0:
        pb = min(wl.batch, args.prefill_batch)
        Hq, Hkv, D, blk = wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size
        nbm = wl.nb_max
        pdims = api.make_dims(pb, Hq, Hkv, D, wl.gate_dim, blk, wl.max_seq_len)
        gq = torch.Generator(device=dev).manual_seed(args.seed + 7)
        pq = torch.randn(pb, Hq, wl.max_seq_len, D, generator=gq, device=dev).to(torch.bfloat16)
        pk, pv = inp["k_cache"][:pb], inp["v_cache"][:pb]
        plen = inp["seq_lens"][:pb]
        pkp = st.kpool[:pb]
        psc = torch.empty(pb, Hkv, nbm, nbm, device=dev)
        pidx = torch.empty(pb, Hkv, nbm, st.kmax, dtype=torch.int32, device=dev)
        pns = torch.empty(pb, Hkv, nbm, dtype=torch.int32, device=dev)
        pout = torch.empty(pb, Hq, wl.max_seq_len, D, dtype=torch.bfloat16, device=dev)
        plse = torch.empty(pb, Hq, wl.max_seq_len, device=dev)
        calls = {
            "gate": lambda: api.seer_prefill_gate_scores(pdims, pq, inp["w_q"], pkp, plen, psc),
            "select": lambda: api.seer_prefill_select_blocks(pdims, psc, plen, wl.budget_tokens, pidx, pns),
            "attention": lambda: api.seer_prefill_attention(pdims, pq, pk, pv, plen, pidx, pns, st.kmax, pout, plse),
        }
        times = {}
        for name, fn in calls.items():
            p_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.prefill_steps)]
            for kk in range(args.prefill_steps + 1):
                prepare_flush()
                evs = p_ev[kk - 1] if kk >= 1 else None
                if evs:
                    evs[0].record(stream)
                fn()
                if evs:
                    evs[1].record(stream)
            torch.cuda.synchronize()
            t_us = float(np.mean([e[0].elapsed_time(e[1]) for e in p_ev])) * 1e3
            times[name] = max_over_ranks([t_us], dev)[0] if world > 1 else t_us
        flops = prefill_flops(lens[:pb], pidx.cpu().numpy(), pns.cpu().numpy(), blk, D, wl.group)
        tpeak, tkind = measured_tensor_peak()
        tflops = flops / (times["attention"] * 1e-6) / 1e12
        prefill = {"batch": pb, "prompt_tokens": [int(x) for x in lens[:pb]],
                   "gate_us": round(times["gate"], 1), "select_us": round(times["select"], 1),
                   "attention_us": round(times["attention"], 1), "attention_flops": flops,
                   "attention_tflops": round(tflops, 1), "bound": "tensor", "peak_tflops": tpeak,
                   "peak_kind": tkind, "frac": round(tflops / tpeak, 4),
                   "flops_counted": "4 D per (query token, causally visible key token of a kept block) per head"}
        del pq, psc, pidx, pns, pout, plse
        torch.cuda.empty_cache()

    # ---- end to end through the public API: host inputs in, host output out, every step.
    # The step's inputs (q and the new token's K/V rows) travel as one packed pinned buffer;
    # seer_append_kv places the token in the caches, the fused step runs, out comes back.
    e2e = None
    if args.e2e_steps > 0:
        B, Hq, Hkv, D = wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim
        nq, nkv = B * Hq * D, B * Hkv * D
        last = torch.from_numpy(np.maximum(lens.astype(np.int64) - 1, 0)).to(dev)
        rows_b = torch.arange(B, device=dev)
        packed = []
        for i, _, _ in sets:
            kn = i["k_cache"][rows_b, :, last, :]  # the token already in the cache: the step is unchanged
            vn = i["v_cache"][rows_b, :, last, :]
            packed.append(torch.cat([i["q"].reshape(-1), kn.reshape(-1), vn.reshape(-1)]).cpu().pin_memory())
        packed_h = packed[0]
        stage = torch.empty_like(packed_h, device=dev)
        q_d = stage[:nq].view(B, Hq, D)
        kn_d = stage[nq:nq + nkv].view(B, Hkv, D)
        vn_d = stage[nq + nkv:].view(B, Hkv, D)
        out_h = torch.empty(B, Hq, D, dtype=torch.bfloat16).pin_memory()
        h2d = packed_h.numel() * 2
        d2h = out_h.numel() * 2
        e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.e2e_steps)]
        for k in range(args.e2e_steps + 5):
            prepare()
            evs = e_ev[k - 5] if k >= 5 else None
            i, s_, _ = sets[k % R]
            if evs:
                evs[0].record(stream)
            stage.copy_(packed[k % R], non_blocking=True)
            api.seer_append_kv(s_.dims, kn_d, vn_d, i["seq_lens"], i["k_cache"], i["v_cache"])
            s_.fused_step(q_d, i["k_cache"], i["v_cache"], i["w_q"], i["w_k"], i["seq_lens"])
            out_h.copy_(s_.out, non_blocking=True)
            if evs:
                evs[1].record(stream)
        torch.cuda.synchronize()
        e2e_us = float(np.mean([e[0].elapsed_time(e[1]) for e in e_ev])) * 1e3
        if world > 1:
            (e2e_us,) = max_over_ranks([e2e_us], dev)
        e2e = {"value": round(e2e_us, 3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h),
               "path": "one packed H2D (q, new K, new V) -> seer_append_kv -> seer_decode_step -> D2H of out"}

    configs = None
    if args.config_steps > 0:
        configs = other_configs(args, dev, world, peak, flush, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        us, cores, desc = oracle_sample_time(wl, host_inputs(inp), args.cpu_seconds)
        cpu = {"value": round(us, 1), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(ms_step * 1e3, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 6),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 KV cache and query, random N(0,1/D) gate weights)",
            "config": {"workload": wl.name, "description": wl.description, "batch": wl.batch,
                       "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                       "gate_dim": wl.gate_dim, "block_size": wl.block_size, "max_seq_len": wl.max_seq_len,
                       "budget_tokens": wl.budget_tokens, "num_splits": st.num_splits,
                       "kept_blocks": blocks, "kept_tokens": toks,
                       "sparsity": round(1 - toks / float(sum(int(x) for x in lens) * wl.num_kv_heads), 4),
                       "parallelism": f"replicas x{world}",
                       "l2": (f"inputs larger than L2: steps rotate over {R} independent input sets "
                              f"({sets_bytes / 2**30:.1f} GiB), no flush" if args.l2 == "rotate" else
                              "256 MiB memset before every step, outside the timed interval"),
                       "timing": "CUDA events per step on the launching stream; mean over steps; max over ranks"},
            "step_bytes": step_bytes,
            "step_hbm_gbs": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
            "step_frac_of_8tbs": round(step_bytes / (ms_step * 1e-3) / 8e12, 4),
            "step_us_p50": round(float(np.median(step_ms)) * 1e3, 3),
            "l2_flush": flushed,
            "separate_calls": separate,
            "dense_baseline": dense,
            "block_mass": block_mass,
            "gate_variants": variants,
            "prefill": prefill,
            "other_workloads": configs,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps,
            "clocks": clocks,
            "wall_s": round(wall, 3),
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
