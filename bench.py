#!/usr/bin/env python
"""Benchmark of the SegPagedAttention hot path on B200.

A step is one pass of the whole hot path over every layer of the workload: storage accounting and
work planning on the host, the build scatter of the layer's K/V into its pages, and the mask-free
paged prefill. The metric is visible-KV TFLOP/s: 4 * D * sum |V(i)| over every (query row, query head)
of every layer, divided by the step time (CUDA events, max over ranks).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference|dense]

With N > 1 every rank runs its own replica of the workload on its own GPU (rank-specific seeds, no
data-path collective: weak scaling); rank 0 prints one JSON line. Under torchrun the ranks come from its
environment; run plainly with --gpus N, bench.py starts the N ranks itself.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "visible-KV TFLOP/s and ms per layer for SegPagedAttention prefill; % roofline"
DEFAULT_WORKLOAD = "dsv4-flash"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["head_sparse_paged_b200/csrc/prefill_sm100.cuh", "head_sparse_paged_b200/csrc/sm100_ptx.cuh",
                  "head_sparse_paged_b200/csrc/plan.h"]


# ----------------------------------------------------------------------------------- utilities

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference", "dense"],
                    help="ours: the SegPaged library; reference: the fp64 oracle on the host cores; dense: "
                         "the dense-layout baseline (PyTorch SDPA, all heads at full context, explicit mask)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--no-mass", action="store_true",
                    help="skip the token-mass / top-k selection measurement (sparse-FFN score)")
    ap.add_argument("--no-rope-gather", action="store_true",
                    help="skip the gather-time RoPE measurement (prefill with per-fragment key re-alignment)")
    ap.add_argument("--no-append", action="store_true",
                    help="skip the fused append-and-attend measurement")
    ap.add_argument("--fragment-tokens", type=int, default=4096,
                    help="tokens per reused fragment in the gather-time RoPE measurement")
    ap.add_argument("--topk-frac", type=float, default=0.25,
                    help="share of each sequence's query tokens the top-k selection keeps")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the one-layer Qwen3-32B- and Llama-3.3-70B-shaped prefill measurements")
    ap.add_argument("--no-dense", action="store_true",
                    help="skip the dense-layout baseline (explicit mask) on an all-global and a mixed layer")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--no-graphs", action="store_true",
                    help="issue each prefill call directly instead of replaying its CUDA graph")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="budget of the oracle sample (per step in --impl reference)")
    return ap.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a float over all ranks (host-side reporting only; not on the data path)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(name: str, rank: int):
    """The workload of one rank: same shapes, rank-specific seed (independent replicas)."""
    from head_sparse_paged_b200 import synth
    w = synth.get(name)
    if rank:
        w = dataclasses.replace(w, seed=w.seed + 100003 * rank)
    return w


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_per_launch(workload: str):
    """DRAM bytes per prefill launch of this workload from profiles/prefill_traffic_<workload>.json (an ncu
    capture summary), if it was taken on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", f"prefill_traffic_{workload}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("kernel_sources_sha256") != kernel_source_hash():
        return None
    v = d.get("dram_bytes_per_launch")
    return float(v) if v is not None else None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every `interval` seconds while active."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, interval: float = 0.1):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.interval = interval
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:   # the NVML handle of the physical GPU behind this CUDA device
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self._reasons_fn(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(self.interval)

    def __enter__(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------------------ oracle timing

def oracle_sample(w, inputs_for_head, seconds: float, seed: int = 0):
    """Times the fp64 oracle on a bounded, seeded sample of the workload's (row, query head) items.

    inputs_for_head(layer, b, kh) -> oracle Problem of that (sequence, KV head). Items are drawn from
    every layer class present, in rounds, until the time budget is spent. Returns (visible TFLOP/s,
    sample description, threads)."""
    import numpy as np
    from head_sparse_paged_b200.counts import visible_counts
    from oracle import reference as orc

    lib = orc.OracleLib()
    rng = np.random.default_rng(seed)
    kinds = {}
    for li in range(w.layers):                       # one layer of each kind (number of global heads)
        kinds.setdefault(int(w.classes[li][..., 0].sum()), li)
    layers = sorted(kinds.values())
    done_flops, spent, items_done = 0.0, 0.0, 0
    scale = 1.0 / math.sqrt(w.head_dim)
    cache = {}
    t_end = time.time() + seconds
    rounds = 0
    while time.time() < t_end and rounds < 64:
        rounds += 1
        for li in layers:
            b = int(rng.integers(w.num_seqs))
            kh = int(rng.integers(w.num_kv_heads))
            key = (li, b, kh)
            if key not in cache:
                if len(cache) > 8:
                    cache.pop(next(iter(cache)))
                cache[key] = inputs_for_head(li, b, kh)
            pb = cache[key]
            Lq = w.q_lens[b]
            rows = rng.integers(0, Lq, size=8)
            items = np.array([(int(r), h) for r in rows for h in range(w.group)], np.int64)
            cnt = visible_counts(w, li, b, kh)
            t0 = time.perf_counter()
            lib.attention(pb, scale, items)
            spent += time.perf_counter() - t0
            done_flops += 4.0 * w.head_dim * float(sum(cnt[int(r)] for r in rows)) * w.group
            items_done += len(items)
            if time.time() >= t_end:
                break
    threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    desc = (f"{items_done} (query row, head) items of layers {layers} drawn at random, timed {spent:.1f} s; "
            f"fp64 C oracle, OpenMP over items")
    return done_flops / spent / 1e12, desc, threads


def oracle_head_inputs_from_synth(w):
    """Oracle inputs regenerated on the CPU from the seeded generators (used by --impl reference)."""
    import numpy as np
    import torch
    from head_sparse_paged_b200 import synth
    from oracle import reference as orc

    dense = {}

    def get(li, b, kh):
        src = 0 if w.layers > 1 else li
        if src not in dense:
            q, k, v = synth.layer_inputs(w, src, device="cpu")
            dense[src] = (k, v)
        k, v = dense[src]
        q = synth.layer_inputs(w, li, device="cpu", parts="q")[0]
        return _head_problem(w, li, b, kh, q, k, v)

    return get


def _head_problem(w, li, b, kh, q, k, v):
    import numpy as np
    from oracle import reference as orc
    G = w.group
    cq, ck = w.cu_q(), w.cu_k()
    qs = q[cq[b]:cq[b + 1], kh * G:(kh + 1) * G].float().cpu().numpy()
    ks = k[ck[b]:ck[b + 1], kh:kh + 1].float().cpu().numpy()
    vs = v[ck[b]:ck[b + 1], kh:kh + 1].float().cpu().numpy()
    if w.rope_theta is not None:
        ks = orc.rope_rotate_bf16(ks, orc.rope_cos_sin(w.rope_theta, [w.rope_deltas[b]], w.head_dim)[0])
    g, S, W = (int(x) for x in w.classes[li, b, kh])
    return orc.Problem(qs, ks, vs, np.array([0, w.q_lens[b]], np.int32), np.array([0, w.ctx_lens[b]], np.int32),
                       np.array([[g]]), np.array([[S]]), np.array([[W]]))


# -------------------------------------------------------------------------------------- arms

def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores, on this workload's config and metric."""
    if rank != 0:
        return 0
    from head_sparse_paged_b200.counts import visible_flops
    w = rank_workload(args.workload, 0)
    get = oracle_head_inputs_from_synth(w)
    per_step = max(0.2, min(20.0, 150.0 / max(1, args.steps + args.warmup), args.cpu_seconds))
    for _ in range(args.warmup):
        oracle_sample(w, get, per_step / 4, seed=1)
    vals = []
    desc = threads = None
    for s in range(args.steps):
        v, desc, threads = oracle_sample(w, get, per_step, seed=100 + s)
        vals.append(v)
    value = statistics.median(vals)
    flops = visible_flops(w)
    ms = flops / (value * 1e12) * 1e3
    from oracle import reference as orc
    stored = 0
    for li in range(w.layers):
        c = w.classes[li]
        stored += orc.pages_bytes(w.cu_k(), w.cu_q(), c[..., 0], c[..., 1], c[..., 2], w.page_size, w.head_dim)[0]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world, stored),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: {desc}; step time extrapolated by visible FLOPs"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def dense_chunk_rows(w, L: int) -> int:
    """Query rows per SDPA call of the dense-layout baseline: each call's boolean mask stays near 2 GB."""
    return max(1, int(2e9 // (w.num_q_heads * L)))


def dense_layer_ms(w, li, q, k_all, v_all, device):
    """Attention time of one layer in the dense layout: every head keeps its full context as a dense
    [Hq, L, D] K/V and visibility is an explicit boolean mask given to PyTorch's scaled_dot_product_attention
    (the masked slow path SegPagedAttention avoids). Query rows are chunked (dense_chunk_rows); each chunk's
    mask is built before its call and only the attention calls are timed, each between its own CUDA events,
    after one untimed pass."""
    import torch
    import torch.nn.functional as F
    G, D = w.group, w.head_dim
    scale = 1.0 / math.sqrt(D)
    cq, ck = w.cu_q(), w.cu_k()
    ms = 0.0
    for b in range(w.num_seqs):
        L, Lq = w.ctx_lens[b], w.q_lens[b]
        if Lq == 0:
            continue
        kk = k_all[ck[b]:ck[b + 1]].transpose(0, 1).repeat_interleave(G, dim=0)[None]   # [1, Hq, L, D]
        vv = v_all[ck[b]:ck[b + 1]].transpose(0, 1).repeat_interleave(G, dim=0)[None]
        qq = q[cq[b]:cq[b + 1]].transpose(0, 1)[None]                                      # [1, Hq, Lq, D]
        cls = torch.from_numpy(w.classes[li, b]).to(device).repeat_interleave(G, dim=0)  # [Hq, 3]
        glob, S, W = cls[:, 0, None, None] != 0, cls[:, 1, None, None], cls[:, 2, None, None]
        j = torch.arange(L, device=device)[None, None, :]
        chunk = dense_chunk_rows(w, L)
        pairs = []
        for rep in range(2):          # the first pass warms up; only the second is timed
            for r0 in range(0, Lq, chunk):
                i = (L - Lq + torch.arange(r0, min(r0 + chunk, Lq), device=device))[None, :, None]
                m = ((j <= i) & (glob | (j < S) | (j > i - W)))[None]
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                F.scaled_dot_product_attention(qq[:, :, r0:r0 + m.shape[2]], kk, vv, attn_mask=m, scale=scale)
                e1.record()
                if rep == 1:
                    pairs.append((e0, e1))
                del m
        torch.cuda.synchronize()
        ms += sum(a.elapsed_time(b_) for a, b_ in pairs)
        del kk, vv
    return ms


def run_dense(args, rank, world, local):
    """Dense-layout baseline on the same GPU (dense_layer_ms), one layer of each kind (number of global heads),
    weighted by how many layers of that kind the workload has."""
    if rank != 0:
        return 0
    import torch
    from head_sparse_paged_b200 import synth
    from head_sparse_paged_b200.counts import visible_flops
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = rank_workload(args.workload, 0)
    kinds = {}
    for li in range(w.layers):
        kinds.setdefault(int(w.classes[li][..., 0].sum()), []).append(li)
    per_layer_ms, ms_step = {}, 0.0
    _, k_all, v_all = synth.layer_inputs(w, 0, device=device)
    for key, lis in kinds.items():
        li = lis[0]
        q = synth.layer_inputs(w, li, device=device, parts="q")[0]
        if w.layers == 1:
            _, k_all, v_all = synth.layer_inputs(w, li, device=device)
        ms_layer = dense_layer_ms(w, li, q, k_all, v_all, device)
        per_layer_ms[f"{len(lis)} layers with {key} global heads"] = ms_layer
        ms_step += ms_layer * len(lis)
    flops = visible_flops(w)
    line = {
        "impl": "dense", "metric": METRIC, "value": flops / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": 1, "ms_per_step": ms_step, "ms_per_layer": ms_step / w.layers, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic", "dense_ms_by_layer_kind": per_layer_ms,
        "query_chunk_rows": {str(L): dense_chunk_rows(w, L) for L in sorted(set(w.ctx_lens))},
        "workload": w.name,
        "note": "PyTorch SDPA with an explicit boolean mask over dense K/V of every head at full context; "
                "value = visible FLOPs / time, so it is directly comparable with the SegPaged line",
    }
    print(json.dumps(line))
    return 0


def workload_config(w, world: int, stored_bytes: int):
    """The `config` object of every arm's line: the workload, how it is replicated, and why L2 cannot hold it.
    stored_bytes: K+V page bytes of all layers (the page pool, which each step streams)."""
    return {"workload": w.name, "description": w.description, "layers": w.layers, "seq_lens": list(w.ctx_lens),
            "q_lens": list(w.q_lens), "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "page_size": w.page_size, "page_order": w.page_order,
            "global_batch": w.num_seqs * world, "parallelism": f"replicas x{world}" if world > 1 else "single",
            "l2": f"inputs larger than L2 (page pool {stored_bytes / 1e9:.2f} GB per replica, all read every step)"
                  if stored_bytes > 126e6 else f"page pool {stored_bytes / 1e6:.1f} MB fits in L2",
            "dense_kv_source": "shared by all layers" if w.layers > 1 else "per layer"}


def run_ours(args, rank, world, local):
    import numpy as np
    import torch
    from head_sparse_paged_b200.counts import visible_flops
    from head_sparse_paged_b200.runner import Runner

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = rank_workload(args.workload, rank)
    runner = Runner(w, device=device, keep_dense=True, shared_dense=(w.layers > 1), mass=not args.no_mass,
                    graphs=not args.no_graphs)
    torch.cuda.synchronize()
    runner.check_status()
    flops_layer = {li: visible_flops(w, [li]) for li in runner.layers}
    flops_step = sum(flops_layer.values())
    stream = torch.cuda.current_stream()
    n_layers = len(runner.layers)

    # per-prefill-launch events (on the launching stream) for the dominant kernel's roofline
    ev = {}

    def mark(li, start):
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        ev.setdefault(li, []).append(e)

    for _ in range(args.warmup):
        runner.full_step()
    torch.cuda.synchronize()
    runner.check_status()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            runner.full_step(on_prefill=mark)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms_total = reduce_max(t0.elapsed_time(t1), world, device)
    runner.check_status()
    prefill_ms = {li: [ev[li][2 * s].elapsed_time(ev[li][2 * s + 1]) for s in range(args.steps)] for li in ev}
    prefill_total_ms = sum(sum(v) for v in prefill_ms.values())
    ms_step = ms_total / args.steps
    value = world * flops_step * args.steps / (ms_total * 1e-3) / 1e12
    achieved = sum(flops_layer[li] * len(prefill_ms[li]) for li in prefill_ms) / (prefill_total_ms * 1e-3) / 1e12
    peaks, src = load_peaks()
    # A kernel timed inside a long run (or one whose clock the power cap held down) is held to the sustained GEMM
    # peak, a short burst at full clocks to the burst peak.
    clocks = clk.summary()
    sustained = ms_total >= 1000.0 or ("sw_power_cap" in (clocks.get("reasons") or []) and
                                       (clocks.get("sm_mhz") or 0) < (clocks.get("sm_max_mhz") or 0))
    tf_name = "bf16_tflops_sustained" if sustained and "bf16_tflops_sustained" in peaks else "bf16_tflops"
    peak_tf = float(peaks[tf_name])
    peak_bw = float(peaks.get("hbm_gbs"))
    traffic = traffic_per_launch(w.name)
    # algorithmic bytes of each prefill launch: stored K/V pages read once, Q read, O and LSE written
    qo_bytes = w.total_q * w.num_q_heads * (w.head_dim * 2 * 2 + 4)
    bytes_layer = {li: runner.state[li].stored_bytes + qo_bytes for li in runner.layers}
    t_tensor = sum(flops_layer.values()) / (peak_tf * 1e12)
    t_hbm = sum(bytes_layer.values()) / (peak_bw * 1e9)
    if t_hbm > t_tensor:
        bound, unit, peak = "hbm", "GB/s", peak_bw
        achieved = sum(bytes_layer[li] * len(prefill_ms[li]) for li in prefill_ms) / (prefill_total_ms * 1e-3) / 1e9
        peak_name = "hbm_gbs"
    else:
        bound, unit, peak = "tensor", "TFLOP/s", peak_tf
        peak_name = tf_name
    kinds = {}
    for li in runner.layers:
        kinds.setdefault("all-global" if runner.state[li].cls[..., 0].all() else "mixed", []).append(li)
    per_kind = {k: {"layers": len(v), "prefill_ms": statistics.mean(statistics.mean(prefill_ms[li]) for li in v),
                    "visible_tflop": flops_layer[v[0]] / 1e12} for k, v in kinds.items()}
    stored = sum(runner.state[li].stored_bytes for li in runner.layers)
    dense = sum(runner.state[li].dense_bytes for li in runner.layers)

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(runner, args, world, device, flops_step)
    mass = None
    if not args.no_mass:
        mass = measure_mass(runner, args, world, device)
    rope_gather = None
    if not args.no_rope_gather and runner.rope is None:
        rope_gather = measure_rope_gather(runner, args, device, flops_layer, prefill_total_ms / args.steps)
    append = None
    if not args.no_append and runner.rope is None:
        append = measure_append(runner, args, device, flops_layer, prefill_total_ms / args.steps)

    # the 32K-128K single-layer configurations and the dense-layout baseline, beside the headline (one GPU only)
    workloads = None
    if world == 1 and not args.no_workloads:
        workloads = measure_workloads(args, device, [n for n in ("qwen3-32b", "llama-3.3-70b") if n != w.name])
    dense_baseline = None
    if world == 1 and not args.no_dense:
        dense_baseline = measure_dense_baseline(runner, device, prefill_ms)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        def inputs(li, b, kh):
            k, v = runner.dense_of(li)
            return _head_problem(w, li, b, kh, runner.state[li].q, k, v)
        v_cpu, desc, threads = oracle_sample(w, inputs, args.cpu_seconds)
        cpu = {"value": v_cpu, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}

    if rank != 0:
        return 0
    cfg = workload_config(w, world, stored)
    launches_layer = {li: 2 + (1 if runner.state[li].info["num_groups"] > 0 else 0) for li in runner.layers}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "ms_per_layer": prefill_total_ms / args.steps / n_layers,
        "prefill_ms_by_layer_kind": per_kind,
        "kv_bytes": {"segpaged": stored, "dense": dense, "ratio": dense / max(stored, 1)},
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "traffic": traffic,
                     "algorithmic_bytes_per_step": sum(bytes_layer.values()),
                     "prefill_tflops": sum(flops_layer[li] * len(prefill_ms[li]) for li in prefill_ms)
                     / (prefill_total_ms * 1e-3) / 1e12,
                     "peak_source": f"{src} {peak_name}", "kernel": "segpaged_prefill_kernel"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "workloads": workloads,
        "dense_baseline": dense_baseline,
        "token_mass": mass,
        "rope_gather": rope_gather,
        "append": append,
        "gpu_launches": args.steps * sum(launches_layer.values()),
        "gpu_launches_note": "per layer and step: build scatter, prefill, and the combine where the plan splits units",
        "prefill_submission": "direct C-ABI call" if args.no_graphs else
                              "CUDA graph of the C-ABI call per layer (captured in warm-up, replayed every step)",
        "clocks": clocks,
    }
    print(json.dumps(line))
    return 0


def _roofline(w, flops: float, nbytes: float, ms: float, peaks: dict, tf_name: str, src: str):
    """Bound (the slower of visible FLOPs at the tensor peak and algorithmic bytes at HBM bandwidth), achieved rate
    and fraction of one launch that took `ms`."""
    peak_tf, peak_bw = float(peaks[tf_name]), float(peaks["hbm_gbs"])
    if nbytes / (peak_bw * 1e9) > flops / (peak_tf * 1e12):
        ach = nbytes / (ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": peak_bw, "unit": "GB/s", "frac": ach / peak_bw,
                "peak_source": f"{src} hbm_gbs"}
    ach = flops / (ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": ach, "peak": peak_tf, "unit": "TFLOP/s", "frac": ach / peak_tf,
            "peak_source": f"{src} {tf_name}"}


def measure_workloads(args, device, names):
    """Prefill of one layer of each named workload (Qwen3-32B-shaped 128K and Llama-3.3-70B-shaped 16-32K batch),
    set up through the same C ABI and timed like the headline's kernel: CUDA events around each launch (the
    prefill, and the combine where the plan splits units), W warm-up launches, then max(K, 30) timed ones, with
    the SM clock sampled every 10 ms. The fraction is taken against the burst GEMM peak, or the sustained one when
    the power cap held the median SM clock below its maximum during the launches."""
    import torch
    from head_sparse_paged_b200 import synth
    from head_sparse_paged_b200.counts import visible_flops
    from head_sparse_paged_b200.runner import Runner
    peaks, src = load_peaks()
    out = {}
    for name in names:
        w = synth.get(name)
        r = Runner(w, device=device, graphs=not args.no_graphs)
        torch.cuda.synchronize()
        r.check_status()
        stream = torch.cuda.current_stream()
        for _ in range(args.warmup):
            r.prefill(0)
        torch.cuda.synchronize()
        ev = []
        with ClockSampler(device.index if device.index is not None else 0, interval=0.01) as clk:
            for _ in range(max(args.steps, 30)):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                r.prefill(0)
                b.record(stream)
                ev.append((a, b))
            torch.cuda.synchronize()
        r.check_status()
        ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
        flops = visible_flops(w, [0])
        nbytes = r.state[0].stored_bytes + w.total_q * w.num_q_heads * (w.head_dim * 2 * 2 + 4)
        ck = clk.summary()
        # held to the sustained GEMM peak when the power cap held the clock down during these launches (median SM
        # clock below the maximum), else to the burst peak
        capped = "sw_power_cap" in (ck.get("reasons") or []) and \
            (ck.get("sm_mhz") or 0) < (ck.get("sm_max_mhz") or 0)
        tf_name = "bf16_tflops_sustained" if capped and "bf16_tflops_sustained" in peaks else "bf16_tflops"
        rl = _roofline(w, flops, nbytes, ms, peaks, tf_name, src)
        out[name] = {"prefill_ms": ms, "visible_tflop": flops / 1e12, "tflops": flops / (ms * 1e-3) / 1e12,
                     "algorithmic_bytes": nbytes, **rl, "split_plan": r.state[0].info["num_groups"] > 0,
                     "clocks": ck, "launches": len(ev)}
        del r
        torch.cuda.empty_cache()
    return out


def measure_dense_baseline(runner, device, prefill_ms):
    """The dense-layout baseline (dense_layer_ms) on the first layer of each kind of the workload (all-global, mixed),
    against the SegPaged prefill of the same layer from the timed steps."""
    w = runner.w
    out = {}
    done = set()
    for li in runner.layers:
        kind = "all-global" if runner.state[li].cls[..., 0].all() else "mixed"
        if kind in done:
            continue
        done.add(kind)
        k, v = runner.dense_of(li)
        ms = dense_layer_ms(w, li, runner.state[li].q, k, v, device)
        ours = statistics.mean(prefill_ms[li])
        out[kind] = {"layer": li, "dense_ms": ms, "segpaged_prefill_ms": ours, "ratio": ms / ours}
    out["query_chunk_rows"] = {str(L): dense_chunk_rows(w, L) for L in sorted(set(w.ctx_lens))}
    out["method"] = ("PyTorch scaled_dot_product_attention over dense K/V of every head at full context with an "
                     "explicit boolean mask, query rows chunked so each mask stays near 2 GB, only the attention "
                     "calls timed (CUDA events), after one untimed pass")
    return out


# MUFU peak for the token-mass pass: 16 ex2 per clock per SM (sm_100), 148 SMs, at the maximum SM clock.
MUFU_EX2_PER_CLK_SM = 16


def measure_mass(runner, args, world, device):
    """Token-mass pass plus top-k selection of every layer, after the timed prefill steps (it needs their
    LSE): CUDA events around each mass launch, K steps after W warm-up steps."""
    import numpy as np
    import torch
    w = runner.w
    stream = torch.cuda.current_stream()
    k_per_seq = torch.tensor([max(1, int(round(args.topk_frac * l))) for l in w.q_lens], dtype=torch.int32,
                             device=device)
    selected = torch.empty(int(k_per_seq.sum().item()), dtype=torch.int32, device=device)
    from head_sparse_paged_b200.counts import mass_pairs
    pairs = {li: mass_pairs(w, li) for li in runner.layers}
    for _ in range(args.warmup):
        for li in runner.layers:
            runner.token_mass(li)
            runner.select_topk(li, k_per_seq, selected)
    torch.cuda.synchronize()
    ev = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index if device.index is not None else 0, interval=0.01) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            for li in runner.layers:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                runner.token_mass(li)
                b.record(stream)
                runner.select_topk(li, k_per_seq, selected)
                ev.append((li, a, b))
        t1.record(stream)
        torch.cuda.synchronize()
    runner.check_status()
    total_ms = t0.elapsed_time(t1)
    mass_ms = sum(a.elapsed_time(b) for _, a, b in ev)
    exps = sum(pairs[li] for li, _, _ in ev)
    peaks, _ = load_peaks()
    clk_hz = float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    peak = MUFU_EX2_PER_CLK_SM * torch.cuda.get_device_properties(device).multi_processor_count * clk_hz
    achieved = exps / (mass_ms * 1e-3)
    ck = clk.summary()
    # the same peak at the SM clock sampled during these launches (under the power cap the clock sits below max)
    at_clock = peak * (ck["sm_mhz"] * 1e6 / clk_hz) if ck.get("sm_mhz") else None
    return {"kernel": "segpaged_mass_kernel (+ reduce)", "ms_per_layer": mass_ms / len(ev),
            "with_topk_ms_per_layer": total_ms / len(ev), "visible_pairs_per_step": sum(pairs.values()),
            "bound": "alu", "achieved": achieved / 1e9, "peak": peak / 1e9, "unit": "G exp2/s",
            "frac": achieved / peak, "peak_source": f"{MUFU_EX2_PER_CLK_SM} ex2/clk/SM x SMs x sm_max_mhz",
            "frac_at_sampled_clock": achieved / at_clock if at_clock else None, "clocks": ck,
            "topk_frac": args.topk_frac}


def measure_rope_gather(runner, args, device, flops_layer, plain_prefill_ms_per_step):
    """Prefill of every layer with gather-time RoPE: each sequence is a run of reused fragments of
    --fragment-tokens tokens, each re-aligned from a seeded original offset to where it now sits. Timed like
    the main prefill launches (CUDA events around each launch), K steps after W warm-up steps."""
    import numpy as np
    import torch
    from head_sparse_paged_b200 import segpaged as sp
    w = runner.w
    rng = np.random.default_rng(w.seed + 4242)
    offs, starts, deltas = [0], [], []
    for L in w.ctx_lens:
        st = list(range(0, L, args.fragment_tokens))
        starts += st
        deltas += [int(s0 - o) for s0, o in zip(st, rng.integers(0, 1 << 16, size=len(st)))]
        offs.append(len(starts))
    tab = sp.segpaged_rope_cos_sin(1e6, deltas, w.head_dim)
    runner.frags = (torch.tensor(offs, dtype=torch.int32, device=device),
                    torch.tensor(starts, dtype=torch.int32, device=device),
                    torch.from_numpy(tab).to(device))
    stream = torch.cuda.current_stream()
    try:
        for _ in range(args.warmup):
            for li in runner.layers:
                runner.prefill(li)
        torch.cuda.synchronize()
        ev = []
        for _ in range(args.steps):
            for li in runner.layers:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                runner.prefill(li)
                b.record(stream)
                ev.append((li, a, b))
        torch.cuda.synchronize()
        runner.check_status()
    finally:
        frags = runner.frags
        runner.frags = None
    ms = sum(a.elapsed_time(b) for _, a, b in ev)
    flops = sum(flops_layer[li] for li, _, _ in ev)
    per_step = ms / args.steps
    # the alternative: one re-alignment pass per layer into a second K pool, then the plain prefill on it
    k_out = torch.empty_like(runner.k_pool)

    def realigned(li):
        st = runner.state[li]
        sp.segpaged_rope_realign(runner.dims, runner.cu_k_dev, runner.ql_dev, st.cls_dev, st.table_dev, st.offs_dev,
                                 *frags, runner.k_pool, k_out, runner.status)
        sp.segpaged_attn_prefill(runner.dims, st.q, k_out, runner.v_pool, st.table_dev, st.units_dev, st.info,
                                 runner.scale, st.o, st.lse, runner.workspace, runner.status)

    for _ in range(args.warmup):
        for li in runner.layers:
            realigned(li)
    torch.cuda.synchronize()
    ev2 = []
    for _ in range(args.steps):
        for li in runner.layers:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            realigned(li)
            b.record(stream)
            ev2.append((li, a, b))
    torch.cuda.synchronize()
    runner.check_status()
    # the caller-level choice between the two (Runner.prefill_rope_auto), timed the same way
    runner.frags = frags
    try:
        for _ in range(args.warmup):
            for li in runner.layers:
                runner.prefill_rope_auto(li, k_out)
        torch.cuda.synchronize()
        ev3, path = [], None
        for _ in range(args.steps):
            for li in runner.layers:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                path = runner.prefill_rope_auto(li, k_out)
                b.record(stream)
                ev3.append((li, a, b))
        torch.cuda.synchronize()
        runner.check_status()
    finally:
        runner.frags = None
    del k_out
    ms2 = sum(a.elapsed_time(b) for _, a, b in ev2)
    ms3 = sum(a.elapsed_time(b) for _, a, b in ev3)
    return {"kernel": "segpaged_prefill_kernel<ROPE>", "fragment_tokens": args.fragment_tokens,
            "auto_path": path, "auto_ms_per_layer": ms3 / len(ev3), "auto_tflops": flops / (ms3 * 1e-3) / 1e12,
            "auto_time_vs_plain_prefill": (ms3 / args.steps) / plain_prefill_ms_per_step,
            "fragments": len(starts), "prefill_ms_per_layer": ms / len(ev),
            "tflops": flops / (ms * 1e-3) / 1e12, "time_vs_plain_prefill": per_step / plain_prefill_ms_per_step,
            "realign_then_prefill_ms_per_layer": ms2 / len(ev2),
            "realign_then_prefill_tflops": flops / (ms2 * 1e-3) / 1e12,
            "realign_time_vs_plain_prefill": (ms2 / args.steps) / plain_prefill_ms_per_step}


def measure_append(runner, args, device, flops_layer, plain_prefill_ms_per_step):
    """Fused append-and-attend for every layer: the query rows' keys and values (gathered from the layer's
    dense K/V) are written into their pool pages by the same launch that attends over them. The pool
    already holds those rows, so the measurement leaves it unchanged. CUDA events around each launch."""
    import numpy as np
    import torch
    from head_sparse_paged_b200 import segpaged as sp
    w = runner.w
    ck = w.cu_k()
    rows = torch.cat([torch.arange(int(ck[b + 1]) - w.q_lens[b], int(ck[b + 1]), device=device)
                      for b in range(w.num_seqs)])
    plans, news = {}, {}
    ws = runner.workspace
    for li in runner.layers:
        st = runner.state[li]
        units, info = sp.segpaged_prefill_plan_append(runner.dims, runner.ctx, runner.ql, st.cls, st.offs,
                                                      runner.split_ctas)
        plans[li] = (torch.from_numpy(np.ascontiguousarray(units)).to(device), info)
        need = sp.segpaged_prefill_workspace_bytes(runner.dims, info)
        if ws.numel() * 4 < need:
            ws = torch.zeros((need + 3) // 4, dtype=torch.int32, device=device)
        key = 0 if runner.shared_dense else li
        if key not in news:
            k, v = runner.dense_of(li)
            news[key] = (k[rows].contiguous(), v[rows].contiguous())
    stream = torch.cuda.current_stream()

    def call(li):
        st = runner.state[li]
        kn, vn = news[0 if runner.shared_dense else li]
        sp.segpaged_attn_prefill_append(runner.dims, st.q, kn, vn, runner.k_pool, runner.v_pool, st.table_dev,
                                        plans[li][0], plans[li][1], runner.scale, st.o, st.lse, ws, runner.status)

    for _ in range(args.warmup):
        for li in runner.layers:
            call(li)
    torch.cuda.synchronize()
    ev = []
    for _ in range(args.steps):
        for li in runner.layers:
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call(li)
            b.record(stream)
            ev.append((li, a, b))
    torch.cuda.synchronize()
    runner.check_status()
    ms = sum(a.elapsed_time(b) for _, a, b in ev)
    flops = sum(flops_layer[li] for li, _, _ in ev)
    return {"kernel": "segpaged_prefill_kernel<append>", "prefill_ms_per_layer": ms / len(ev),
            "tflops": flops / (ms * 1e-3) / 1e12,
            "appended_bytes_per_layer": 2 * int(rows.numel()) * w.num_kv_heads * w.head_dim * 2,
            "time_vs_plain_prefill": (ms / args.steps) / plain_prefill_ms_per_step}


def measure_e2e(runner, args, world, device, flops_step):
    """Same metric through the public API with host buffers: every step copies the queries of every
    layer and the work plan from pinned host memory and reads O and LSE back into pinned host memory.
    The copies run on their own streams, ahead of the compute stream (plans and queries) and behind it
    (outputs), ordered by events, as a pipelined serving loop would run them."""
    import torch
    q_host = {li: runner.state[li].q.cpu().pin_memory() for li in runner.layers}
    o_host = {li: torch.empty_like(runner.state[li].o, device="cpu").pin_memory() for li in runner.layers}
    l_host = {li: torch.empty_like(runner.state[li].lse, device="cpu").pin_memory() for li in runner.layers}
    h2d = sum(q_host[li].numel() * 2 + runner.state[li].units.nbytes for li in runner.layers)
    d2h = sum(o_host[li].numel() * 2 + l_host[li].numel() * 4 for li in runner.layers)
    comp = torch.cuda.current_stream()
    s_in = torch.cuda.Stream(device=device)
    s_out = torch.cuda.Stream(device=device)
    # per layer: last compute that read Q / wrote O, last read-back of O
    q_free = {li: None for li in runner.layers}
    o_free = {li: None for li in runner.layers}

    def step():
        ready = {}
        for li in runner.layers:
            # Storage accounting and planning on the host; the plan and the queries go up on the input
            # stream as soon as the layer's buffers are free. The compute stream issues no host copies:
            # a small plan upload queued there would wait behind the large query copies on the copy engine.
            runner.account_layer(li)
            runner.plan_layer(li)
            with torch.cuda.stream(s_in):
                if q_free[li] is not None:
                    s_in.wait_event(q_free[li])
                runner.upload_plan(li, s_in)
                runner.state[li].q.copy_(q_host[li], non_blocking=True)
                ready[li] = torch.cuda.Event()
                ready[li].record(s_in)
        for li in runner.layers:
            comp.wait_event(ready[li])
            if o_free[li] is not None:
                comp.wait_event(o_free[li])
            runner.build_layer(li, comp)
            runner.prefill(li, comp)
            done = torch.cuda.Event()
            done.record(comp)
            q_free[li] = done
            with torch.cuda.stream(s_out):            # outputs back while the next layers compute
                s_out.wait_event(done)
                o_host[li].copy_(runner.state[li].o, non_blocking=True)
                l_host[li].copy_(runner.state[li].lse, non_blocking=True)
                o_free[li] = torch.cuda.Event()
                o_free[li].record(s_out)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    steps = max(1, min(args.steps, 5))
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    s_in.wait_event(t0)
    s_out.wait_event(t0)
    for _ in range(steps):
        step()
    for li in runner.layers:                          # the step ends when every read-back has landed
        comp.wait_event(o_free[li])
    t1.record(comp)
    torch.cuda.synchronize()
    ms = reduce_max(t0.elapsed_time(t1), world, device)
    return {"value": world * flops_step * steps / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ms / steps,
            "copies": "plans and queries in on one stream, outputs out on another, overlapped with compute "
                      "layer by layer"}


def _free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _rank_entry(target, argv, env):
    os.environ.update(env)
    sys.exit(int(target(argv) or 0))


def spawn_ranks(nprocs: int, target, argv) -> int:
    """Runs target(argv) as ranks 0 .. nprocs-1 of one job on this node, each in a fresh process (spawn, so no
    CUDA state is inherited) with the environment torchrun would give it (RANK, LOCAL_RANK, WORLD_SIZE,
    MASTER_ADDR=127.0.0.1, a free MASTER_PORT). Rank r uses GPU r. Returns the largest exit code of the ranks."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = []
    for r in range(nprocs):
        env = {"RANK": str(r), "LOCAL_RANK": str(r), "WORLD_SIZE": str(nprocs), "LOCAL_WORLD_SIZE": str(nprocs),
               "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)}
        p = ctx.Process(target=_rank_entry, args=(target, list(argv), env))
        p.start()
        procs.append(p)
    rc = 0
    for p in procs:
        p.join()
        code = p.exitcode if p.exitcode is not None else 1
        rc = max(rc, code if code >= 0 else 1)
    return rc


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    args = parse_args(argv)
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # started plainly with --gpus N: run the N ranks here, one process and one GPU each
        return spawn_ranks(args.gpus, main, argv)
    rank, world, local = dist_env()
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but the job has {world} ranks", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.impl == "dense":
        return run_dense(args, rank, world, local)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        # NCCL carries only the reporting barrier and max-over-ranks reduction: the replicas share no data
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        return run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
