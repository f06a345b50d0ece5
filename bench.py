#!/usr/bin/env python
"""Benchmark of the paged-KV attention step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: the host work
partition (pa_plan_build), then the cache write and varlen paged attention in
one call (pa_reshape_and_attention: the scatter kernel, the split-KV decode
kernel + combine, and the tensor-core prefill kernel when the batch holds long
segments; with --two-calls, pa_reshape_and_cache then pa_attention_varlen).  Inputs are
seeded and synthetic with the shapes of the named workload (model names give
attention shapes only; no weights).  Default workload: the 8192-token mixed
chunked-prefill step with the Qwen2.5-1.5B attention shape (1152 decodes, a
2048-token chunk on 6144 cached tokens, fresh prompts of 1024/1536/2432).

Timing: W untimed warm-up steps, then K timed steps bracketed by a barrier and
torch.cuda.synchronize() on both sides.  L2 is flushed before every step: a
1 GiB write, then a read of another 1 GiB buffer, so that a step starts with
none of its data in L2 and no dirty lines of the flush buffer either (their
write-back would otherwise be charged to the step's first kernel).  Each
step's device time is taken with CUDA events on the launching stream,
excluding the flush; the host plan for a step is built and its kernels
queued while the flush runs, so the events see device time rather than host
launch overhead.  Multi-GPU (torchrun): every rank runs its own batch of
the same shape (weak scaling, no collective on the data path); the reported
time is the max over ranks.

The JSON line adds: roofline (dominant kernel, timed in the same run with
CUDA events around it on its stream, in a second pass of K identical steps,
since event records cost GPU time of their own; for the decode kernel also
a device copy of the same bytes timed the same way, what a plain copy
reaches in one launch at that size), the scatter kernel's own
roofline (back-to-back launches on distinct inputs and slots, after an L2
flush), e2e (same metric through the public API with host buffers: after a
flush and a synchronize, the host clock runs from before the step's plan
build through the copy of its inputs, kept in one page-locked buffer, to the
device, the step itself and the copy of its output back, until that copy has
landed; the step's e2e time is the larger of that host interval and the
events around the same work), the host cost of a plan build on an idle
plan, the CPU oracle as a reported baseline, SM clocks sampled during the
timed region, the number of library kernels launched, and kv_transfer:
pa_kv_export and pa_kv_import of every request's whole history, each timed
alone (GB/s and the fraction of the measured HBM bandwidth).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "paged-attn decode KV GB/s (% of HBM peak); mixed-batch attn tokens/s, % roofline"
DEFAULT_WORKLOAD = "mixed_qwen25_1p5b_t8192"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 1 << 30


# ---------------------------------------------------------------------------
# accounting
# ---------------------------------------------------------------------------

def step_bytes(lay: W.Layout) -> dict:
    """Algorithmic bytes of one step: every distinct KV byte the attention must
    read once, q read, out written, the scatter's read of k/v and write of the
    cache rows, and the block-table entries and lengths read."""
    T, Hq, Hkv, D = lay.num_tokens, lay.num_q_heads, lay.num_kv_heads, lay.head_dim
    kv = lay.kv_bytes_read()
    qo = 2 * T * Hq * D * 2
    scatter = 2 * (2 * T * Hkv * D * 2)
    used_blocks = int(sum(-(-int(n) // 16) for n in lay.seq_lens))
    meta = used_blocks * 4 + lay.num_seqs * 8 + T * 8
    return {"kv": kv, "qo": qo, "scatter": scatter, "meta": meta, "total": kv + qo + scatter + meta}


def decode_prefill_split(lay: W.Layout, info: dict):
    """Algorithmic work of the two kernels, from the plan: the decode
    kernel's KV bytes (the keys its rows attend: all of a row's keys, or
    those after a shared prefix the prefill kernel attends; K and V of one
    kv head per key, no padding of a row's last block) + q/out of its rows,
    and the prefill kernel's flops (4 D per (query, visible key) pair and
    query head, shared-prefix pairs included)."""
    Hq, D = lay.num_q_heads, lay.head_dim
    dec = lay.q_lens <= 16
    dec_tokens = int(lay.q_lens[dec].sum())
    kv_dec = int(info["decode_kv_keys"]) * D * 2 * 2
    flops = 4 * D * Hq * int(info["prefill_causal_pairs"])
    return {"decode_bytes": kv_dec + 2 * dec_tokens * Hq * D * 2, "prefill_flops": flops}


def is_decode_workload(lay: W.Layout) -> bool:
    return bool(np.all(lay.q_lens <= 1))


def dims_for(pa, lay):
    return pa.Dims(lay.num_tokens, lay.num_seqs, lay.num_q_heads, lay.num_kv_heads,
                   lay.head_dim, lay.num_blocks, lay.max_blocks_per_seq, 16)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(names) -> str:
    h = hashlib.sha1()
    for n in names:
        with open(os.path.join(ROOT, "paged_kv_attention_token_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def profiled_traffic(kernel: str, workload: str, src_hash: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "counters.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload)
    if not e or e.get("source_hash") != src_hash:
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock and throttle reasons sampled every ~2 ms through NVML in a
    background thread while the timed region runs."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device: torch.device):
        self.device = device
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self._nvml = None
        self._h = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        self._nvml = pynvml
        props = torch.cuda.get_device_properties(self.device)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
            except Exception:
                pass
        try:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def start(self):
        import threading
        try:
            self._h = self._handle()
            nv = self._nvml
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
        except Exception:
            self._h = None
            return
        self._stop = threading.Event()

        def loop():
            nv = self._nvml
            while not self._stop.is_set():
                try:
                    self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                    self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    pass
                time.sleep(0.002)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=5)
        if not self.samples:
            return None
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(names), "source": "nvml"}


# ---------------------------------------------------------------------------
# CPU oracle (reported baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample_seqs(lay: W.Layout, budget_macs: float, seed: int = 0):
    """Segments whose oracle cost fits the budget (all of them if it does)."""
    cost = []
    for L, n in zip(lay.q_lens.astype(np.int64), lay.seq_lens.astype(np.int64)):
        keys = int(L * (n - L) + L * (L + 1) // 2)
        cost.append(2 * keys * lay.num_q_heads * lay.head_dim)
    cost = np.array(cost, dtype=np.float64)
    if cost.sum() <= budget_macs:
        return list(range(lay.num_seqs)), cost.sum()
    rng = np.random.default_rng(seed)
    order = rng.permutation(lay.num_seqs)
    pick, acc = [], 0.0
    for i in order:
        if acc + cost[i] > budget_macs and pick:
            continue
        pick.append(int(i))
        acc += cost[i]
    return sorted(pick), acc


def time_oracle(batch: W.Batch, seconds: float, budget_macs: float):
    """Run the oracle (scatter + attention) on a bounded sample of the batch
    until `seconds` have passed; returns per-run seconds and what was run."""
    import oracle as O
    lay = batch.layout
    seqs, _ = oracle_sample_seqs(lay, budget_macs)
    hs = W.host_subset(batch, seqs)
    sub = W.Layout(lay.name, lay.num_q_heads, lay.num_kv_heads, lay.head_dim, lay.num_blocks,
                   lay.q_lens[seqs], lay.seq_lens[seqs], lay.block_tables[seqs], lay.poison_block,
                   lay.shared_prefix_blocks)
    threads = O.default_threads()
    runs = []
    t_end = time.perf_counter() + seconds
    while True:
        kc, vc = hs.k_cache.copy(), hs.v_cache.copy()
        t0 = time.perf_counter()
        O.reshape_and_cache(hs.k, hs.v, hs.slot_mapping, kc, vc)
        O.attention_varlen(hs.q, kc, vc, hs.block_tables, hs.cu_seqlens_q, hs.seq_lens,
                           batch.scale, threads=threads)
        runs.append(time.perf_counter() - t0)
        if time.perf_counter() > t_end:
            break
    units = {"bytes": step_bytes(sub)["total"] if len(seqs) else 0, "tokens": int(lay.q_lens[seqs].sum()),
             "seqs": len(seqs)}
    return runs, units, threads


def baseline_value(decode: bool, units: dict, sec: float) -> float:
    return units["bytes"] / sec / 1e9 if decode else units["tokens"] / sec


# ---------------------------------------------------------------------------
# the reference arm: the CPU oracle, as it stands
# ---------------------------------------------------------------------------

def max_over_ranks(value: float, dist, device) -> float:
    """The job's figure for a per-rank time: the max over ranks (each rank's
    own value when there is one rank)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(workload: str, rank: int) -> int:
    """Seed of a rank's batch: every rank draws its own batch of the same shape."""
    return W.WORKLOADS[workload][1] + 7919 * rank


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    lay = W.layout(args.workload)
    decode = is_decode_workload(lay)
    # inputs are drawn on the GPU when there is one (faster for big pools);
    # only the oracle's host run is timed
    batch = W.make_batch(lay, device="cuda" if torch.cuda.is_available() else "cpu")
    per_step = []
    budget = 2.0e9
    runs_all = []
    units = None
    threads = 1
    for i in range(args.warmup + args.steps):
        runs, units, threads = time_oracle(batch, 0.0, budget)
        if i >= args.warmup:
            runs_all.extend(runs)
    sec = statistics.mean(runs_all)
    value = baseline_value(decode, units, sec)
    unit = "GB/s" if decode else "tokens/s"
    sample = (f"{units['seqs']} of {lay.num_seqs} segments ({units['tokens']} query tokens), "
              "oracle scatter + attention per step")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": args.workload, "shape": lay.description},
           "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import paged_kv_attention_token_b200 as pa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    pa.load_library()

    lay = W.layout(args.workload, seed=rank_seed(args.workload, rank))
    decode = is_decode_workload(lay)
    batch = W.make_batch(lay, device=dev)
    acct = step_bytes(lay)
    bt, cu, sl, slots = batch.device_ints(dev)
    h_cu, h_sl = lay.cu_seqlens_q, lay.seq_lens
    h_bt = lay.block_tables  # host copy: lets the planner find shared prefixes
    kc, vc = batch.k_cache.clone(), batch.v_cache.clone()
    out = torch.empty_like(batch.q)
    dims = dims_for(pa, lay)
    plan0 = pa.Plan(h_cu, h_sl, dims, device=local, block_tables=h_bt)
    info = plan0.info()
    ws = pa.workspace_for(plan0, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_read = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.zeros((), dtype=torch.float32, device=dev)

    def flush_l2(v):
        """Evict L2: write one buffer larger than L2, then read another (clean lines)."""
        flush.fill_(v)
        torch.sum(flush_read, dim=0, out=flush_sink)
    stream = torch.cuda.current_stream(dev)
    # the scatter, then the kernels the attention call launches (plan info);
    # the fused call stages the prefill segments' keys in its scatter launch
    launches_per_step = (1 if lay.num_tokens else 0) + info["attention_launches"]  # scatter + attention
    if not args.two_calls and lay.num_tokens and info["num_staged_kv_tiles"] > 0:
        launches_per_step -= 1

    # two plans rebuilt in turn, as an engine keeps them across steps
    plan_pool = [pa.Plan(h_cu, h_sl, dims, device=local, block_tables=h_bt), pa.Plan(h_cu, h_sl, dims, device=local, block_tables=h_bt)]
    step_no = [0]

    def one_step(trace=None, ev=None):
        flush_l2(1)
        plan = plan_pool[step_no[0] % 2].rebuild(h_cu, h_sl, dims, h_bt)
        step_no[0] += 1
        if ev is not None:
            ev[0].record(stream)
        if trace is not None or args.two_calls:  # the traced entry point is the two-call one
            pa.reshape_and_cache(batch.k, batch.v, slots, kc, vc, stream=stream)
            pa.attention_varlen(batch.q, kc, vc, bt, cu, sl, batch.scale, out, plan, ws,
                                stream=stream, trace=trace)
        else:
            pa.reshape_and_attention(batch.k, batch.v, slots, batch.q, kc, vc, bt, cu, sl, batch.scale, out,
                                     plan, ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        return plan

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize(dev)

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    plans = []
    wall0 = time.perf_counter()
    for i in range(args.steps):
        plans.append(one_step(None, evs[i]))
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - wall0
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = sum(step_ms)
    max_total_ms = max_over_ranks(total_ms, dist, dev)
    ms_per_step = max_total_ms / args.steps

    if decode:
        unit = "GB/s"
        value = world * acct["total"] * args.steps / (max_total_ms * 1e-3) / 1e9
    else:
        unit = "tokens/s"
        value = world * lay.num_tokens * args.steps / (max_total_ms * 1e-3)

    # Roofline of the dominant kernel (the split-KV decode kernel).  Event
    # records cost GPU time, so the kernel is timed in a second pass of K
    # steps, identical to the timed ones, with events around that kernel only
    # (and, in a third pass, around the other stages of the call).
    peaks, peak_kind = load_peaks()

    def copy_at_size(nbytes):
        """A device copy moving the same bytes (half read, half written), timed
        like the kernels (L2 flushed first, events on the stream): what one
        launch of a plain copy reaches at this size, where fixed launch and
        ramp costs weigh against the HBM rate of the peak (a large copy)."""
        half = max(16, (nbytes // 2) // 16 * 16)
        src = torch.ones(half, dtype=torch.uint8, device=dev)
        dst = torch.empty(half, dtype=torch.uint8, device=dev)
        times = []
        for i in range(max(3, args.warmup) + max(5, args.steps)):
            flush_l2(5)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            dst.copy_(src)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i >= max(3, args.warmup):
                times.append(e0.elapsed_time(e1))
        ms = statistics.mean(times)
        gbs = 2 * half / (ms * 1e-3) / 1e9
        del src, dst
        return {"ms": ms, "gbs": gbs, "frac_of_peak": gbs / peaks["hbm_gbs"],
                "how": "torch copy_ of the same bytes (half read, half written), L2 flushed, events, mean"}

    def traced_pass(stages):
        trs = [pa.Trace(stages=stages) for _ in range(args.steps)]
        for i in range(args.steps):
            one_step(trs[i], None)
        torch.cuda.synchronize(dev)
        return [t.elapsed_ms() for t in trs]

    dec_ms = statistics.mean(s["decode"] for s in traced_pass(("decode",)))
    other = traced_pass(("plan_wait", "combine", "staging", "prefill"))
    comb_ms = statistics.mean(s["combine"] for s in other)
    wait_ms = statistics.mean(s["plan_wait"] for s in other)
    prefill_ms = statistics.mean(s["prefill"] for s in other)  # the prefill kernel alone
    staging_ms = statistics.mean(s["staging"] for s in other)
    split = decode_prefill_split(lay, info)
    roofline_decode = roofline_prefill = None
    dec_bytes = split["decode_bytes"]
    if dec_bytes and dec_ms > 0:
        achieved = dec_bytes / (dec_ms * 1e-3) / 1e9
        src_hash = kernel_source_hash(["decode.cu", "common.cuh", "kernels.h", "plan.h"])
        roofline_decode = {"bound": "hbm", "kernel": "decode_kernel", "achieved": achieved,
                           "peak": peaks["hbm_gbs"], "peak_kind": peak_kind, "unit": "GB/s",
                           "frac": achieved / peaks["hbm_gbs"],
                           "traffic": profiled_traffic("decode_kernel", args.workload, src_hash),
                           "algorithmic_bytes": dec_bytes, "ms": dec_ms, "source_hash": src_hash,
                           "copy_at_size": copy_at_size(dec_bytes)}
        roofline_decode["copy_at_size"]["decode_frac_of_it"] = achieved / roofline_decode["copy_at_size"]["gbs"]
    # when the plan runs the prefill kernel beside the decode kernel, it has
    # overlap_sms of the SMs: its peak is that share of the GPU's
    side_by_side = bool(info["num_decode_units"] and info["num_prefill_tiles"] and info["overlap_sms"] > 0)
    sm_share = info["overlap_sms"] / info["num_sms"] if side_by_side else 1.0
    # head_dim 128 with an even group runs on the pair kernel (2-SM MMAs)
    prefill_kernel = "prefill_pair_kernel" if info["prefill_pair"] else "prefill_kernel"
    if split["prefill_flops"] and prefill_ms > 0:
        tflops = split["prefill_flops"] / (prefill_ms * 1e-3) / 1e12
        pre_hash = kernel_source_hash(["prefill.cu", "common.cuh", "kernels.h", "plan.h"])
        roofline_prefill = {"bound": "tensor", "kernel": prefill_kernel, "achieved": tflops,
                            "peak": peaks["bf16_tflops"] * sm_share,
                            "peak_kind": peak_kind + " (burst bf16" +
                            (f", x {info['overlap_sms']}/{info['num_sms']} SMs beside the decode kernel)"
                             if side_by_side else ")"),
                            "unit": "TFLOP/s", "frac": tflops / (peaks["bf16_tflops"] * sm_share),
                            "traffic": profiled_traffic(prefill_kernel, args.workload, pre_hash),
                            "algorithmic_flops": split["prefill_flops"], "ms": prefill_ms,
                            "source_hash": pre_hash}
        if not side_by_side and info["num_staged_kv_tiles"] > 0:
            # the K/V staging kernel that precedes it (one extra read and write
            # of the prefill segments' keys), timed in the same traced pass
            roofline_prefill["staging_ms"] = staging_ms
            roofline_prefill["frac_with_staging"] = split["prefill_flops"] / ((prefill_ms + staging_ms) * 1e-3) / 1e12 / \
                (peaks["bf16_tflops"] * sm_share)
    # "roofline" is the dominant kernel's: the one with the longer device time
    # (side by side, both span about the step; the decode kernel, which
    # bounds the step through HBM, is reported)
    cands = [r for r in (roofline_decode, roofline_prefill) if r is not None]
    if side_by_side and roofline_decode is not None:
        roofline = roofline_decode
    else:
        roofline = max(cands, key=lambda r: r["ms"]) if cands else None
    # whole step against its roofline: the slower of the tensor-bound prefill
    # time and the HBM-bound time of every algorithmic byte of the step
    t_roof = max(split["prefill_flops"] / (peaks["bf16_tflops"] * 1e12),
                 acct["total"] / (peaks["hbm_gbs"] * 1e9))
    step_roofline = {"t_roofline_ms": t_roof * 1e3, "t_measured_ms": ms_per_step,
                     "frac": t_roof * 1e3 / ms_per_step}

    # host cost of a plan build (and its table upload), on an idle plan
    torch.cuda.synchronize(dev)
    plan_build_us = []
    for i in range(max(20, args.steps)):
        t0 = time.perf_counter()
        plan_pool[i % 2].rebuild(h_cu, h_sl, dims, h_bt)
        plan_build_us.append((time.perf_counter() - t0) * 1e6)

    # the scatter kernel alone: back-to-back launches on distinct copies of
    # the step's K/V, each writing its own slots in blocks no request owns,
    # after an L2 flush
    scatter = None
    T, Hkv, D = lay.num_tokens, lay.num_kv_heads, lay.head_dim
    free = np.setdiff1d(np.arange(lay.num_blocks), np.append(lay.used_blocks(), lay.poison_block))
    need = -(-T // 16)
    nsets = min(8, len(free) // need) if T else 0
    if nsets:
        tok = np.arange(T, dtype=np.int64)
        sc_slots = [torch.from_numpy(free[s * need:(s + 1) * need].astype(np.int64)[tok // 16] * 16 + tok % 16).to(dev)
                    for s in range(nsets)]
        sc_k = [batch.k.clone() for _ in range(nsets)]
        sc_v = [batch.v.clone() for _ in range(nsets)]
        sc_ms = []
        for i in range(args.warmup + args.steps):
            flush_l2(4)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for s_ in range(nsets):
                pa.reshape_and_cache(sc_k[s_], sc_v[s_], sc_slots[s_], kc, vc, stream=stream)
            e1.record(stream)
            if i >= args.warmup:
                sc_ms.append((e0, e1))
        torch.cuda.synchronize(dev)
        per_launch_ms = statistics.mean(a.elapsed_time(b) for a, b in sc_ms) / nsets
        sc_bytes = 2 * (2 * T * Hkv * D * 2) + T * 8   # k, v read; cache rows written; slots read
        sc_gbs = sc_bytes / (per_launch_ms * 1e-3) / 1e9
        sc_hash = kernel_source_hash(["scatter.cu", "scatter.cuh", "common.cuh", "kernels.h", "plan.h"])
        scatter = {"bound": "hbm", "kernel": "reshape_and_cache_kernel", "achieved": sc_gbs,
                   "peak": peaks["hbm_gbs"], "peak_kind": peak_kind, "unit": "GB/s",
                   "frac": sc_gbs / peaks["hbm_gbs"],
                   "traffic": profiled_traffic("reshape_and_cache_kernel", args.workload, sc_hash),
                   "algorithmic_bytes": sc_bytes, "ms": per_launch_ms, "source_hash": sc_hash,
                   "how": f"{nsets} back-to-back launches on distinct inputs and slots after an L2 flush, "
                          "events around all of them"}
        del sc_k, sc_v, sc_slots

    # e2e: public API with host buffers; H2D of the step's inputs, D2H of out
    e2e = None
    if not args.no_e2e:
        # the step's host inputs live in one page-locked buffer (each at a
        # 256-byte offset) and cross to the device in one copy
        srcs = (("q", batch.q), ("k", batch.k), ("v", batch.v), ("slots", slots),
                ("bt", bt), ("cu", cu), ("sl", sl))
        offs, nbytes = {}, 0
        for n, x in srcs:
            offs[n] = nbytes
            nbytes += -(-x.numel() * x.element_size() // 256) * 256
        h_stage = torch.zeros(nbytes, dtype=torch.uint8, pin_memory=True)
        d_stage = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        dev_in = {}
        for n, x in srcs:
            nb = x.numel() * x.element_size()
            h_stage[offs[n]:offs[n] + nb].copy_(x.detach().contiguous().view(-1).view(torch.uint8).cpu())
            dev_in[n] = d_stage[offs[n]:offs[n] + nb].view(x.dtype).view(x.shape)
        out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        # inputs, plus the plan tables each step's build uploads
        h2d = nbytes + info["table_bytes"]
        d2h = out_host.numel() * out_host.element_size()
        e_ms, e_wall_ms, e_ev_ms = [], [], []
        for i in range(args.warmup + args.steps):
            flush_l2(2)
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0 = time.perf_counter()
            e0.record(stream)
            d_stage.copy_(h_stage, non_blocking=True)
            plan = plan_pool[i % 2].rebuild(h_cu, h_sl, dims, h_bt)
            if args.two_calls:
                pa.reshape_and_cache(dev_in["k"], dev_in["v"], dev_in["slots"], kc, vc, stream=stream)
                pa.attention_varlen(dev_in["q"], kc, vc, dev_in["bt"], dev_in["cu"], dev_in["sl"],
                                    batch.scale, out, plan, ws, stream=stream)
            else:
                pa.reshape_and_attention(dev_in["k"], dev_in["v"], dev_in["slots"], dev_in["q"], kc, vc,
                                         dev_in["bt"], dev_in["cu"], dev_in["sl"], batch.scale, out, plan, ws,
                                         stream=stream)
            out_host.copy_(out, non_blocking=True)
            e1.record(stream)
            e1.synchronize()
            wall_ms = (time.perf_counter() - t0) * 1e3
            if i >= args.warmup:
                ev_ms = e0.elapsed_time(e1)
                e_wall_ms.append(wall_ms)
                e_ev_ms.append(ev_ms)
                e_ms.append(max(wall_ms, ev_ms))
        e_total = max_over_ranks(sum(e_ms), dist, dev)
        e_val = (world * acct["total"] * args.steps / (e_total * 1e-3) / 1e9) if decode else \
            (world * lay.num_tokens * args.steps / (e_total * 1e-3))
        e2e = {"value": e_val, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_total / args.steps,
               "host_ms_per_step": statistics.mean(e_wall_ms), "events_ms_per_step": statistics.mean(e_ev_ms),
               "includes": "plan build and table upload, H2D of inputs, scatter + attention, D2H of out"}

    # KV export / import of every request's whole history (the local half of
    # moving a request's KV between instances), each call timed alone with
    # events after an L2 flush; algorithmic bytes: K and V of every token,
    # read once and written once
    kv_transfer = None
    if not args.no_kv_transfer:
        cu_t = torch.from_numpy(np.concatenate([[0], np.cumsum(lay.seq_lens)]).astype(np.int32)).to(dev)
        n_tok = int(lay.seq_lens.sum())
        k_buf = torch.empty((n_tok, lay.num_kv_heads, lay.head_dim), dtype=torch.bfloat16, device=dev)
        v_buf = torch.empty_like(k_buf)
        xfer_bytes = 2 * 2 * k_buf.numel() * k_buf.element_size()

        def time_calls(fn):
            ms = []
            for i in range(args.warmup + args.steps):
                flush_l2(3)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                if i >= args.warmup:
                    ms.append((e0, e1))
            torch.cuda.synchronize(dev)
            return statistics.mean(a.elapsed_time(b) for a, b in ms)

        exp_ms = time_calls(lambda: pa.kv_export(kc, vc, bt, cu_t, k_buf, v_buf, stream=stream))
        # (importing the exported history back writes every slot the same value)
        imp_ms = time_calls(lambda: pa.kv_import(k_buf, v_buf, bt, cu_t, kc, vc, stream=stream))
        exp_gbs, imp_gbs = xfer_bytes / (exp_ms * 1e-3) / 1e9, xfer_bytes / (imp_ms * 1e-3) / 1e9
        kv_transfer = {"tokens": n_tok, "bytes_per_call": xfer_bytes,
                       "export": {"ms": exp_ms, "GB/s": exp_gbs, "frac": exp_gbs / peaks["hbm_gbs"]},
                       "import": {"ms": imp_ms, "GB/s": imp_gbs, "frac": imp_gbs / peaks["hbm_gbs"]},
                       "peak_kind": peak_kind}
        del k_buf, v_buf

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host_batch = batch
        runs, units, threads = time_oracle(host_batch, args.cpu_seconds, 2.0e9)
        sec = statistics.mean(runs)
        cpu = {"value": baseline_value(decode, units, sec), "unit": unit, "cores": threads,
               "kind": "oracle",
               "sample": f"{units['seqs']} of {lay.num_seqs} segments ({units['tokens']} query tokens), "
                         f"oracle scatter + attention, {len(runs)} runs, mean {sec:.3f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "shape": lay.description,
                       "bytes_per_step": acct["total"], "kv_bytes_per_step": acct["kv"],
                       "kv_bytes_logical_per_step": lay.kv_bytes_logical(),
                       "tokens_per_step": lay.num_tokens,
                       "l2": "flushed before every timed step (1 GiB write, then 1 GiB read; outside the events)",
                       "plan_us_host": statistics.median(plan_build_us),
                       "plan_us_host_note": "pa_plan_build on an idle plan (host partition + table upload), "
                                            "median",
                       "step_api": ("pa_reshape_and_cache + pa_attention_varlen" if args.two_calls
                                    else "pa_reshape_and_attention"),
                       "stages_ms": {"plan_wait": wait_ms, "decode": dec_ms, "combine": comb_ms,
                                     "staging": staging_ms if not side_by_side else None,
                                     "prefill": prefill_ms,
                                     "scatter": scatter["ms"] if scatter else None,
                                     "note": "separate traced passes; event records add GPU time"},
                       "parallelism": f"replicas x{world} (weak: one batch per GPU)",
                       "wall_s_timed_region": wall},
            "roofline": roofline,
            "roofline_decode": roofline_decode,
            "roofline_prefill": roofline_prefill,
            "roofline_scatter": scatter,
            "kv_transfer": kv_transfer,
            "step_roofline": step_roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--two-calls", action="store_true",
                    help="step through pa_reshape_and_cache + pa_attention_varlen instead of the fused call")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-kv-transfer", action="store_true", help="skip timing pa_kv_export / pa_kv_import")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
