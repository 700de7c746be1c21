#!/usr/bin/env python
"""Benchmark of the paged decode step: reshape_and_cache (+ copy_blocks when the
step has copy-on-write pairs) + paged decode attention, on synthetic workloads.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|ID]
                    [--impl ours|reference] [--batch B] [--e2e-steps E]
                    [--shared-prefix | --prefill | --swap]

One step = one pass of the whole hot path over one batch: the step's
copy_blocks, then reshape_and_cache of the new tokens, then decode attention
of every sequence's new query over its paged context (inputs resident in HBM).
The headline workload is the Llama-2-7B-shaped fp16 batch (64 sequences, 32
heads x 128, contexts U[128, 2048], 16-token blocks, pool of 8192 blocks).
With no --workload, the same JSON line also carries (one GPU only):
  per_workload  the same step and fields on every other decode workload at full
                size (Llama-3-70B-shaped GQA, long context, shared-prefix
                sampling with plain and with shared-prefix decode, FP8 pools),
                with the CUDA-core kernel timed beside the tensor-core one on
                the GQA shapes (kernel_ab);
  warm_l2       decode of a batch that fits the L2, with and without a flush;
  paging_cost   decode on contiguous block tables against shuffled ones;
  prefill       paged chunked prefill (TFLOP/s), with the multi-query kernel beside it;
  swap_blocks   blocks swapped out to page-locked host memory and back.

Under torchrun (N > 1) every rank runs its own replica of the workload on its
own GPU (weak scaling; the path has no exchange step, so there is no
collective on the data path). Timing is on the device with CUDA events, max
over ranks. Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only other implementation
there is) on a bounded sample of the same workload, on rank 0.

--swap measures swap_blocks instead (preemption by swapping): whole blocks of
the Llama-2-7B-shaped pool moved device -> page-locked host and back, against
a plain cudaMemcpyAsync of the same bytes timed in the same run.

--shared-prefix (with --workload 5) runs the step's decode with
pa_decode_shared_prefix: each group's shared blocks are read once per group.

--prefill measures paged chunked prefill in TFLOP/s: 8 sequences with
U[0, 2048] cached tokens each take a 512-token chunk (Llama-3-70B-shaped, bf16).
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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_418_b200 import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
METRIC = "paged decode attention KV GB/s"
HEADLINE = "llama2-7b-fp16"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default=None,
                   help="measure this workload alone (default: the Llama-2-7B-shaped batch as "
                        "the headline, plus every other decode workload in per_workload)")
    p.add_argument("--no-suite", action="store_true",
                   help="default run: measure the headline workload only")
    p.add_argument("--skip-prefill", action="store_true",
                   help="default run: leave out the prefill measurement")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=None)
    p.add_argument("--batch", type=int, default=None,
                   help="fewer sequences of the same workload (profiling captures)")
    p.add_argument("--shared-prefix", action="store_true",
                   help="decode the shared-prefix workload with pa_decode_shared_prefix")
    p.add_argument("--prefill", action="store_true",
                   help="measure paged prefill attention (causal chunks) instead of decode")
    p.add_argument("--swap", action="store_true",
                   help="measure swap_blocks (device <-> pinned host) instead of the decode step")
    return p.parse_args()


def workload_id(x) -> int:
    return int(x) if str(x).isdigit() else W.WORKLOAD_IDS[x]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def config_of(w: W.Workload, world: int, l2_note: str):
    extra = ({"k_cache": W.DTYPE_NAMES[w.kv_dtype], "v_cache": W.DTYPE_NAMES[w.v_dtype],
              "k_scale": w.k_scale, "v_scale": w.v_scale} if w.fp8 else {})
    return {**extra,
        "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": w.D,
        "block_size": w.block_size, "num_blocks": w.num_blocks, "dtype": W.DTYPE_NAMES[w.dtype],
        "context_lens": {"sum": int(w.context_lens.sum()), "mean": float(w.context_lens.mean()),
                         "max": int(w.context_lens.max())},
        "new_tokens": int(len(w.slot_mapping)), "cow_pairs": int(len(w.block_mapping)),
        "partition_size": w.partition_size or "auto",
        "kv_bytes_per_step": w.kv_bytes(), "seed": w.seed,
        "parallelism": f"replicas x{world} (no collective on the data path)",
        "l2": l2_note,
    }


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_smi_id(local_rank: int) -> str:
    """The id nvidia-smi knows this process's GPU by (UUID when torch exposes it)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(local_rank).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            return vis.split(",")[local_rank].strip()
        return str(local_rank)


# ----------------------------------------------------------------------------
# reference arm / CPU baseline: the fp64 oracle on a bounded sample
# ----------------------------------------------------------------------------
def oracle_sample_rows(w: W.Workload, budget_s: float, rng_seed: int = 0):
    """Pick (b, hq) rows, longest-first interleaved with random, until the
    estimated oracle time reaches the budget (calibrated on a few rows)."""
    import oracle
    rng = np.random.default_rng(rng_seed)
    all_rows = np.array([(b, h) for b in range(w.B) for h in range(w.Hq)], dtype=np.int32)
    order = rng.permutation(len(all_rows))
    probe = all_rows[order[:8]]
    t = time.perf_counter()
    oracle_decode_rows(w, w.k_cache, w.v_cache, probe)
    dt = max(time.perf_counter() - t, 1e-4)
    tok = float(w.context_lens[probe[:, 0]].sum())
    per_token = dt / tok
    budget_tokens = budget_s / per_token
    chosen, acc = [], 0.0
    for i in order:
        if acc >= budget_tokens:
            break
        chosen.append(all_rows[i])
        acc += float(w.context_lens[all_rows[i][0]])
    return np.array(chosen, dtype=np.int32)


def oracle_cache_ops(w: W.Workload, kc, vc):
    """The step's copy_blocks and reshape_and_cache on host pools (oracle)."""
    import oracle
    if len(w.block_mapping):
        oracle.copy_blocks(kc, vc, w.block_mapping, w.kv_dtype)
    if w.mixed:
        oracle.reshape_and_cache_mixed(kc, vc, w.new_key, w.new_value, w.dtype, w.kv_dtype,
                                       w.v_dtype, w.k_scale, w.v_scale, w.slot_mapping)
    elif w.fp8:
        oracle.reshape_and_cache_fp8(kc, vc, w.new_key, w.new_value, w.dtype, w.k_scale,
                                     w.v_scale, w.slot_mapping)
    else:
        oracle.reshape_and_cache(kc, vc, w.new_key, w.new_value, w.slot_mapping, w.dtype)


def oracle_decode_rows(w: W.Workload, kc, vc, rows):
    import oracle
    if w.mixed:
        return oracle.decode_mixed(w.q, w.dtype, kc, w.kv_dtype, w.k_scale, vc, w.v_dtype,
                                   w.v_scale, w.block_tables, w.context_lens, w.scale, rows=rows)
    if w.fp8:
        return oracle.decode_kv(w.q, w.dtype, kc, vc, oracle.FP8, w.k_scale, w.v_scale,
                                w.block_tables, w.context_lens, w.scale, rows=rows)
    return oracle.decode(w.q, kc, vc, w.dtype, w.block_tables, w.context_lens, w.scale,
                         rows=rows)


def run_oracle(w: W.Workload, rows: np.ndarray, reps: int = 1):
    """Time the oracle's share of a step: the step's cache ops on host pools and
    decode of the sampled rows. Returns (seconds, kv_bytes_equivalent)."""
    import oracle
    kc, vc = w.k_cache, w.v_cache                       # in place; the step is idempotent
    total = 0.0
    for _ in range(reps):
        t = time.perf_counter()
        oracle_cache_ops(w, kc, vc)
        oracle_decode_rows(w, kc, vc, rows)
        total += time.perf_counter() - t
    frac = float(w.context_lens[rows[:, 0]].sum()) / (w.Hq * float(w.context_lens.sum()))
    return total, w.kv_bytes() * frac * reps


def reference_arm(args, w: W.Workload, rank: int, world: int):
    if rank != 0:
        return None
    import oracle
    cores = oracle.max_threads()
    steps = max(1, args.steps)
    # each step a bounded sample: about 2 minutes of oracle time for the whole run
    rows = oracle_sample_rows(w, budget_s=max(0.05, min(3.0, 120.0 / steps)))
    for _ in range(max(0, min(args.warmup, 1))):
        run_oracle(w, rows[:4])
    secs, byts = run_oracle(w, rows, reps=steps)
    value = byts / secs / 1e9
    sample = (f"{len(rows)} of {w.B * w.Hq} (sequence, query head) rows per step "
              f"({100.0 * len(rows) / (w.B * w.Hq):.1f}%), plus the step's full "
              f"reshape_and_cache/copy_blocks; value scaled by the rows' share of KV bytes")
    # the same oracle on one core: decode of a ~3 s sample of rows
    rows1 = oracle_sample_rows(w, budget_s=3.0 / max(1, cores), rng_seed=1)
    t = time.perf_counter()
    oracle.decode_mixed(w.q, w.dtype, w.k_cache, w.kv_dtype, w.k_scale, w.v_cache, w.v_dtype,
                        w.v_scale, w.block_tables, w.context_lens, w.scale, rows=rows1,
                        n_threads=1)
    secs1 = time.perf_counter() - t
    oracle.decode_mixed(w.q, w.dtype, w.k_cache, w.kv_dtype, w.k_scale, w.v_cache, w.v_dtype,
                        w.v_scale, w.block_tables, w.context_lens, w.scale, rows=rows1[:1],
                        n_threads=cores)
    frac1 = float(w.context_lens[rows1[:, 0]].sum()) / (w.Hq * float(w.context_lens.sum()))
    one_core = {"value": round(w.kv_bytes() * frac1 / secs1 / 1e9, 4), "unit": "GB/s",
                "sample": f"decode of {len(rows1)} rows on 1 thread, {secs1:.1f} s"}
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, 1, "host memory"),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample, "one_core": one_core},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return line


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
KERNEL_SOURCES = {
    "cuda-core": ["decode_simt.cu"],
    "tcgen05": ["decode_tc.cu", "tc_ptx.cuh", "decode_simt.cu"],  # merge kernel: decode_simt.cu
    "shared-prefix": ["decode_prefix_tc.cu", "decode_tc.cu", "tc_ptx.cuh", "decode_simt.cu"],
    "prefill": ["prefill_tc.cu", "tc_ptx.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of what a kernel path's device code is built from: its kernel files,
    the device helpers, and the launch-argument struct (declarations of other
    entry points do not change the kernels, so they are left out)."""
    import re
    csrc = os.path.join(ROOT, "paged_kv_cache_418_b200", "csrc")
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel] + ["pa_common.cuh"]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    internal = open(os.path.join(csrc, "pa_internal.h")).read()
    struct = "PrefillLaunch" if kernel == "prefill" else "DecodeArgs"
    m = re.search(r"struct " + struct + r" \{.*?\};", internal, re.S)
    h.update((m.group(0) if m else internal).encode())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, workload: str):
    """DRAM bytes per launch of a workload's kernel from a committed ncu summary,
    or None when there is none for it or the kernel's sources changed since."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(workload)
    if not rec or rec.get("kernel") != kernel or rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


class Decoder:
    """One workload's device tensors and its decode step through the C ABI."""

    def __init__(self, w: W.Workload, dev, cascade: bool = False):
        import torch
        from paged_kv_cache_418_b200 import ops
        self.w, self.dev, self.cascade, self.ops = w, dev, cascade, ops
        self.t = W.to_torch(w, dev)
        self.stream = torch.cuda.current_stream(dev)
        self.out = torch.empty((w.B, w.Hq, w.D), dtype=self.t["torch_dtype"], device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        t = self.t
        if cascade:
            if "prefix_blocks" not in w.meta:
                raise SystemExit("--shared-prefix needs a workload with groups "
                                 "(shared-prefix-sampling-bf16)")
            ng, nc, pb = w.meta["groups"], w.meta["children"], w.meta["prefix_blocks"]
            self.group = (torch.full((w.B,), pb, dtype=torch.int32, device=dev),
                          torch.arange(0, ng * nc + 1, nc, dtype=torch.int32, device=dev),
                          torch.arange(ng * nc, dtype=torch.int32, device=dev), nc, pb)
            self.ws = ops.shared_prefix_workspace_for(t["q"], t["k_cache"], w.max_context_len, pb,
                                                      w.partition_size)
        else:
            self.ws = ops.workspace_for(t["q"], t["k_cache"], w.max_context_len, w.partition_size)

    def plan(self):
        w = self.w
        return self.ops.pa_decode_plan(W.FP8 if w.fp8 else w.kv_dtype, w.B, w.Hq, w.Hkv, w.D,
                                       w.block_size, w.max_context_len, w.partition_size)

    def cache_ops(self):
        w, t, ops = self.w, self.t, self.ops
        if len(w.block_mapping):
            ops.pa_copy_blocks(t["k_cache"], t["v_cache"], t["block_mapping"], self.err, self.stream)
        if w.mixed:
            ops.pa_reshape_and_cache_kv(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                        w.k_scale, w.v_scale, t["slot_mapping"], self.err,
                                        self.stream)
        elif w.fp8:
            ops.pa_reshape_and_cache_fp8(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                         w.k_scale, w.v_scale, t["slot_mapping"], self.err,
                                         self.stream)
        else:
            ops.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                     t["slot_mapping"], self.err, self.stream)

    def decode(self):
        w, t, ops = self.w, self.t, self.ops
        if self.cascade:
            g_shared, g_off, g_mem, nc, pb = self.group
            ops.pa_decode_shared_prefix(self.out, t["q"], t["k_cache"], t["v_cache"],
                                        t["block_tables"], t["context_lens"], g_shared, g_off,
                                        g_mem, nc, pb, w.scale, w.max_context_len,
                                        w.partition_size, self.ws, self.err, self.stream)
        elif w.mixed:
            ops.pa_decode_kv(self.out, t["q"], t["k_cache"], t["v_cache"], w.k_scale, w.v_scale,
                             t["block_tables"], t["context_lens"], w.scale, w.max_context_len,
                             w.partition_size, self.ws, self.err, self.stream)
        elif w.fp8:
            ops.pa_decode_fp8(self.out, t["q"], t["k_cache"], t["v_cache"], w.k_scale, w.v_scale,
                              t["block_tables"], t["context_lens"], w.scale, w.max_context_len,
                              w.partition_size, self.ws, self.err, self.stream)
        else:
            ops.pa_decode(self.out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                          t["context_lens"], w.scale, w.max_context_len, w.partition_size,
                          self.ws, self.err, self.stream)

    def step(self, ev=None):
        """One step: the step's copy-on-write pairs, its new tokens, then decode."""
        self.cache_ops()
        if ev is not None:
            ev[0].record(self.stream)
        self.decode()
        if ev is not None:
            ev[1].record(self.stream)

    def check(self, when: str):
        import torch
        torch.cuda.synchronize(self.dev)
        if int(self.err.item()) != 0:
            raise RuntimeError(f"{self.w.name}: device error flag {int(self.err.item())} {when}")


def time_decode_only(d: Decoder, K: int, flush_buf=None) -> float:
    """Mean event-timed duration (ms) of K back-to-back decode calls (L2 flushed
    before each when flush_buf is given)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    for _ in range(3):
        d.decode()
    for e0, e1 in evs:
        if flush_buf is not None:
            flush_buf.zero_()
        e0.record(d.stream)
        d.decode()
        e1.record(d.stream)
    d.check("while timing decode")
    return sum(a.elapsed_time(b) for a, b in evs) / K


def measure(args, w: W.Workload, rank: int, world: int, local_rank: int, *,
            cascade: bool = False, cuda_core_ab: bool = False):
    """Time the step on one workload: W warm-up steps, K timed steps (barrier and
    synchronize on both sides, max over ranks), then the end-to-end loop through
    the same API with host buffers. Returns rank 0's fields (None elsewhere)."""
    import torch
    import torch.distributed as dist

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    d = Decoder(w, dev, cascade)
    t, stream = d.t, d.stream
    kernel, P, psize = d.plan()
    launches_per_step = (1 if len(w.block_mapping) else 0) + 1 + 1 + (1 if P > 1 or cascade else 0) \
        + (1 if cascade else 0)
    unique = w.unique_kv_bytes()
    flush = unique < 2 * L2_BYTES
    l2_note = ("L2 flushed before every step (workload smaller than 2x L2)" if flush else
               f"inputs larger than L2 (KV {unique / 1e9:.2f} GB distinct > 126 MB)")
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if flush else None

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    for _ in range(args.warmup):
        d.step()
    d.check("during warm-up")

    K = args.steps
    dec_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)] if flush else None
    sampler = ClockSampler(gpu_smi_id(local_rank))
    if rank == 0:
        sampler.start()
    barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(K):
        if flush:
            flush_buf.zero_()
            step_ev[i][0].record(stream)
        d.step(dec_ev[i])
        if flush:
            step_ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop() if rank == 0 else None
    if flush:
        ms = sum(a.elapsed_time(b) for a, b in step_ev)
    else:
        ms = t_start.elapsed_time(t_end)
    dec_ms = sum(a.elapsed_time(b) for a, b in dec_ev) / K
    ms, dec_ms = max_over_ranks([ms, dec_ms], world, dev)
    d.check("during timing")

    # end to end through the public API: the step's inputs staged in one page-locked
    # host buffer and sent with one copy (as an engine stages a step's inputs),
    # the step, and the output read back; the device inputs the step reads are
    # views into the buffer the copy fills
    names = [k for k in ("q", "new_key", "new_value", "slot_mapping", "block_tables",
                         "context_lens", "block_mapping") if k in t]
    offs, total = {}, 0
    for k in names:
        offs[k] = total
        total += (t[k].numel() * t[k].element_size() + 255) // 256 * 256
    host_buf = torch.zeros(max(total, 1), dtype=torch.uint8).pin_memory()
    dev_buf = torch.empty(max(total, 1), dtype=torch.uint8, device=dev)
    for k in names:
        n = t[k].numel() * t[k].element_size()
        if n:
            host_buf[offs[k]:offs[k] + n].copy_(t[k].contiguous().reshape(-1).view(torch.uint8).cpu())
        t[k] = dev_buf[offs[k]:offs[k] + n].view(t[k].dtype).view(t[k].shape)
    out_host = torch.empty(d.out.shape, dtype=d.out.dtype).pin_memory()
    h2d = total
    d2h = d.out.numel() * d.out.element_size()
    Ke = args.e2e_steps or max(1, min(K, 200))
    for _ in range(2):
        dev_buf.copy_(host_buf, non_blocking=True)
        d.step()
        out_host.copy_(d.out, non_blocking=True)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_ms = 0.0
    for i in range(Ke):
        if flush:
            flush_buf.zero_()
        e0.record(stream)
        dev_buf.copy_(host_buf, non_blocking=True)
        d.step()
        out_host.copy_(d.out, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        e_ms += e0.elapsed_time(e1)
    (e_ms,) = max_over_ranks([e_ms], world, dev)
    barrier()

    # the same decode forced onto the CUDA-core kernel (evidence for the tensor-core choice)
    ab = None
    if cuda_core_ab and kernel == 2 and not cascade and rank == 0 and world == 1:
        tc_us = 1e3 * time_decode_only(d, K, flush_buf)
        os.environ["PA_DECODE_KERNEL"] = "simt"
        try:
            cc_us = 1e3 * time_decode_only(d, K, flush_buf)
        finally:
            del os.environ["PA_DECODE_KERNEL"]
        ab = {"decode_us_tcgen05": round(tc_us, 2), "decode_us_cuda_core": round(cc_us, 2),
              "cuda_core_over_tcgen05": round(cc_us / tc_us, 3),
              "how": f"{K} decode calls back to back per kernel, same inputs, same loop"}
    if rank != 0:
        return None

    kv = w.kv_bytes()
    value = job_value(kv, K, world, ms)
    peak, peak_src = peaks()
    kname = {1: "cuda-core", 2: "tcgen05"}[kernel] if not cascade else "shared-prefix"
    # the cascade reads each distinct K/V byte once: its algorithmic bytes are the distinct ones
    alg = unique if cascade else kv
    achieved = alg / (dec_ms / 1e3) / 1e9
    traffic = traffic_record(kname, w.name + (" (pa_decode_shared_prefix)" if cascade else ""))
    e2e_value = job_value(kv, Ke, world, e_ms)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": W.DTYPE_NAMES[w.dtype], "data": "synthetic",
        "config": config_of(w, world, l2_note),
        "pct_of_hbm_peak": round(100.0 * (value / world) / peak, 2),
        "seq_steps_per_s": round(w.B * K * world / (ms / 1e3), 1),
        "decode_us": round(dec_ms * 1e3, 2),
        "decode_plan": {"kernel": kname if cascade else {1: "cuda-core", 2: "tcgen05"}[kernel],
                        "partitions": P,
                        "partition_tokens": psize},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic,
                     "traffic_ratio": round(traffic / alg, 4) if traffic else None,
                     "peak_source": f"hbm_gbs ({peak_src})",
                     "kernel": ("pa_decode_shared_prefix (suffix pass + prefix pass + merge)"
                                if cascade else "pa_decode (partition pass + merge)") + ", per launch",
                     "algorithmic_bytes": alg},
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": Ke},
    }
    if ab is not None:
        line["kernel_ab"] = ab
    del d
    torch.cuda.empty_cache()
    return line


def ours_arm(args, w: W.Workload, rank: int, world: int, local_rank: int):
    return measure(args, w, rank, world, local_rank,
                   cascade=bool(getattr(args, "shared_prefix", False)))


SUITE = [  # (workload id, shared-prefix decode) measured beside the headline by default
    (3, False), (4, False), (5, False), (5, True), (6, False), (7, False), (8, False)]


def suite(args, local_rank: int):
    """Every other decode workload at full size, one GPU: the same step and
    fields as the headline (plus the CUDA-core A/B on the tensor-core shapes),
    each with a bounded oracle sample as its CPU baseline."""
    out = {}
    for k, cascade in SUITE:
        w = W.make_workload(k, seed=rank_seed(k, 0))
        line = measure(args, w, 0, 1, local_rank, cascade=cascade, cuda_core_ab=True)
        line["cpu_baseline"] = cpu_baseline(w, budget_s=3.0)
        keep = ("value", "unit", "ms_per_step", "decode_us", "kernel_ab",
                "seq_steps_per_s", "pct_of_hbm_peak", "decode_plan",
                "roofline", "gpu_launches", "clocks", "e2e", "cpu_baseline", "config", "dtype")
        out[w.name + (" (pa_decode_shared_prefix)" if cascade else "")] = \
            {k2: line[k2] for k2 in keep if k2 in line}
        del w
    return out


def warm_l2(args, local_rank: int):
    """Decode of a Llama-2-7B-shaped batch small enough for the 126 MB L2 (4
    sequences), back to back without a flush (warm) and with the L2 flushed
    before each call (cold)."""
    import torch
    dev = torch.device("cuda", local_rank)
    w = W.make_workload(2, seed=rank_seed(2, 0), batch=4)
    d = Decoder(w, dev)
    d.cache_ops()
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    K = max(20, args.steps)
    warm = time_decode_only(d, K)
    cold = time_decode_only(d, K, flush_buf)
    kv = w.kv_bytes()
    peak, _ = peaks()
    del d, flush_buf
    torch.cuda.empty_cache()
    return {"workload": w.name, "kv_bytes": kv, "calls": K,
            "decode_us_warm": round(warm * 1e3, 2), "gbs_warm": round(kv / (warm / 1e3) / 1e9, 1),
            "decode_us_cold": round(cold * 1e3, 2), "gbs_cold": round(kv / (cold / 1e3) / 1e9, 1),
            "frac_of_hbm_peak_warm": round(kv / (warm / 1e3) / 1e9 / peak, 4),
            "note": "decode calls back to back; warm = no flush (the batch stays in L2), "
                    "cold = 252 MB written before each call"}


def paging_cost(args, local_rank: int):
    """The same decode on the same lengths and bytes, with each sequence's
    blocks contiguous (identity-like table) instead of popped from a shuffled
    free list: what non-contiguous physical blocks cost the kernel."""
    import torch
    dev = torch.device("cuda", local_rank)
    res = {}
    for k in (2, 3):
        K = max(20, args.steps)
        times = {}
        for layout in ("contiguous", "shuffled"):
            w = W.make_workload(k, seed=rank_seed(k, 0), contiguous=layout == "contiguous")
            d = Decoder(w, dev)
            d.cache_ops()
            times[layout] = time_decode_only(d, K)
            kv = w.kv_bytes()
            del d, w
            torch.cuda.empty_cache()
        res[W.WORKLOADS[k]] = {
            "decode_us_contiguous": round(times["contiguous"] * 1e3, 2),
            "decode_us_shuffled": round(times["shuffled"] * 1e3, 2),
            "paging_overhead_pct": round(100.0 * (times["shuffled"] / times["contiguous"] - 1), 2),
            "kv_bytes": kv, "calls": K}
    res["note"] = ("decode calls back to back (inputs larger than L2); contiguous = every "
                   "sequence's blocks are consecutive physical ids, shuffled = ids popped from "
                   "a seeded permutation of the pool (the benchmark's layout)")
    return res


def rank_seed(k: int, rank: int) -> int:
    """Seed of workload k on one rank: every replica gets its own batch."""
    return 1000 + k + 7919 * rank


def max_over_ranks(vals, world: int, device):
    """Elementwise max of per-rank timings (ms) over all ranks; identity at N=1."""
    if world <= 1:
        return [float(v) for v in vals]
    import torch
    import torch.distributed as dist
    tt = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return [float(v) for v in tt.tolist()]


def job_value(kv_bytes_per_step: int, steps: int, world: int, ms: float) -> float:
    """Whole-job algorithmic GB/s: every rank streams its own batch of kv_bytes per
    step (weak scaling), and the job takes the slowest rank's time."""
    return kv_bytes_per_step * steps * world / (ms / 1e3) / 1e9


def cpu_baseline(w: W.Workload, budget_s: float = 10.0):
    """The oracle as it stands on the host cores: whole steps repeated until
    about budget_s of CPU work, or a sample of rows if one step is longer."""
    import oracle
    all_rows = np.array([(b, h) for b in range(w.B) for h in range(w.Hq)], dtype=np.int32)
    rows = oracle_sample_rows(w, budget_s=budget_s)
    if len(rows) < len(all_rows):
        secs, byts = run_oracle(w, rows, reps=1)
        reps = 1
    else:
        rows = all_rows
        secs, byts = run_oracle(w, rows, reps=1)
        reps = 1
        while secs < budget_s and reps < 1000:
            s2, b2 = run_oracle(w, rows, reps=1)
            secs, byts, reps = secs + s2, byts + b2, reps + 1
    return {"value": round(byts / secs / 1e9, 4), "unit": "GB/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": (f"{len(rows)} of {w.B * w.Hq} (sequence, query head) rows "
                       f"({100.0 * len(rows) / (w.B * w.Hq):.1f}%) per step plus the step's "
                       f"cache ops, {reps} step(s), {secs:.1f} s of host time; value scaled "
                       f"by the rows' share of KV bytes")}


SWAP_METRIC = "swap_blocks GB/s (device <-> page-locked host)"


def swap_arm(args, rank: int, world: int, local_rank: int):
    """Blocks of the Llama-2-7B-shaped pool (16 tokens x 32 heads x 128, fp16:
    128 KiB per block per pool) swapped out to a pinned host pool and back in."""
    import torch
    from paged_kv_cache_418_b200 import ops
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    nd, nh, bs, hkv, d = 8192, 2048, 16, 32, 128
    rng = np.random.default_rng(rank_seed(7, rank))
    dk = torch.randn((nd, bs, hkv, d), dtype=torch.float16, device=dev)
    dv = torch.randn((nd, bs, hkv, d), dtype=torch.float16, device=dev)
    hk = torch.empty((nh, bs, hkv, d), dtype=torch.float16).pin_memory()
    hv = torch.empty((nh, bs, hkv, d), dtype=torch.float16).pin_memory()
    out_map = np.stack([rng.choice(nd, nh, replace=False), rng.permutation(nh)], 1)
    in_map = np.stack([rng.permutation(nh), rng.choice(nd, nh, replace=False)], 1)
    out_map = torch.from_numpy(out_map.astype(np.int64)).to(dev)
    in_map = torch.from_numpy(in_map.astype(np.int64)).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    moved = 2 * nh * bs * hkv * d * 2                 # K + V bytes per direction

    def timed(fn, reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / reps

    swap_out = lambda: ops.pa_swap_blocks(hk, hv, dk, dv, out_map, err, stream)
    swap_in = lambda: ops.pa_swap_blocks(dk, dv, hk, hv, in_map, err, stream)
    flat_d = dk[:nh].view(-1)
    flat_h = hk.view(-1)
    copy_out = lambda: (flat_h.copy_(flat_d, non_blocking=True), hv.view(-1).copy_(dv[:nh].view(-1), non_blocking=True))
    copy_in = lambda: (flat_d.copy_(flat_h, non_blocking=True), dv[:nh].view(-1).copy_(hv.view(-1), non_blocking=True))
    K = max(1, min(args.steps, 20))
    for _ in range(max(3, args.warmup)):
        swap_out(); swap_in()
    torch.cuda.synchronize(dev)
    t_out, t_in = timed(swap_out, K), timed(swap_in, K)
    c_out, c_in = timed(copy_out, K), timed(copy_in, K)
    torch.cuda.synchronize(dev)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())}")
    (t_out, t_in) = max_over_ranks([t_out, t_in], world, dev)
    g = lambda ms: moved / (ms / 1e3) / 1e9
    value = 2 * moved * world / ((t_out + t_in) / 1e3) / 1e9
    peak = 2 * moved / ((c_out + c_in) / 1e3) / 1e9
    # oracle: the same block copies between two host pools, on a sample of blocks
    import oracle
    n_s = 256
    sk, sv = hk[:n_s].numpy(), hv[:n_s].numpy()
    tk, tv = np.empty_like(sk), np.empty_like(sv)
    pairs = np.stack([np.arange(n_s), np.random.default_rng(0).permutation(n_s)], 1)
    t0, reps = time.perf_counter(), 0
    while time.perf_counter() - t0 < 2.0:
        oracle.swap_blocks(tk, tv, sk, sv, pairs)
        reps += 1
    cpu = 2 * n_s * bs * hkv * d * 2 * reps / (time.perf_counter() - t0) / 1e9
    return {
        "metric": SWAP_METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": max(3, args.warmup), "ms_per_step": round(t_out + t_in, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": "swap llama2-7b-shaped blocks", "blocks_per_direction": nh,
                   "block_bytes_k_plus_v": 2 * bs * hkv * d * 2, "device_pool_blocks": nd,
                   "mapping": "random distinct device ids <-> permuted host ids"},
        "swap_out_gbs": round(g(t_out), 2), "swap_in_gbs": round(g(t_in), 2),
        "roofline": {"bound": "host-link", "achieved": round(2 * moved / ((t_out + t_in) / 1e3) / 1e9, 2),
                     "peak": round(peak, 2), "unit": "GB/s",
                     "frac": round(peak and (2 * moved / ((t_out + t_in) / 1e3) / 1e9) / peak, 4),
                     "traffic": None,
                     "peak_source": "cudaMemcpyAsync of the same bytes (contiguous, copy engine), this run",
                     "memcpy_out_gbs": round(g(c_out), 2), "memcpy_in_gbs": round(g(c_in), 2)},
        "gpu_launches": 2 * K,
        "e2e": {"value": round(value, 2), "unit": "GB/s", "h2d_bytes_per_step": moved,
                "d2h_bytes_per_step": moved},
        "cpu_baseline": {"value": round(cpu, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"{n_s} blocks host->host, {reps} repetitions in 2 s"},
    }


PREFILL_METRIC = "paged prefill attention TFLOP/s"


def prefill_case(rank: int):
    """Chunked prefill of a Llama-3-70B-shaped batch: 8 sequences with U[0, 2048]
    cached tokens each take a 512-token chunk (64 query heads over 8 KV heads,
    D = 128, bf16, 16-token blocks)."""
    rng = np.random.default_rng(rank_seed(8, rank))
    prior = rng.integers(0, 2049, size=8)
    return W.build_prefill_case("prefill-chunk512-llama3-70b-bf16", W.BF16, Hq=64, Hkv=8, D=128,
                                block_size=16, prior_lens=prior, new_lens=[512] * 8,
                                seed=rank_seed(8, rank))


def prefill_arm(args, rank: int, world: int, local_rank: int):
    import torch
    import oracle
    from paged_kv_cache_418_b200 import ops
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    c = prefill_case(rank)
    t = W.prefill_to_torch(c, dev)
    out = torch.empty((c.T, c.Hq, c.D), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    run = lambda: ops.pa_prefill(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                 t["context_lens"], t["query_start"], c.max_query_len, c.scale,
                                 c.max_context_len, err, stream)
    for _ in range(max(3, args.warmup)):
        run()
    torch.cuda.synchronize(dev)
    K = max(1, min(args.steps, 200))
    sampler = ClockSampler(gpu_smi_id(local_rank))
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        run()
    e1.record(stream)
    e1.synchronize()
    clocks = sampler.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())}")
    ms = e0.elapsed_time(e1) / K
    (ms,) = max_over_ranks([ms], world, dev)
    flops = c.attention_flops()
    tflops = flops / (ms / 1e3) / 1e12
    # the same calls on the multi-query kernel (key rows on the MMA's M), same loop
    os.environ["PA_PREFILL_KERNEL"] = "mq"
    try:
        for _ in range(3):
            run()
        e0.record(stream)
        for _ in range(K):
            run()
        e1.record(stream)
        e1.synchronize()
        ms_mq = e0.elapsed_time(e1) / K
    finally:
        del os.environ["PA_PREFILL_KERNEL"]
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    peak = float(json.load(open(path))["bf16_tflops"]) if os.path.exists(path) else 1590.0
    # end to end: the query from pinned host memory, the output back, every call
    hq = t["q"].cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(K):
        t["q"].copy_(hq, non_blocking=True)
        run()
        hout.copy_(out, non_blocking=True)
    e3.record(stream)
    e3.synchronize()
    e_ms = e2.elapsed_time(e3) / K
    # oracle on the host cores: the first sequence's chunk (a bounded sample)
    sub = W.build_prefill_case("sample", W.BF16, Hq=64, Hkv=8, D=128, block_size=16,
                               prior_lens=[int(c.context_lens[0]) - 512], new_lens=[64],
                               seed=1)
    t0 = time.perf_counter()
    oracle.prefill(sub.q, sub.k_cache, sub.v_cache, W.BF16, sub.block_tables, sub.context_lens,
                   sub.query_start, sub.scale)
    cpu_s = time.perf_counter() - t0
    return {
        "metric": PREFILL_METRIC, "value": round(tflops * world, 2), "unit": "TFLOP/s",
        "n_gpus": world, "steps": K, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": c.name, "B": c.B, "Hq": c.Hq, "Hkv": c.Hkv, "head_dim": c.D,
                   "block_size": c.block_size, "new_tokens": c.T,
                   "prior_tokens": int((c.context_lens - 512).sum()),
                   "flops_per_step": flops, "l2": "K/V of the batch read once per 8-token "
                   "query chunk; inputs resident, no flush (compute-bound)"},
        "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                     "traffic": traffic_record("prefill", c.name),
                     "peak_source": "bf16_tflops (measured, burst)",
                     "kernel": "prefill_fa_kernel (query rows on the MMA's M), per launch; "
                               "algorithmic flops 4*D per (query head, attended key)"},
        "kernel_ab": {"tflops_rows_on_m": round(tflops, 2),
                      "tflops_multi_query": round(flops / (ms_mq / 1e3) / 1e12, 2),
                      "ms_rows_on_m": round(ms, 5), "ms_multi_query": round(ms_mq, 5),
                      "how": f"{K} calls back to back per kernel, same inputs"},
        "gpu_launches": K,
        "clocks": clocks,
        "e2e": {"value": round(flops / (e_ms / 1e3) / 1e12 * world, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": hq.numel() * hq.element_size(),
                "d2h_bytes_per_step": hout.numel() * hout.element_size()},
        "cpu_baseline": {"value": round(sub.attention_flops() / cpu_s / 1e12, 6),
                         "unit": "TFLOP/s", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": f"64 of the first sequence's 512 new tokens, {cpu_s:.1f} s"},
    }


def prefill_reference_arm(args):
    """The oracle on the host cores for the prefill workload: a bounded sample of
    each step (64 new tokens of one sequence), scaled to TFLOP/s of the sample."""
    import oracle
    c = prefill_case(0)
    sub = W.build_prefill_case("sample", W.BF16, Hq=64, Hkv=8, D=128, block_size=16,
                               prior_lens=[int(c.context_lens[0]) - 512], new_lens=[64], seed=1)
    steps = max(1, min(args.steps, 5))
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.prefill(sub.q, sub.k_cache, sub.v_cache, W.BF16, sub.block_tables,
                       sub.context_lens, sub.query_start, sub.scale)
    secs = time.perf_counter() - t0
    value = sub.attention_flops() * steps / secs / 1e12
    sample = f"64 new tokens of one sequence per step, {steps} step(s), {secs:.1f} s"
    return {"impl": "reference", "metric": PREFILL_METRIC, "value": round(value, 6),
            "unit": "TFLOP/s", "n_gpus": 1, "steps": steps, "warmup": 0,
            "ms_per_step": round(1e3 * secs / steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": c.name, "sample": sample},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                             "cores": oracle.max_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.prefill:
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps(prefill_reference_arm(args)), flush=True)
            return 0
        if world > 1:
            return 0 if rank else (print(json.dumps({"impl": args.impl, "unavailable":
                "prefill measurement runs on one GPU"})) or 0)
        print(json.dumps(prefill_arm(args, rank, world, int(os.environ.get("LOCAL_RANK", "0")))),
              flush=True)
        return 0
    if args.swap:
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if args.impl == "reference" or world > 1:
            return 0 if rank else (print(json.dumps({"impl": args.impl, "unavailable":
                "swap measurement runs on one GPU with --impl ours"})) or 0)
        line = swap_arm(args, rank, world, int(os.environ.get("LOCAL_RANK", "0")))
        print(json.dumps(line), flush=True)
        return 0
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    default_run = args.workload is None
    k = workload_id(args.workload or HEADLINE)
    seed = rank_seed(k, rank)
    if args.impl == "reference":
        if rank != 0:
            return 0
        w = W.make_workload(k, seed=seed, batch=args.batch)
        line = reference_arm(args, w, rank, world)
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local_rank))
    w = W.make_workload(k, seed=seed, batch=args.batch)
    try:
        line = ours_arm(args, w, rank, world, local_rank)
        if rank == 0 and world == 1:
            line["cpu_baseline"] = cpu_baseline(w)
        elif rank == 0:
            line["cpu_baseline"] = {"value": None, "unit": "GB/s", "cores": 0, "kind": "oracle",
                                    "sample": "timed at N=1 only"}
    finally:
        if world > 1:
            dist.destroy_process_group()
    del w
    if rank == 0 and default_run and not args.no_suite:
        if world == 1 and args.batch is None:
            # the other workloads of the same step, and two reference measurements
            line["per_workload"] = suite(args, local_rank)
            line["warm_l2"] = warm_l2(args, local_rank)
            line["paging_cost"] = paging_cost(args, local_rank)
            keep = ("metric", "value", "unit", "ms_per_step", "roofline", "kernel_ab", "clocks",
                    "e2e", "cpu_baseline", "config", "gpu_launches")
            if not args.skip_prefill:
                pf = prefill_arm(args, 0, 1, local_rank)
                line["prefill"] = {k2: pf[k2] for k2 in keep if k2 in pf}
            sw = swap_arm(args, 0, 1, local_rank)
            line["swap_blocks"] = {k2: sw[k2] for k2 in keep + ("swap_out_gbs", "swap_in_gbs")
                                   if k2 in sw}
        else:
            line["per_workload"] = {"note": "measured at N=1 only (one GPU)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
