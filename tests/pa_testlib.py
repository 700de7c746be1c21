"""Shared helpers of the GPU parity tests: run one decode step through the
C-ABI on the device, and the same step through the fp64 oracle on the host.

Tolerances (attention): max abs error <= 1e-5 for fp32 inputs and <= 4e-3
for fp16 / bf16 inputs when the kernel writes fp32 output. When it writes the
input type, the fp32 result within that bound is then rounded once more, so
|out - oracle| <= ATOL + ulp(out) / 2 (a correctly rounded 16-bit output can by
itself be more than 4e-3 from the exact value: bf16 values in [2, 4) are 2^-6
apart). With FP8 pools the bound is the query type's: the oracle reads the
very codes the kernel reads (times the same scales), so only the kernel's
fp32 arithmetic and the output rounding separate the two.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200.workloads import BF16, F16, F32, FP8, Workload, to_torch

ATOL = {F32: 1e-5, F16: 4e-3, BF16: 4e-3}
TORCH_DT = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}


def device_inputs(w: Workload, device="cuda"):
    return to_torch(w, device)


def device_step(w: Workload, t=None, out_dtype=None, partition_size=None, err=None,
                stream=None, do_cache_ops=True, max_context_len=None):
    """copy_blocks -> reshape_and_cache -> decode on the device; returns (out, tensors)."""
    t = device_inputs(w) if t is None else t
    dev = t["q"].device
    err = torch.zeros(1, dtype=torch.int32, device=dev) if err is None else err
    if do_cache_ops:
        if len(w.block_mapping):
            ops.pa_copy_blocks(t["k_cache"], t["v_cache"], t["block_mapping"], err, stream)
        if w.mixed:
            ops.pa_reshape_and_cache_kv(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                        w.k_scale, w.v_scale, t["slot_mapping"], err, stream)
        elif w.fp8:
            ops.pa_reshape_and_cache_fp8(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                         w.k_scale, w.v_scale, t["slot_mapping"], err, stream)
        else:
            ops.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                     t["slot_mapping"], err, stream)
    odt = TORCH_DT[w.dtype] if out_dtype is None else out_dtype
    out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=odt, device=dev)
    psize = w.partition_size if partition_size is None else partition_size
    mcl = w.max_context_len if max_context_len is None else max_context_len
    ws = ops.workspace_for(t["q"], t["k_cache"], mcl, psize)
    if w.mixed:
        ops.pa_decode_kv(out, t["q"], t["k_cache"], t["v_cache"], w.k_scale, w.v_scale,
                         t["block_tables"], t["context_lens"], w.scale, mcl, psize, ws, err,
                         stream)
    elif w.fp8:
        ops.pa_decode_fp8(out, t["q"], t["k_cache"], t["v_cache"], w.k_scale, w.v_scale,
                          t["block_tables"], t["context_lens"], w.scale, mcl, psize, ws, err,
                          stream)
    else:
        ops.pa_decode(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                      t["context_lens"], w.scale, mcl, psize, ws, err, stream)
    t["workspace"] = ws
    t["err"] = err
    return out, t


def oracle_step(w: Workload, rows=None, do_cache_ops=True):
    """The same step on host copies of the pools, in fp64."""
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    if do_cache_ops:
        if len(w.block_mapping):
            assert not w.mixed, "copy-on-write pairs over pools of two element types"
            oracle.copy_blocks(kc, vc, w.block_mapping, w.kv_dtype)
        if w.mixed:
            oracle.reshape_and_cache_mixed(kc, vc, w.new_key, w.new_value, w.dtype, w.kv_dtype,
                                           w.v_dtype, w.k_scale, w.v_scale, w.slot_mapping)
        elif w.fp8:
            oracle.reshape_and_cache_fp8(kc, vc, w.new_key, w.new_value, w.dtype, w.k_scale,
                                         w.v_scale, w.slot_mapping)
        else:
            oracle.reshape_and_cache(kc, vc, w.new_key, w.new_value, w.slot_mapping, w.dtype)
    if w.mixed:
        out = oracle.decode_mixed(w.q, w.dtype, kc, w.kv_dtype, w.k_scale, vc, w.v_dtype,
                                  w.v_scale, w.block_tables, w.context_lens, w.scale, rows=rows)
    elif w.fp8:
        out = oracle.decode_kv(w.q, w.dtype, kc, vc, FP8, w.k_scale, w.v_scale, w.block_tables,
                               w.context_lens, w.scale, rows=rows)
    else:
        out = oracle.decode(w.q, kc, vc, w.dtype, w.block_tables, w.context_lens, w.scale,
                            rows=rows)
    return out, kc, vc


def assert_attention_close(got: torch.Tensor, ref: np.ndarray, dtype: int, what=""):
    g = got.detach().to("cpu")
    if g.dtype == torch.float32:
        err = np.abs(g.numpy().astype(np.float64) - ref)
        assert np.isfinite(g.numpy()).all(), f"{what}: non-finite output"
        worst = float(err.max()) if err.size else 0.0
        assert worst <= ATOL[dtype], f"{what}: max abs error {worst:.3e} > {ATOL[dtype]:.0e}"
        return worst
    # 16-bit output: the fp32 bound plus the output's own half-ulp rounding
    gf = g.to(torch.float64)
    assert torch.isfinite(gf).all(), f"{what}: non-finite output"
    mant = 7 if g.dtype == torch.bfloat16 else 10
    e = torch.floor(torch.log2(gf.abs().clamp_min(2.0 ** -14)))
    half_ulp = torch.pow(2.0, e - mant - 1)
    err = (gf - torch.from_numpy(ref)).abs()
    bad = err > ATOL[dtype] + half_ulp
    assert not bad.any(), f"{what}: {int(bad.sum())} outputs beyond {ATOL[dtype]:.0e} + ulp/2"
    return float(err.max())


def bits(t: torch.Tensor) -> torch.Tensor:
    """Bit pattern view for exact comparisons (NaN payloads included)."""
    if t.dtype == torch.uint8:
        return t
    return t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)


def host_bits(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint8:
        return torch.from_numpy(np.ascontiguousarray(a))
    v = a.view(np.int32) if a.dtype == np.float32 else a.view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(v))


def sample_rows(w: Workload, n: int, seed: int = 0) -> np.ndarray:
    """(b, hq) rows for spot checks: the longest and shortest sequences, all heads of
    one sequence, and random ones."""
    rng = np.random.default_rng(seed)
    ctx = w.context_lens
    rows = {(int(np.argmax(ctx)), 0), (int(np.argmax(ctx)), w.Hq - 1),
            (int(np.argmin(ctx)), w.Hq // 2)}
    b0 = int(rng.integers(w.B))
    for hq in range(0, w.Hq, max(1, w.Hq // 8)):
        rows.add((b0, hq))
    while len(rows) < n:
        rows.add((int(rng.integers(w.B)), int(rng.integers(w.Hq))))
    return np.array(sorted(rows), dtype=np.int32)
