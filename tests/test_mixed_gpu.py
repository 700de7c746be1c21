"""Pools of two element types (K as FP8 E4M3 codes beside a 16-bit V pool, and
the reverse), FP8 pools under grouped-query attention, and both load
schedules of the CUDA-core kernel, on the GPU through the C ABI against the
fp64 oracle. The bound is the query type's (4e-3 for 16-bit queries): the
oracle reads the very codes and values the kernel reads, times the same scales.
"""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200 import workloads as W
from pa_testlib import assert_attention_close, device_inputs, device_step, oracle_step

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["prefetch", "no-prefetch"])
def load_schedule(request, monkeypatch):
    monkeypatch.setenv("PA_SIMT_PREFETCH", "1" if request.param == "prefetch" else "0")
    return request.param


@pytest.mark.parametrize("which", [7, 8])
@pytest.mark.parametrize("out_f32", [True, False])
def test_shrunk_mixed_and_fp8_gqa_workloads_full_parity(which, out_f32, load_schedule):
    w = W.shrink_workload(which, seed=300 + which)
    out, t = device_step(w, out_dtype=torch.float32 if out_f32 else None)
    ref, kc, vc = oracle_step(w)
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    assert_attention_close(out, ref, w.dtype, w.name)
    assert np.array_equal(t["k_cache"].cpu().view(torch.uint8).numpy().reshape(-1),
                          kc.view(np.uint8).reshape(-1))
    assert np.array_equal(t["v_cache"].cpu().view(torch.uint8).numpy().reshape(-1),
                          vc.view(np.uint8).reshape(-1))


SHAPES = [(D, bs, G) for D in (64, 128) for bs in (16, 32) for G in (1, 2, 4, 8, 16)]


@pytest.mark.parametrize("D,bs,G", SHAPES)
@pytest.mark.parametrize("kv", ["k8", "v8"])
def test_every_shape_with_one_fp8_pool(D, bs, G, kv, load_schedule):
    rng = np.random.default_rng(D * 11 + bs * 5 + G + (kv == "v8"))
    Hkv = 2
    ctx = [1, bs - 1, bs, bs + 1, 2 * bs + 3, 37, 129, 600]
    nb = sum((c + bs - 1) // bs for c in ctx) + 5
    dt = W.BF16 if kv == "k8" else W.F16
    w = W.build_decode_case("mixed-sweep", dt, B=len(ctx), Hq=Hkv * G, Hkv=Hkv, D=D,
                            block_size=bs, num_blocks=nb, context_lens=ctx,
                            seed=int(rng.integers(1 << 30)), kv_fp8=kv == "k8",
                            v_fp8=kv == "v8", k_scale=0.45, v_scale=0.8)
    assert w.mixed
    for psize in (0, bs, 8 * bs):
        out, t = device_step(w, out_dtype=torch.float32, partition_size=psize)
        ref, _, _ = oracle_step(w)
        torch.cuda.synchronize()
        assert int(t["err"].item()) == 0
        assert_attention_close(out, ref, dt, f"{kv} psize={psize}")


def test_reshape_and_cache_kv_writes_codes_and_copies_bit_exactly():
    for k8 in (True, False):
        w = W.build_decode_case("rac-kv", W.BF16, B=7, Hq=8, Hkv=4, D=128, block_size=16,
                                num_blocks=40, context_lens=[1, 15, 16, 17, 33, 100, 64],
                                seed=17 + k8, kv_fp8=k8, v_fp8=not k8, k_scale=0.05,
                                v_scale=0.02)             # small scales: saturated codes occur
        t = device_inputs(w)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ops.pa_reshape_and_cache_kv(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                    w.k_scale, w.v_scale, t["slot_mapping"], err)
        kc, vc = w.k_cache.copy(), w.v_cache.copy()
        oracle.reshape_and_cache_mixed(kc, vc, w.new_key, w.new_value, w.dtype, w.kv_dtype,
                                       w.v_dtype, w.k_scale, w.v_scale, w.slot_mapping)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert np.array_equal(t["k_cache"].cpu().view(torch.uint8).numpy().reshape(-1),
                              kc.view(np.uint8).reshape(-1))
        assert np.array_equal(t["v_cache"].cpu().view(torch.uint8).numpy().reshape(-1),
                              vc.view(np.uint8).reshape(-1))


def test_mixed_pools_need_a_16_bit_query():
    q = torch.zeros(2, 4, 128, dtype=torch.float32, device="cuda")
    kc = torch.zeros(4, 16, 4, 128, dtype=torch.uint8, device="cuda")
    vc = torch.zeros(4, 16, 4, 128, dtype=torch.float32, device="cuda")
    tables = torch.zeros(2, 4, dtype=torch.int32, device="cuda")
    lens = torch.ones(2, dtype=torch.int32, device="cuda")
    out = torch.zeros(2, 4, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(ops.PAError) as e:
        ops.pa_decode_kv(out, q, kc, vc, 0.5, 1.0, tables, lens, 0.1, 16)
    assert e.value.status == 3
    # a 16-bit pool of another type than the query's is refused too
    vc16 = torch.zeros(4, 16, 4, 128, dtype=torch.float16, device="cuda")
    qb = q.to(torch.bfloat16)
    with pytest.raises(ops.PAError) as e:
        ops.pa_decode_kv(out, qb, kc, vc16, 0.5, 1.0, tables, lens, 0.1, 16)
    assert e.value.status == 3


# -- FP8 pools on the tensor cores (grouped-query shapes, 16-bit query) ------------
@pytest.mark.parametrize("qdt", [W.F16, W.BF16])
@pytest.mark.parametrize("G,Hkv", [(4, 4), (8, 8)])
@pytest.mark.parametrize("bs", [16, 32])
def test_fp8_pools_on_the_tensor_cores(qdt, G, Hkv, bs):
    ctx = [1, bs - 1, bs, 33, 129, 700, 2049, 64]
    nb = sum((c + bs - 1) // bs for c in ctx) + 5
    w = W.build_decode_case("fp8-tc", qdt, B=len(ctx), Hq=G * Hkv, Hkv=Hkv, D=128, block_size=bs,
                            num_blocks=nb, context_lens=ctx, seed=G * 100 + bs + qdt, kv_fp8=True)
    assert ops.pa_decode_plan(W.FP8, w.B, w.Hq, w.Hkv, w.D, bs, w.max_context_len)[0] == 2
    for out_f32 in (True, False):
        out, t = device_step(w, out_dtype=torch.float32 if out_f32 else None)
        ref, _, _ = oracle_step(w)
        torch.cuda.synchronize()
        assert int(t["err"].item()) == 0
        assert_attention_close(out, ref, qdt, f"G={G} bs={bs} f32={out_f32}")


@pytest.mark.parametrize("qdt", [W.F16, W.BF16])
@pytest.mark.parametrize("ctx,G", [
    ([5000, 37, 1, 800, 4096, 33, 64, 3000] + [17] * 20 + [2049, 700], 8),   # many pieces
    ([300 + 37 * i for i in range(150)], 4),           # many whole sequences per CTA
])
def test_fp8_tensor_cores_over_long_walks(qdt, ctx, G):
    """Every CTA walks many tiles, so each stage of the ring serves K and V in
    turn many times over, and sequences are cut into pieces across CTAs."""
    nb = sum((c + 15) // 16 for c in ctx) + 5
    w = W.build_decode_case("fp8-tc-long", qdt, B=len(ctx), Hq=G * 8, Hkv=8, D=128,
                            block_size=16, num_blocks=nb, context_lens=ctx, seed=G + qdt,
                            kv_fp8=True, k_boost_frac=0.02)
    assert ops.pa_decode_plan(W.FP8, w.B, w.Hq, w.Hkv, w.D, 16, w.max_context_len)[0] == 2
    out, t = device_step(w, out_dtype=torch.float32)
    ref, _, _ = oracle_step(w)
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    assert_attention_close(out, ref, qdt, f"G={G}")


@pytest.mark.parametrize("qdt", [W.F16, W.BF16])
def test_fp8_tensor_core_widening_is_exact_for_every_code(qdt):
    """One token with weight exactly 1: o = value(code) * v_scale, for every finite
    E4M3 code (subnormals and +-448 included), through the tensor-core kernel's
    in-place widening of the codes to the query's 16-bit type."""
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    D, Hkv, G = 128, 4, 8
    w = W.build_decode_case("fp8-tc-codes", qdt, B=1, Hq=G * Hkv, Hkv=Hkv, D=D, block_size=16,
                            num_blocks=4, context_lens=[2], seed=13, kv_fp8=True, v_scale=0.37)
    assert ops.pa_decode_plan(W.FP8, 1, G * Hkv, Hkv, D, 16, 2)[0] == 2
    codes = np.concatenate([finite, finite, finite[:Hkv * D - 2 * len(finite)]]).reshape(Hkv, D)
    blk = w.block_tables[0, 0]
    w.v_cache[blk, 0] = codes
    w.k_cache[blk, 0] = 0x00                                   # k0 = 0: score 0
    one = W.round_to_storage(np.ones(1, dtype=np.float32), qdt)[0]
    w.q[:] = one
    w.new_key[:] = W.round_to_storage(np.full(1, -1e4, dtype=np.float32), qdt)[0]
    out, t = device_step(w, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    exp = (oracle.widen(codes, oracle.FP8) * w.v_scale).astype(np.float32)   # [Hkv, D]
    exp = np.repeat(exp[None], G, axis=0).transpose(1, 0, 2).reshape(1, G * Hkv, D)
    assert torch.equal(out.cpu(), torch.from_numpy(exp))
