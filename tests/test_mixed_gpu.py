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
