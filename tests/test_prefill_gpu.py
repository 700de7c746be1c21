"""Paged prefill (causal, chunked) on the GPU against the fp64 oracle, on both
prefill kernels: the default one (query rows on the MMA's M) and the
multi-query kernel (key rows on M), chosen with PA_PREFILL_KERNEL."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200 import workloads as W
from pa_testlib import assert_attention_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["rows-on-m", "multi-query"])
def prefill_kernel(request, monkeypatch):
    if request.param == "multi-query":
        monkeypatch.setenv("PA_PREFILL_KERNEL", "mq")
    else:
        monkeypatch.delenv("PA_PREFILL_KERNEL", raising=False)
    return request.param


def _run(c, out_dtype=torch.float32, ctx=None):
    t = W.prefill_to_torch(c, "cuda")
    if ctx is not None:
        t["context_lens"] = torch.from_numpy(np.asarray(ctx, dtype=np.int32)).cuda()
    out = torch.full((c.T, c.Hq, c.D), float("nan"), dtype=out_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.pa_prefill(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                   t["query_start"], c.max_query_len, c.scale, c.max_context_len, err)
    torch.cuda.synchronize()
    return out, err


SHAPES = [(dt, G, bs) for dt in (W.F16, W.BF16) for G in (1, 2, 4, 8, 16) for bs in (16, 32)]


@pytest.mark.parametrize("dtype,G,bs", SHAPES)
def test_prefill_every_shape(dtype, G, bs):
    c = W.build_prefill_case("pf", dtype, Hq=2 * G, Hkv=2, D=128, block_size=bs,
                             prior_lens=[0, 5, 130, bs, 300, 7], new_lens=[1, 40, 0, 2 * bs + 3, 129, 64],
                             seed=G * 10 + bs + dtype)
    out, err = _run(c)
    ref = oracle.prefill(c.q, c.k_cache, c.v_cache, dtype, c.block_tables, c.context_lens,
                         c.query_start, c.scale)
    assert int(err.item()) == 0
    assert_attention_close(out, ref, dtype, f"G={G} bs={bs}")


def test_prefill_long_chunk_with_peaked_scores_and_16bit_output():
    rng = np.random.default_rng(8)
    c = W.build_prefill_case("pf-long", W.BF16, Hq=64, Hkv=8, D=128, block_size=16,
                             prior_lens=[2000, 0], new_lens=[700, 300], seed=9)
    # a few large K rows move the reference maxima mid-sequence (the lazy rescale)
    kc = c.k_cache.view(np.uint16)
    boost = W.round_to_storage((rng.standard_normal((40, 8, 128)) * 100).astype(np.float32), W.BF16)
    rows = rng.choice(2700, 40, replace=False)
    for i, tok in enumerate(rows):
        kc[c.block_tables[0, tok // 16], tok % 16] = boost[i]
    out, err = _run(c, out_dtype=torch.bfloat16)
    ref = oracle.prefill(c.q, c.k_cache, c.v_cache, W.BF16, c.block_tables, c.context_lens,
                         c.query_start, c.scale)
    assert int(err.item()) == 0
    assert_attention_close(out, ref, W.BF16, "long")


def test_prefill_bad_lengths_are_flagged():
    c = W.build_prefill_case("pf-bad", W.F16, Hq=8, Hkv=2, D=128, block_size=16,
                             prior_lens=[10, 4], new_lens=[5, 6], seed=4)
    out, err = _run(c, ctx=[15, 3])                 # the second sequence holds fewer than 6
    assert int(err.item()) & ops.PA_DEV_BAD_CTX
    ref = oracle.prefill(c.q, c.k_cache, c.v_cache, W.F16, c.block_tables, c.context_lens,
                         c.query_start, c.scale)
    assert_attention_close(out[:5], ref[:5], W.F16, "good sequence")


def test_prefill_rejects_unsupported_shapes_before_launch():
    c = W.build_prefill_case("pf-f32", W.F32, Hq=4, Hkv=4, D=128, block_size=16,
                             prior_lens=[3], new_lens=[2], seed=1)
    t = W.prefill_to_torch(c, "cuda")
    out = torch.empty((c.T, c.Hq, c.D), dtype=torch.float32, device="cuda")
    with pytest.raises(ops.PAError) as e:
        ops.pa_prefill(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                       t["context_lens"], t["query_start"], c.max_query_len, c.scale,
                       c.max_context_len)
    assert e.value.status == 4


def test_prefill_bad_block_id_is_flagged_and_left_out():
    c = W.build_prefill_case("pf-badblk", W.BF16, Hq=16, Hkv=2, D=128, block_size=16,
                             prior_lens=[300], new_lens=[40], seed=12)
    t = W.prefill_to_torch(c, "cuda")
    t["block_tables"][0, 3] = c.num_blocks + 5              # tokens 48..63 unreachable
    out = torch.full((c.T, c.Hq, c.D), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.pa_prefill(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                   t["query_start"], c.max_query_len, c.scale, c.max_context_len, err)
    torch.cuda.synchronize()
    assert int(err.item()) & ops.PA_DEV_BAD_BLOCK_ID
    assert torch.isfinite(out).all()


def _codes_like(pool, dtype, rng):
    """An FP8 code pool with the same filled rows as a 16-bit pool (random codes
    there, the NaN code where the 16-bit pool holds NaN)."""
    filled = ~np.isnan(W.storage_to_float64(pool, dtype)).any(axis=-1)
    codes = np.full(pool.shape, 0x7F, dtype=np.uint8)
    codes[filled] = W.random_e4m3_codes(rng, (int(filled.sum()), pool.shape[-1]))
    return codes


@pytest.mark.parametrize("k8,v8", [(True, True), (True, False), (False, True)])
@pytest.mark.parametrize("qdt,G,bs", [(W.BF16, 8, 16), (W.F16, 1, 32), (W.BF16, 4, 32),
                                      (W.F16, 16, 16)])
def test_prefill_over_fp8_and_mixed_pools(k8, v8, qdt, G, bs, prefill_kernel):
    if prefill_kernel == "multi-query":
        pytest.skip("FP8 pools run on the kernel with the query rows on M")
    rng = np.random.default_rng(G * 7 + bs + 3 * k8 + v8)
    c = W.build_prefill_case("pf-fp8", qdt, Hq=2 * G, Hkv=2, D=128, block_size=bs,
                             prior_lens=[0, 5, 130, 300], new_lens=[40, 1, 2 * bs + 3, 129],
                             seed=G * 10 + bs + qdt)
    kc = _codes_like(c.k_cache, qdt, rng) if k8 else c.k_cache
    vc = _codes_like(c.v_cache, qdt, rng) if v8 else c.v_cache
    ks, vs = float(np.float32(0.3)), float(np.float32(0.6))
    t = W.prefill_to_torch(c, "cuda")
    tk = torch.from_numpy(kc).cuda() if k8 else t["k_cache"]
    tv = torch.from_numpy(vc).cuda() if v8 else t["v_cache"]
    for out_dtype in (torch.float32, {W.BF16: torch.bfloat16, W.F16: torch.float16}[qdt]):
        out = torch.full((c.T, c.Hq, c.D), float("nan"), dtype=out_dtype, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ops.pa_prefill_kv(out, t["q"], tk, tv, ks, vs, t["block_tables"], t["context_lens"],
                          t["query_start"], c.max_query_len, c.scale, c.max_context_len, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        ref = oracle.prefill_mixed(c.q, qdt, kc, oracle.FP8 if k8 else qdt, ks, vc,
                                   oracle.FP8 if v8 else qdt, vs, c.block_tables, c.context_lens,
                                   c.query_start, c.scale)
        assert_attention_close(out, ref, qdt, f"k8={k8} v8={v8} G={G} out={out_dtype}")


def test_prefill_kv_refuses_an_fp32_query(prefill_kernel):
    q = torch.zeros(4, 8, 128, dtype=torch.float32, device="cuda")
    kc = torch.zeros(4, 16, 2, 128, dtype=torch.uint8, device="cuda")
    tables = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    lens = torch.full((1,), 4, dtype=torch.int32, device="cuda")
    qs = torch.tensor([0, 4], dtype=torch.int32, device="cuda")
    out = torch.zeros(4, 8, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(ops.PAError) as e:
        ops.pa_prefill_kv(out, q, kc, kc, 0.5, 0.5, tables, lens, qs, 4, 0.1, 64)
    assert e.value.status in (3, 4)
