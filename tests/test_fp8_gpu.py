"""FP8 (E4M3) KV cache on the GPU, through the C ABI, against the fp64 oracle.

The pools hold E4M3 codes with one scale per pool; reshape_and_cache_fp8
quantises new rows (bit-exact against the oracle's quantiser) and
pa_decode_fp8 attends over code * scale (within the query type's bound).
"""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200 import workloads as W
from pa_testlib import (assert_attention_close, bits, device_inputs, device_step, host_bits,
                        oracle_step, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("out_f32", [True, False])
def test_shrunk_fp8_workload_full_parity(out_f32):
    w = W.shrink_workload(6, seed=606)
    out, t = device_step(w, out_dtype=torch.float32 if out_f32 else None)
    ref, kc, vc = oracle_step(w)
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    assert_attention_close(out, ref, w.dtype, w.name)
    assert torch.equal(t["k_cache"].cpu(), host_bits(kc))
    assert torch.equal(t["v_cache"].cpu(), host_bits(vc))


SHAPES = [(qdt, D, bs, G) for qdt in (W.F32, W.F16, W.BF16) for D in (64, 128) for bs in (16, 32)
          for G in (1, 2, 4, 8, 16)]


@pytest.mark.parametrize("qdt,D,bs,G", SHAPES)
def test_every_shape_over_fp8_pools(qdt, D, bs, G):
    rng = np.random.default_rng(D * 5 + bs * 3 + G + 11 * qdt)
    Hkv = 2
    ctx = [1, bs - 1, bs, bs + 1, 2 * bs + 3, 37, 129, 200]
    nb = sum((c + bs - 1) // bs for c in ctx) + 5
    w = W.build_decode_case("fp8-shape-sweep", qdt, B=len(ctx), Hq=Hkv * G, Hkv=Hkv, D=D,
                            block_size=bs, num_blocks=nb, context_lens=ctx,
                            seed=int(rng.integers(1 << 30)), kv_fp8=True)
    ref, _, _ = oracle_step(w)
    for psize in (0, bs, 2 * bs):
        out, t = device_step(w, out_dtype=torch.float32, partition_size=psize)
        torch.cuda.synchronize()
        assert int(t["err"].item()) == 0
        assert_attention_close(out, ref, qdt, f"psize={psize}")


@pytest.mark.parametrize("src,Hkv,D,bs", [(W.F32, 4, 64, 16), (W.F16, 32, 128, 16),
                                          (W.BF16, 8, 128, 32), (W.BF16, 1, 64, 16)])
def test_reshape_and_cache_fp8_bit_exact(src, Hkv, D, bs):
    rng = np.random.default_rng(Hkv * 3 + D + bs + src)
    nb, T = 40, 57
    kc = np.full((nb, bs, Hkv, D), 0x7F, dtype=np.uint8)
    vc = kc.copy()
    # K spans subnormal to saturating quotients; V is plain N(0, 1)
    mag = np.float32(2.0) ** rng.integers(-14, 11, size=(T, Hkv, 1)).astype(np.float32)
    key = W.round_to_storage(rng.standard_normal((T, Hkv, D)).astype(np.float32) * mag, src)
    val = W.round_to_storage(rng.standard_normal((T, Hkv, D)).astype(np.float32), src)
    slots = rng.choice(nb * bs, size=T, replace=False).astype(np.int64)
    slots[::7] = -1
    ks, vs = float(np.float32(0.173)), float(np.float32(0.0123))

    def dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(a).cuda()

    dk, dv = dev(kc), dev(vc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.pa_reshape_and_cache_fp8(dev(key), dev(val), dk, dv, ks, vs,
                                 torch.from_numpy(slots).cuda(), err)
    oracle.reshape_and_cache_fp8(kc, vc, key, val, src, ks, vs, slots)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(dk.cpu(), torch.from_numpy(kc))
    assert torch.equal(dv.cpu(), torch.from_numpy(vc))
    assert np.isin(kc, [0x7E, 0xFE]).any() and np.isin(kc & 0x78, [0]).any()  # saturated, subnormal


def test_fp8_entry_points_reject_bad_scales_before_launch():
    w = W.shrink_workload(6, seed=7, B=2, max_ctx=20)
    t = device_inputs(w)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    for ks, vs in ((0.0, 1.0), (1.0, -1.0), (float("inf"), 1.0), (1.0, float("nan"))):
        with pytest.raises(ops.PAError) as e:
            ops.pa_decode_fp8(out, t["q"], t["k_cache"], t["v_cache"], ks, vs, t["block_tables"],
                              t["context_lens"], w.scale, w.max_context_len)
        assert e.value.status == 2
        with pytest.raises(ops.PAError) as e:
            ops.pa_reshape_and_cache_fp8(t["new_key"], t["new_value"], t["k_cache"],
                                         t["v_cache"], ks, vs, t["slot_mapping"])
        assert e.value.status == 2


def test_fp8_one_token_is_the_scaled_v_row():
    w = W.build_decode_case("fp8-one-token", W.BF16, B=3, Hq=8, Hkv=2, D=128, block_size=16,
                            num_blocks=5, context_lens=[1] * 3, seed=5, kv_fp8=True)
    out, t = device_step(w, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _, kc, vc = oracle_step(w)
    v = oracle.widen(vc, oracle.FP8) * w.v_scale                      # exact in float64
    exp = np.stack([v[s // 16, s % 16] for s in w.slot_mapping])       # [B, Hkv, D]
    exp = np.repeat(exp, 4, axis=1).astype(np.float32)                 # hq reads KV head hq // 4
    # one token: p = 1, o = value(code) * v_scale, one fp32 product
    assert torch.equal(out.cpu(), torch.from_numpy(exp))


@pytest.mark.parametrize("which", [6, 8])
def test_full_size_fp8_workload_sampled_parity(which):
    """The FP8 workloads at full size as the benchmark launches them: the MHA
    batch (CUDA cores) and the Llama-3-70B-shaped GQA batch (tensor cores, every
    CTA walking dozens of tiles through the stage ring)."""
    w = W.make_workload(which)
    out, t = device_step(w)
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.reshape_and_cache_fp8(kc, vc, w.new_key, w.new_value, w.dtype, w.k_scale, w.v_scale,
                                 w.slot_mapping)
    for got, exp in ((t["k_cache"], kc), (t["v_cache"], vc)):
        assert torch.equal(got, torch.from_numpy(exp).to(got.device))
    del t
    rows = sample_rows(w, 48, seed=which)
    ref = oracle.decode_kv(w.q, w.dtype, kc, vc, oracle.FP8, w.k_scale, w.v_scale,
                           w.block_tables, w.context_lens, w.scale, rows=rows)
    got = out[torch.from_numpy(rows[:, 0]).long(), torch.from_numpy(rows[:, 1]).long()]
    assert_attention_close(got, ref, w.dtype, w.name)
    assert torch.isfinite(out.float()).all()


def test_every_finite_code_reaches_the_output_exactly():
    """One token per sequence: o = value(code) * v_scale, a single fp32 product, for
    every finite E4M3 code (subnormals and +-448 included) on the V path."""
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    D, Hkv, B = 128, 1, 2
    w = W.build_decode_case("fp8-all-codes", W.F32, B=B, Hq=Hkv, Hkv=Hkv, D=D, block_size=16,
                            num_blocks=4, context_lens=[2] * B, seed=12, kv_fp8=True,
                            v_scale=0.37)
    # token 0 of each sequence carries the codes in V; token 1 (the new one) is
    # masked out by a query/key pair that gives it weight exactly 0 in fp32
    codes = np.concatenate([finite, finite[:2 * D - len(finite)]]).reshape(B, Hkv, D)
    for b in range(B):
        blk = w.block_tables[b, 0]
        w.v_cache[blk, 0] = codes[b]
        w.k_cache[blk, 0] = 0x00                               # k0 = 0: score 0
    w.q[:] = 1.0
    w.new_key[:] = -1e4                                        # k1 * q very negative: weight 0
    out, t = device_step(w, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    exp = (oracle.widen(codes, oracle.FP8) * w.v_scale).astype(np.float32)
    assert torch.equal(out.cpu(), torch.from_numpy(exp))


def test_heavy_tailed_codes_within_derived_bound():
    """Codes over the whole E4M3 range (values up to 448 times the scale). The
    kernel's scores are fp32 dot products: each is within D * 2^-24 * scale *
    sum_d |q_d k_d| of exact, and a score error e moves a softmax average by at
    most 2 e max|v| (plus fp32 rounding of the average itself)."""
    rng = np.random.default_rng(21)
    ctx = [3, 17, 40, 100]
    nb = sum((c + 15) // 16 for c in ctx) + 2
    w = W.build_decode_case("fp8-heavy", W.F32, B=4, Hq=8, Hkv=2, D=64, block_size=16,
                            num_blocks=nb, context_lens=ctx, seed=22, kv_fp8=True)
    for name in ("k_cache", "v_cache"):
        pool = getattr(w, name)
        filled = pool != 0x7F
        pool[filled] = W.random_e4m3_codes(rng, int(filled.sum()), lo=0, hi=15)
    out, t = device_step(w, out_dtype=torch.float32)
    ref, kc, vc = oracle_step(w)
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    got = out.cpu().numpy().astype(np.float64)
    G, D = w.Hq // w.Hkv, w.D
    for b in range(w.B):
        n = int(w.context_lens[b])
        rows = [(w.block_tables[b, i // 16], i % 16) for i in range(n)]
        kv = np.stack([oracle.widen(kc[r], oracle.FP8) for r in rows]) * w.k_scale   # [n, Hkv, D]
        vv = np.stack([oracle.widen(vc[r], oracle.FP8) for r in rows]) * w.v_scale
        for hq in range(w.Hq):
            h = hq // G
            qa = np.abs(w.q[b, hq].astype(np.float64))
            smax = w.scale * (np.abs(kv[:, h]) @ qa).max()
            vmax = np.abs(vv[:, h]).max()
            bound = 2.0 * vmax * (2.0 * D * 2.0 ** -24 * smax) + 1e-5 * max(1.0, vmax)
            err = np.abs(got[b, hq] - ref[b, hq]).max()
            assert err <= bound, (b, hq, err, bound)
