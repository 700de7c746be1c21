"""Pins of the fp64 oracle to things other than itself.

Each check is chosen so that a plausible mistake in the oracle (a wrong
gather index, a transposed head mapping, a sign or scale slip in the softmax,
a dropped merge term, a bad f16/bf16 decoding) fails at least one of them:

* library routines: torch's scaled_dot_product_attention (float64, with its
  own GQA grouping), numpy's float16 and torch's bfloat16 widening;
* closed forms: one token, zero query / zero scale, constant and shifted V,
  the large-scale limit (the arg-max row);
* an unshifted brute force (no max subtraction) on tiny inputs;
* invariance under any relabelling of physical blocks; one-block tables;
* the split/merge identity for any partition size;
* the worked examples printed on the pages (tests/golden).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_418_b200.workloads import (BF16, F16, F32, nan_fill, round_to_storage,
                                               storage_to_float64)

RNG = np.random.default_rng


def _paged_from_contiguous(kc_list, vc_list, bs, dtype, rng, extra_blocks=3):
    """Scatter per-sequence contiguous K/V ([ctx, Hkv, D] storage arrays) into a
    NaN-poisoned pool through a random permutation of block ids (block-wise
    reshapes, independent of the oracle's per-token gather)."""
    B = len(kc_list)
    hkv, d = kc_list[0].shape[1:]
    nblk = [(len(k) + bs - 1) // bs for k in kc_list]
    nb = sum(nblk) + extra_blocks
    perm = rng.permutation(nb)
    kp, vp = nan_fill((nb, bs, hkv, d), dtype), nan_fill((nb, bs, hkv, d), dtype)
    tables = np.full((B, max(max(nblk), 1)), -1, dtype=np.int32)
    used = 0
    for b in range(B):
        ids = perm[used:used + nblk[b]]
        used += nblk[b]
        tables[b, :nblk[b]] = ids
        n = len(kc_list[b])
        padk = nan_fill((nblk[b] * bs, hkv, d), dtype)
        padv = nan_fill((nblk[b] * bs, hkv, d), dtype)
        padk[:n], padv[:n] = kc_list[b], vc_list[b]
        kp[ids] = padk.reshape(nblk[b], bs, hkv, d)
        vp[ids] = padv.reshape(nblk[b], bs, hkv, d)
    return kp, vp, tables


def _rand(rng, shape, dtype, scale=1.0):
    return round_to_storage(rng.standard_normal(shape).astype(np.float32) * scale, dtype)


def _sdpa(q64, k64, v64, scale):
    """torch SDPA in float64: q [Hq, D], k/v [ctx, Hkv, D] -> [Hq, D]."""
    q = torch.from_numpy(q64)[None, :, None, :]
    k = torch.from_numpy(np.ascontiguousarray(k64.transpose(1, 0, 2)))[None]
    v = torch.from_numpy(np.ascontiguousarray(v64.transpose(1, 0, 2)))[None]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale,
                                                         enable_gqa=q.shape[1] != k.shape[1])
    return o[0, :, 0, :].numpy()


# -- element decoding ---------------------------------------------------------
def test_widen_f16_every_bit_pattern_matches_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.widen(bits.view(np.float16), oracle.F16)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    assert np.array_equal(ours[~nan], ref[~nan])


def test_widen_bf16_every_bit_pattern_matches_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.widen(bits, oracle.BF16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    assert np.array_equal(ours[~nan], ref[~nan])


# -- gather: the pages' worked examples ------------------------------------------
def test_gather_follows_the_block_table_example(golden_dir):
    """Block table 0->17, 1->42, 2->8 ("五十三" section 8), 16-token blocks."""
    g = json.load(open(os.path.join(golden_dir, "block_table_example.json")))
    bs, table = g["block_size"], np.array(g["logical_to_physical"], dtype=np.int32)
    nb = 64
    pool = np.zeros((nb, bs, 1, 2), dtype=np.float32)
    pool[:, :, 0, 0] = np.arange(nb)[:, None]          # each row knows its block
    pool[:, :, 0, 1] = np.arange(bs)[None, :]          # ... and its row in the block
    rows = oracle.gather(pool, oracle.F32, table, 40)[:, 0, :]
    # token 0 -> block 17 row 0; token 20 -> block 42 row 4; token 35 -> block 8 row 3
    assert tuple(rows[0]) == (17, 0) and tuple(rows[20]) == (42, 4) and tuple(rows[35]) == (8, 3)
    assert tuple(rows[15]) == (17, 15) and tuple(rows[16]) == (42, 0)


def test_gather_rejects_out_of_range_block():
    pool = np.zeros((4, 2, 1, 1), dtype=np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.gather(pool, oracle.F32, np.array([0, 4]), 3)
    with pytest.raises(oracle.OracleError):
        oracle.gather(pool, oracle.F32, np.array([0, -1]), 3)


# -- decode vs a library routine -------------------------------------------------
@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs", [(F32, 4, 4, 64, 16), (F16, 8, 2, 32, 4),
                                              (BF16, 8, 1, 16, 8), (BF16, 16, 2, 128, 16)])
def test_decode_matches_torch_sdpa(dtype, Hq, Hkv, D, bs):
    rng = RNG(11 + dtype + Hq)
    ctxs = [1, 5, bs, bs + 1, 3 * bs - 1, 37]
    kc = [_rand(rng, (n, Hkv, D), dtype) for n in ctxs]
    vc = [_rand(rng, (n, Hkv, D), dtype) for n in ctxs]
    kp, vp, tables = _paged_from_contiguous(kc, vc, bs, dtype, rng)
    q = _rand(rng, (len(ctxs), Hq, D), dtype)
    scale = 1.0 / math.sqrt(D)
    out = oracle.decode(q, kp, vp, dtype, tables, np.array(ctxs), scale)
    for b in range(len(ctxs)):
        ref = _sdpa(storage_to_float64(q[b], dtype), storage_to_float64(kc[b], dtype),
                    storage_to_float64(vc[b], dtype), scale)
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)


def test_decode_rows_subset_equals_full():
    rng = RNG(3)
    kc = [_rand(rng, (n, 2, 16), BF16) for n in (7, 30)]
    vc = [_rand(rng, (n, 2, 16), BF16) for n in (7, 30)]
    kp, vp, tables = _paged_from_contiguous(kc, vc, 8, BF16, rng)
    q = _rand(rng, (2, 6, 16), BF16)
    full = oracle.decode(q, kp, vp, BF16, tables, np.array([7, 30]), 0.25)
    rows = np.array([[1, 5], [0, 0], [1, 2]])
    sub = oracle.decode(q, kp, vp, BF16, tables, np.array([7, 30]), 0.25, rows=rows)
    for i, (b, h) in enumerate(rows):
        assert np.array_equal(sub[i], full[b, h])


# -- closed forms -------------------------------------------------------------------
@pytest.mark.parametrize("dtype", [F32, F16, BF16])
def test_one_token_returns_its_v_row_exactly(dtype):
    rng = RNG(5)
    kc = [_rand(rng, (1, 2, 32), dtype, 3.0) for _ in range(3)]
    vc = [_rand(rng, (1, 2, 32), dtype) for _ in range(3)]
    kp, vp, tables = _paged_from_contiguous(kc, vc, 4, dtype, rng)
    q = _rand(rng, (3, 4, 32), dtype, 5.0)
    out = oracle.decode(q, kp, vp, dtype, tables, np.ones(3), 0.17)
    for b in range(3):
        for hq in range(4):
            assert np.array_equal(out[b, hq], storage_to_float64(vc[b][0, hq // 2], dtype))


def test_zero_query_or_zero_scale_gives_mean_of_v():
    rng = RNG(6)
    n = 23
    kc, vc = [_rand(rng, (n, 1, 8), F32)], [_rand(rng, (n, 1, 8), F32)]
    kp, vp, tables = _paged_from_contiguous(kc, vc, 4, F32, rng)
    mean = vc[0][:, 0, :].astype(np.float64).mean(axis=0)
    q0 = np.zeros((1, 1, 8), dtype=np.float32)
    np.testing.assert_allclose(oracle.decode(q0, kp, vp, F32, tables, [n], 1.0)[0, 0], mean,
                               rtol=0, atol=1e-14)
    q = _rand(rng, (1, 1, 8), F32)
    np.testing.assert_allclose(oracle.decode(q, kp, vp, F32, tables, [n], 0.0)[0, 0], mean,
                               rtol=0, atol=1e-14)


def test_constant_and_shifted_v():
    rng = RNG(8)
    n, D = 19, 8
    k = _rand(rng, (n, 1, D), F32)
    c = rng.standard_normal(D).astype(np.float32)
    vconst = np.broadcast_to(c, (n, 1, D)).copy()
    # bf16-representable values in f32 storage, so that v + 0.5 is exact
    v = storage_to_float64(_rand(rng, (n, 1, D), BF16), BF16).astype(np.float32)
    q = _rand(rng, (1, 1, D), F32)
    kp, vp, t = _paged_from_contiguous([k], [vconst], 4, F32, RNG(1))
    np.testing.assert_allclose(oracle.decode(q, kp, vp, F32, t, [n], 0.5)[0, 0], c, atol=1e-14, rtol=0)
    kp1, vp1, t1 = _paged_from_contiguous([k], [v], 4, F32, RNG(2))
    kp2, vp2, t2 = _paged_from_contiguous([k], [v + np.float32(0.5)], 4, F32, RNG(2))
    o1 = oracle.decode(q, kp1, vp1, F32, t1, [n], 0.5)[0, 0]
    o2 = oracle.decode(q, kp2, vp2, F32, t2, [n], 0.5)[0, 0]
    np.testing.assert_allclose(o2, o1 + 0.5, rtol=0, atol=1e-14)


def test_large_scale_limit_picks_the_argmax_row():
    """softmax(scale * s) -> one-hot at arg max s; a sign slip picks the arg min."""
    rng = RNG(9)
    n, D = 40, 16
    k = _rand(rng, (n, 1, D), F32)
    v = _rand(rng, (n, 1, D), F32)
    q = _rand(rng, (1, 1, D), F32)
    kp, vp, t = _paged_from_contiguous([k], [v], 8, F32, rng)
    s = k[:, 0, :].astype(np.float64) @ q[0, 0].astype(np.float64)
    i = int(np.argmax(s))
    gap = np.sort(s)[-1] - np.sort(s)[-2]
    out = oracle.decode(q, kp, vp, F32, t, [n], 800.0 / gap)[0, 0]
    np.testing.assert_allclose(out, v[i, 0], rtol=0, atol=1e-12)


def test_unshifted_brute_force_on_tiny_inputs():
    """exp(s_i) without the max shift, summed with math.fsum, on small scores."""
    rng = RNG(10)
    for trial in range(20):
        bs = int(rng.choice([1, 2, 4]))
        n = int(rng.integers(1, 21))
        D = int(rng.integers(1, 9))
        Hkv, G = int(rng.integers(1, 3)), int(rng.integers(1, 3))
        k = _rand(rng, (n, Hkv, D), F32, 0.5)
        v = _rand(rng, (n, Hkv, D), F32)
        q = _rand(rng, (1, Hkv * G, D), F32, 0.5)
        kp, vp, t = _paged_from_contiguous([k], [v], bs, F32, rng)
        out = oracle.decode(q, kp, vp, F32, t, [n], 0.3)[0]
        for hq in range(Hkv * G):
            h = hq // G
            w = [math.exp(0.3 * math.fsum(float(q[0, hq, d]) * float(k[i, h, d]) for d in range(D)))
                 for i in range(n)]
            den = math.fsum(w)
            ref = [math.fsum(w[i] * float(v[i, h, d]) for i in range(n)) / den for d in range(D)]
            np.testing.assert_allclose(out[hq], ref, rtol=0, atol=1e-12)


def test_empty_context_is_zero():
    rng = RNG(12)
    kp = _rand(rng, (4, 4, 1, 8), F32)
    out = oracle.decode(_rand(rng, (2, 1, 8), F32), kp, kp, F32,
                        np.array([[0], [1]], dtype=np.int32), [0, 3], 1.0)
    assert np.array_equal(out[0, 0], np.zeros(8))


# -- paging invariances -------------------------------------------------------------
def test_relabelling_physical_blocks_is_bit_exact():
    rng = RNG(13)
    ctxs = [9, 33, 2]
    kc = [_rand(rng, (n, 2, 16), F16) for n in ctxs]
    vc = [_rand(rng, (n, 2, 16), F16) for n in ctxs]
    kp, vp, tables = _paged_from_contiguous(kc, vc, 4, F16, rng)
    q = _rand(rng, (3, 4, 16), F16)
    o1 = oracle.decode(q, kp, vp, F16, tables, ctxs, 0.25)
    pi = rng.permutation(kp.shape[0])          # block b moves to pi[b]
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[pi], vp2[pi] = kp, vp
    t2 = np.where(tables >= 0, pi[np.maximum(tables, 0)], -1).astype(np.int32)
    o2 = oracle.decode(q, kp2, vp2, F16, t2, ctxs, 0.25)
    assert np.array_equal(o1, o2)


def test_one_block_per_sequence_equals_unpaged_attention():
    rng = RNG(14)
    n = 27
    k, v = _rand(rng, (n, 2, 16), BF16), _rand(rng, (n, 2, 16), BF16)
    q = _rand(rng, (1, 4, 16), BF16)
    kp, vp = k.reshape(1, n, 2, 16), v.reshape(1, n, 2, 16)
    out = oracle.decode(q, kp, vp, BF16, np.zeros((1, 1), dtype=np.int32), [n], 0.25)[0]
    ref = _sdpa(storage_to_float64(q[0], BF16), storage_to_float64(k, BF16),
                storage_to_float64(v, BF16), 0.25)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


# -- split / merge ------------------------------------------------------------------
@pytest.mark.parametrize("psize", [1, 3, 8, 16, 64, 1000])
def test_partitioned_merge_equals_single_pass(psize):
    rng = RNG(15)
    ctxs = [1, 17, 64, 100]
    kc = [_rand(rng, (n, 2, 8), BF16, 2.0) for n in ctxs]
    vc = [_rand(rng, (n, 2, 8), BF16) for n in ctxs]
    kp, vp, tables = _paged_from_contiguous(kc, vc, 4, BF16, rng)
    q = _rand(rng, (4, 4, 8), BF16)
    ref = oracle.decode(q, kp, vp, BF16, tables, ctxs, 0.7)
    out, m, l, acc = oracle.decode_partitioned(q, kp, vp, BF16, tables, ctxs, 0.7, psize)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # partials: each partition's own max / sum / weighted sum, empty ones marked
    for b, n in enumerate(ctxs):
        for hq in range(4):
            k64 = storage_to_float64(kc[b][:, hq // 2], BF16)
            v64 = storage_to_float64(vc[b][:, hq // 2], BF16)
            s = 0.7 * (k64 @ storage_to_float64(q[b, hq], BF16))
            for j in range(m.shape[2]):
                lo, hi = j * psize, min((j + 1) * psize, n)
                if lo >= n:
                    assert m[b, hq, j] == -np.inf and l[b, hq, j] == 0.0
                    continue
                assert m[b, hq, j] == s[lo:hi].max()
                w = np.exp(s[lo:hi] - s[lo:hi].max())
                np.testing.assert_allclose(l[b, hq, j], w.sum(), rtol=1e-13)
                np.testing.assert_allclose(acc[b, hq, j], w @ v64[lo:hi], rtol=0, atol=1e-12)


# -- reshape_and_cache / copy_blocks ------------------------------------------------
def test_reshape_and_cache_writes_exactly_the_named_slots():
    rng = RNG(16)
    nb, bs, hkv, d = 6, 16, 2, 8
    kp, vp = nan_fill((nb, bs, hkv, d), BF16), nan_fill((nb, bs, hkv, d), BF16)
    key, val = _rand(rng, (4, hkv, d), BF16), _rand(rng, (4, hkv, d), BF16)
    slots = np.array([37, -1, 0, 95], dtype=np.int64)
    k0, v0 = kp.copy(), vp.copy()
    oracle.reshape_and_cache(kp, vp, key, val, slots, BF16)
    # slot 37 = block 2 row 5; slot 0 = block 0 row 0; slot 95 = block 5 row 15
    assert np.array_equal(kp[2, 5], key[0]) and np.array_equal(vp[2, 5], val[0])
    assert np.array_equal(kp[0, 0], key[2]) and np.array_equal(vp[5, 15], val[3])
    touched = np.zeros((nb, bs), dtype=bool)
    touched[2, 5] = touched[0, 0] = touched[5, 15] = True
    assert np.array_equal(kp[~touched], k0[~touched]) and np.array_equal(vp[~touched], v0[~touched])
    with pytest.raises(oracle.OracleError):
        oracle.reshape_and_cache(kp, vp, key[:1], val[:1], np.array([96]), BF16)


def test_reshape_then_one_token_decode_returns_written_row():
    rng = RNG(17)
    kp, vp = nan_fill((5, 4, 2, 8), F16), nan_fill((5, 4, 2, 8), F16)
    key, val = _rand(rng, (1, 2, 8), F16), _rand(rng, (1, 2, 8), F16)
    oracle.reshape_and_cache(kp, vp, key, val, np.array([3 * 4]), F16)
    out = oracle.decode(_rand(rng, (1, 4, 8), F16), kp, vp, F16,
                        np.array([[3]], dtype=np.int32), [1], 0.3)
    for hq in range(4):
        assert np.array_equal(out[0, hq], val[0, hq // 2].astype(np.float64))


def test_copy_blocks_copies_whole_blocks_from_a_snapshot():
    rng = RNG(18)
    kp, vp = _rand(rng, (8, 4, 2, 8), F32), _rand(rng, (8, 4, 2, 8), F32)
    k0, v0 = kp.copy(), vp.copy()
    pairs = np.array([[1, 5], [5, 6], [2, 7]], dtype=np.int64)   # 5 is a src and a dst
    oracle.copy_blocks(kp, vp, pairs, F32)
    assert np.array_equal(kp[5], k0[1]) and np.array_equal(vp[5], v0[1])
    assert np.array_equal(kp[6], k0[5]) and np.array_equal(vp[6], v0[5])   # old contents
    assert np.array_equal(kp[7], k0[2])
    for b in (0, 1, 2, 3, 4):
        assert np.array_equal(kp[b], k0[b]) and np.array_equal(vp[b], v0[b])
    with pytest.raises(oracle.OracleError):
        oracle.copy_blocks(kp, vp, np.array([[0, 8]]), F32)


# -- FP8 (E4M3) pools ------------------------------------------------------------
def _torch_e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def test_fp8_decoding_of_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    got, ref = oracle.widen(codes, oracle.FP8), _torch_e4m3_to_f64(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])
    assert np.isnan(got[[0x7F, 0xFF]]).all() and np.isnan(got).sum() == 2
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_fp8_encoding_matches_torch_rounding_in_range():
    rng = RNG(41)
    x = np.concatenate([rng.standard_normal(40000).astype(np.float32) * np.float32(s)
                        for s in (2.0 ** -12, 1e-3, 0.05, 1.0, 20.0, 150.0)])
    # exact midpoints between neighbouring codes (ties go to the even code)
    vals = oracle.widen(np.arange(0x7E, dtype=np.uint8), oracle.FP8)
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    x = x[np.abs(x) < 448]
    got = oracle.fp8_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_fp8_encoding_saturates_and_round_trips():
    special = np.array([448, 449, 463.9, 464, 1e6, np.inf, -448, -1e30, -np.inf, 0.0, -0.0,
                        2.0 ** -10, 2.0 ** -10 * 1.001, 3 * 2.0 ** -10], dtype=np.float32)
    assert oracle.fp8_encode(special).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE,
                                                    0xFE, 0xFE, 0x00, 0x80, 0x00, 0x01, 0x02]
    assert oracle.fp8_encode(np.array([np.nan], dtype=np.float32))[0] == 0x7F
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    back = oracle.fp8_encode(oracle.widen(finite, oracle.FP8).astype(np.float32))
    assert np.array_equal(back, finite)


def test_reshape_and_cache_fp8_quantises_the_named_slots():
    rng = RNG(42)
    nb, bs, hkv, d, T = 6, 16, 2, 32, 5
    ks, vs = np.float32(0.37), np.float32(0.005)          # V quotients reach past 448
    for src in (F32, F16, BF16):
        kp = np.full((nb, bs, hkv, d), 0x7F, dtype=np.uint8)
        vp = kp.copy()
        key = _rand(rng, (T, hkv, d), src, scale=3.0)
        val = _rand(rng, (T, hkv, d), src)
        slots = np.array([37, -1, 0, 95, 50], dtype=np.int64)
        oracle.reshape_and_cache_fp8(kp, vp, key, val, src, float(ks), float(vs), slots)
        # independent path: numpy float32 division, torch's E4M3 cast (saturation by clipping)
        kx = (storage_to_float64(key, src).astype(np.float32) / ks).clip(-448, 448)
        vx = (storage_to_float64(val, src).astype(np.float32) / vs).clip(-448, 448)
        kq = torch.from_numpy(kx).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        vq = torch.from_numpy(vx).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        touched = np.zeros((nb, bs), dtype=bool)
        for t, s in enumerate(slots):
            if s < 0:
                continue
            assert np.array_equal(kp[s // bs, s % bs], kq[t])
            assert np.array_equal(vp[s // bs, s % bs], vq[t])
            touched[s // bs, s % bs] = True
        assert (kp[~touched] == 0x7F).all() and (vp[~touched] == 0x7F).all()
        assert np.isin(vp[touched], [0x7E, 0xFE]).any()      # saturated codes occur
    with pytest.raises(oracle.OracleError):
        oracle.reshape_and_cache_fp8(kp, vp, key, val, F32, 0.0, 1.0, slots)


@pytest.mark.parametrize("qdt,Hq,Hkv,D,bs", [(F16, 8, 2, 32, 4), (BF16, 4, 4, 16, 8),
                                            (F32, 16, 2, 128, 16)])
def test_decode_kv_over_fp8_pools_matches_torch_sdpa(qdt, Hq, Hkv, D, bs):
    from paged_kv_cache_418_b200.workloads import random_e4m3_codes
    rng = RNG(43 + Hq + D)
    ctxs = [1, 7, bs, bs + 3, 40]
    kc = [random_e4m3_codes(rng, (n, Hkv, D)) for n in ctxs]
    vc = [random_e4m3_codes(rng, (n, Hkv, D)) for n in ctxs]
    # a paged layout of code pools (block-wise, NaN code in the gaps)
    nblk = [(n + bs - 1) // bs for n in ctxs]
    nb = sum(nblk) + 2
    perm = rng.permutation(nb)
    kp = np.full((nb, bs, Hkv, D), 0x7F, dtype=np.uint8)
    vp = kp.copy()
    tables = np.full((len(ctxs), max(nblk)), -1, dtype=np.int32)
    used = 0
    for b, n in enumerate(ctxs):
        ids = perm[used:used + nblk[b]]
        used += nblk[b]
        tables[b, :nblk[b]] = ids
        pk = np.full((nblk[b] * bs, Hkv, D), 0x7F, dtype=np.uint8)
        pv = pk.copy()
        pk[:n], pv[:n] = kc[b], vc[b]
        kp[ids], vp[ids] = pk.reshape(-1, bs, Hkv, D), pv.reshape(-1, bs, Hkv, D)
    q = _rand(rng, (len(ctxs), Hq, D), qdt)
    ks, vs, scale = float(np.float32(0.3)), float(np.float32(0.7)), 1.0 / math.sqrt(D)
    out = oracle.decode_kv(q, qdt, kp, vp, oracle.FP8, ks, vs, tables, np.array(ctxs), scale)
    for b in range(len(ctxs)):
        ref = _sdpa(storage_to_float64(q[b], qdt), _torch_e4m3_to_f64(kc[b]) * ks,
                    _torch_e4m3_to_f64(vc[b]) * vs, scale)
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)


def test_decode_kv_with_one_type_equals_decode():
    rng = RNG(44)
    kc = [_rand(rng, (n, 2, 16), BF16) for n in (3, 9)]
    vc = [_rand(rng, (n, 2, 16), BF16) for n in (3, 9)]
    kp, vp, tables = _paged_from_contiguous(kc, vc, 4, BF16, rng)
    q = _rand(rng, (2, 4, 16), BF16)
    a = oracle.decode(q, kp, vp, BF16, tables, [3, 9], 0.25)
    b = oracle.decode_kv(q, BF16, kp, vp, BF16, 1.0, 1.0, tables, [3, 9], 0.25)
    assert np.array_equal(a, b)


# -- one element type per pool (K in FP8, V in 16 bits, or the reverse) -------------
def _code_layout(rng, ctxs, bs, Hkv, D, k_fp8: bool, v_fp8: bool, dt):
    """Per-sequence contiguous K/V (FP8 codes or dt values) scattered block-wise
    into pools through a random permutation; empty slots hold NaN (0x7F for codes)."""
    from paged_kv_cache_418_b200.workloads import random_e4m3_codes
    mk = lambda fp8, n: (random_e4m3_codes(rng, (n, Hkv, D)) if fp8
                         else _rand(rng, (n, Hkv, D), dt))
    kc = [mk(k_fp8, n) for n in ctxs]
    vc = [mk(v_fp8, n) for n in ctxs]
    nblk = [(n + bs - 1) // bs for n in ctxs]
    nb = sum(nblk) + 2
    perm = rng.permutation(nb)
    kp = nan_fill((nb, bs, Hkv, D), oracle.FP8 if k_fp8 else dt)
    vp = nan_fill((nb, bs, Hkv, D), oracle.FP8 if v_fp8 else dt)
    tables = np.full((len(ctxs), max(nblk)), -1, dtype=np.int32)
    used = 0
    for b, n in enumerate(ctxs):
        ids = perm[used:used + nblk[b]]
        used += nblk[b]
        tables[b, :nblk[b]] = ids
        pk = nan_fill((nblk[b] * bs, Hkv, D), oracle.FP8 if k_fp8 else dt)
        pv = nan_fill((nblk[b] * bs, Hkv, D), oracle.FP8 if v_fp8 else dt)
        pk[:n], pv[:n] = kc[b], vc[b]
        kp[ids], vp[ids] = pk.reshape(-1, bs, Hkv, D), pv.reshape(-1, bs, Hkv, D)
    return kc, vc, kp, vp, tables


@pytest.mark.parametrize("k_fp8,v_fp8,dt,Hq,Hkv,D,bs", [
    (True, False, BF16, 8, 2, 32, 4),      # the explainer's K fp8 / V bf16
    (True, False, F16, 16, 2, 128, 16),
    (False, True, BF16, 4, 4, 16, 8),      # and the reverse
])
def test_decode_mixed_pool_types_match_torch_sdpa(k_fp8, v_fp8, dt, Hq, Hkv, D, bs):
    rng = RNG(61 + Hq + D)
    ctxs = [1, 7, bs, bs + 3, 40]
    kc, vc, kp, vp, tables = _code_layout(rng, ctxs, bs, Hkv, D, k_fp8, v_fp8, dt)
    q = _rand(rng, (len(ctxs), Hq, D), dt)
    ks, vs, scale = float(np.float32(0.3)), float(np.float32(0.7)), 1.0 / math.sqrt(D)
    kdt, vdt = (oracle.FP8 if k_fp8 else dt), (oracle.FP8 if v_fp8 else dt)
    out = oracle.decode_mixed(q, dt, kp, kdt, ks, vp, vdt, vs, tables, np.array(ctxs), scale)
    for b in range(len(ctxs)):
        k64 = _torch_e4m3_to_f64(kc[b]) * ks if k_fp8 else storage_to_float64(kc[b], dt)
        v64 = _torch_e4m3_to_f64(vc[b]) * vs if v_fp8 else storage_to_float64(vc[b], dt)
        ref = _sdpa(storage_to_float64(q[b], dt), k64, v64, scale)
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=1e-12)


def test_decode_mixed_with_one_type_equals_decode_kv():
    rng = RNG(62)
    for fp8, dt in ((True, F16), (False, BF16)):
        kc, vc, kp, vp, tables = _code_layout(rng, [3, 9, 17], 4, 2, 16, fp8, fp8, dt)
        q = _rand(rng, (3, 4, 16), dt)
        pdt = oracle.FP8 if fp8 else dt
        a = oracle.decode_kv(q, dt, kp, vp, pdt, 0.5, 0.25, tables, [3, 9, 17], 0.3)
        b = oracle.decode_mixed(q, dt, kp, pdt, 0.5, vp, pdt, 0.25, tables, [3, 9, 17], 0.3)
        assert np.array_equal(a, b)


def test_reshape_and_cache_mixed_quantises_one_pool_and_copies_the_other():
    rng = RNG(63)
    nb, bs, hkv, d, T = 6, 16, 2, 32, 5
    ks, vs = np.float32(0.37), np.float32(0.6)
    slots = np.array([37, -1, 0, 95, 50], dtype=np.int64)
    for src in (F16, BF16):
        key = _rand(rng, (T, hkv, d), src, scale=3.0)
        val = _rand(rng, (T, hkv, d), src)
        for k_fp8 in (True, False):
            kp = nan_fill((nb, bs, hkv, d), oracle.FP8 if k_fp8 else src)
            vp = nan_fill((nb, bs, hkv, d), src if k_fp8 else oracle.FP8)
            k0, v0 = kp.copy(), vp.copy()
            oracle.reshape_and_cache_mixed(kp, vp, key, val, src,
                                           oracle.FP8 if k_fp8 else src,
                                           src if k_fp8 else oracle.FP8, float(ks), float(vs),
                                           slots)
            q_src, q_pool, q_sc = (key, kp, ks) if k_fp8 else (val, vp, vs)
            c_src, c_pool = (val, vp) if k_fp8 else (key, kp)
            # the quantised pool: numpy float32 division, torch's E4M3 cast
            x = (storage_to_float64(q_src, src).astype(np.float32) / q_sc).clip(-448, 448)
            codes = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            touched = np.zeros((nb, bs), dtype=bool)
            for t, s in enumerate(slots):
                if s < 0:
                    continue
                assert np.array_equal(q_pool[s // bs, s % bs], codes[t])
                assert np.array_equal(c_pool[s // bs, s % bs].view(np.uint16),
                                      c_src[t].view(np.uint16))          # bit for bit
                touched[s // bs, s % bs] = True
            assert np.array_equal(kp[~touched].view(np.uint8), k0[~touched].view(np.uint8))
            assert np.array_equal(vp[~touched].view(np.uint8), v0[~touched].view(np.uint8))
    with pytest.raises(oracle.OracleError):             # a 16-bit pool of another type
        oracle.reshape_and_cache_mixed(nan_fill((nb, bs, hkv, d), oracle.FP8),
                                       nan_fill((nb, bs, hkv, d), F16), key, val, BF16,
                                       oracle.FP8, F16, 0.5, 0.5, slots)


@pytest.mark.parametrize("k_fp8,v_fp8", [(True, True), (True, False)])
def test_prefill_mixed_over_fp8_pools_matches_sdpa_with_a_causal_mask(k_fp8, v_fp8):
    rng = RNG(64)
    dt, Hq, Hkv, D, bs = BF16, 8, 2, 32, 4
    prior, new = [0, 5, 17], [7, 1, 9]
    ctxs = [p + n for p, n in zip(prior, new)]
    kc, vc, kp, vp, tables = _code_layout(rng, ctxs, bs, Hkv, D, k_fp8, v_fp8, dt)
    T = sum(new)
    q = _rand(rng, (T, Hq, D), dt)
    qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    ks, vs, scale = float(np.float32(0.4)), float(np.float32(0.9)), 1.0 / math.sqrt(D)
    kdt, vdt = (oracle.FP8 if k_fp8 else dt), (oracle.FP8 if v_fp8 else dt)
    out = oracle.prefill_mixed(q, dt, kp, kdt, ks, vp, vdt, vs, tables, np.array(ctxs), qs, scale)
    for b in range(3):
        n, ctx = new[b], ctxs[b]
        k64 = _torch_e4m3_to_f64(kc[b]) * ks if k_fp8 else storage_to_float64(kc[b], dt)
        v64 = _torch_e4m3_to_f64(vc[b]) * vs if v_fp8 else storage_to_float64(vc[b], dt)
        q64 = storage_to_float64(q[qs[b]:qs[b + 1]], dt)
        pos = ctx - n + np.arange(n)
        mask = torch.from_numpy(np.arange(ctx)[None, :] <= pos[:, None])
        qt = torch.from_numpy(np.ascontiguousarray(q64.transpose(1, 0, 2)))[None]
        kt = torch.from_numpy(np.ascontiguousarray(k64.transpose(1, 0, 2)))[None]
        vt = torch.from_numpy(np.ascontiguousarray(v64.transpose(1, 0, 2)))[None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=mask, scale=scale, enable_gqa=True)[0].numpy()
        got = out[qs[b]:qs[b + 1]].transpose(1, 0, 2)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


# -- swap_blocks ---------------------------------------------------------------------
def test_swap_blocks_moves_whole_blocks_between_pools():
    rng = RNG(45)
    src_k, src_v = _rand(rng, (9, 4, 2, 8), F16), _rand(rng, (9, 4, 2, 8), F16)
    dst_k, dst_v = _rand(rng, (5, 4, 2, 8), F16), _rand(rng, (5, 4, 2, 8), F16)
    d0k, d0v = dst_k.copy(), dst_v.copy()
    pairs = np.array([[8, 0], [3, 4], [3, 2]], dtype=np.int64)
    oracle.swap_blocks(dst_k, dst_v, src_k, src_v, pairs)
    for s, d in pairs:
        assert np.array_equal(dst_k[d], src_k[s]) and np.array_equal(dst_v[d], src_v[s])
    assert np.array_equal(dst_k[[1]], d0k[[1]]) and np.array_equal(dst_v[[1]], d0v[[1]])
    with pytest.raises(oracle.OracleError):
        oracle.swap_blocks(dst_k, dst_v, src_k, src_v, np.array([[9, 0]]))
    with pytest.raises(oracle.OracleError):
        oracle.swap_blocks(dst_k, dst_v, src_k, src_v, np.array([[0, 5]]))


# -- chunked prefill ---------------------------------------------------------------
@pytest.mark.parametrize("dtype,Hq,Hkv,D,bs", [(F16, 8, 2, 32, 4), (BF16, 4, 4, 16, 8),
                                              (F32, 6, 3, 64, 16)])
def test_prefill_matches_sdpa_with_a_bottom_right_causal_mask(dtype, Hq, Hkv, D, bs):
    from paged_kv_cache_418_b200.workloads import build_prefill_case
    c = build_prefill_case("pf", dtype, Hq, Hkv, D, bs, prior_lens=[0, 5, 17, 0],
                           new_lens=[7, 1, 9, 0], seed=50 + D)
    out = oracle.prefill(c.q, c.k_cache, c.v_cache, dtype, c.block_tables, c.context_lens,
                         c.query_start, c.scale)
    for b in range(c.B):
        n = int(c.query_start[b + 1] - c.query_start[b])
        if n == 0:
            continue
        ctx = int(c.context_lens[b])
        # contiguous K/V by block-wise reshape of the table's blocks (not per token)
        blk = c.block_tables[b, :(ctx + bs - 1) // bs]
        k64 = storage_to_float64(c.k_cache[blk].reshape(-1, Hkv, D)[:ctx], dtype)
        v64 = storage_to_float64(c.v_cache[blk].reshape(-1, Hkv, D)[:ctx], dtype)
        q64 = storage_to_float64(c.q[c.query_start[b]:c.query_start[b + 1]], dtype)
        pos = ctx - n + np.arange(n)
        mask = torch.from_numpy(np.arange(ctx)[None, :] <= pos[:, None])     # [n, ctx]
        qt = torch.from_numpy(np.ascontiguousarray(q64.transpose(1, 0, 2)))[None]
        kt = torch.from_numpy(np.ascontiguousarray(k64.transpose(1, 0, 2)))[None]
        vt = torch.from_numpy(np.ascontiguousarray(v64.transpose(1, 0, 2)))[None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=mask, scale=c.scale, enable_gqa=Hq != Hkv)[0].numpy()
        got = out[c.query_start[b]:c.query_start[b + 1]].transpose(1, 0, 2)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_prefill_first_token_of_an_empty_sequence_is_its_v_row():
    from paged_kv_cache_418_b200.workloads import build_prefill_case
    c = build_prefill_case("pf1", BF16, 8, 2, 16, 4, prior_lens=[0], new_lens=[5], seed=3)
    out = oracle.prefill(c.q, c.k_cache, c.v_cache, BF16, c.block_tables, c.context_lens,
                         c.query_start, c.scale)
    v0 = storage_to_float64(c.v_cache[c.block_tables[0, 0], 0], BF16)     # token 0, [Hkv, D]
    for hq in range(8):
        assert np.array_equal(out[0, hq], v0[hq // 4])
    with pytest.raises(oracle.OracleError):
        bad = c.context_lens.copy()
        bad[0] = 3                                   # fewer tokens than the chunk holds
        oracle.prefill(c.q, c.k_cache, c.v_cache, BF16, c.block_tables, bad, c.query_start, c.scale)


def test_prefill_row_ignores_keys_after_its_position():
    """Causality as an invariance: overwriting the K/V of every position after a
    new token's own leaves that token's output bit-identical, and the output of
    the chunk's last token (which sees everything) changes."""
    from paged_kv_cache_418_b200.workloads import build_prefill_case
    c = build_prefill_case("pf-causal", BF16, 8, 2, 32, 4, prior_lens=[6], new_lens=[9], seed=77)
    out = oracle.prefill(c.q, c.k_cache, c.v_cache, BF16, c.block_tables, c.context_lens,
                         c.query_start, c.scale)
    ctx, n, bs = int(c.context_lens[0]), 9, 4
    rng = RNG(5)
    for i in range(n - 1):                       # new token i sits at position ctx - n + i
        pos = ctx - n + i
        kc, vc = c.k_cache.copy(), c.v_cache.copy()
        for t in range(pos + 1, ctx):
            blk = c.block_tables[0, t // bs]
            kc[blk, t % bs] = _rand(rng, kc.shape[2:], BF16, 3.0)
            vc[blk, t % bs] = _rand(rng, vc.shape[2:], BF16, 3.0)
        out2 = oracle.prefill(c.q, kc, vc, BF16, c.block_tables, c.context_lens,
                              c.query_start, c.scale)
        assert np.array_equal(out2[:i + 1], out[:i + 1])
        assert not np.allclose(out2[n - 1], out[n - 1])


def test_oracle_result_does_not_depend_on_the_thread_count():
    """Each (sequence, head) row is computed alone, so one thread and many give
    the same bits (the CPU baseline may use either)."""
    threads = oracle.max_threads()
    rng = RNG(11)
    B, Hq, Hkv, D, bs = 5, 8, 2, 32, 4
    ctx = [1, 7, 13, 4, 9]
    kc = [_rand(rng, (n, Hkv, D), BF16) for n in ctx]
    vc = [_rand(rng, (n, Hkv, D), BF16) for n in ctx]
    kp, vp, tables = _paged_from_contiguous(kc, vc, bs, BF16, rng)
    q = _rand(rng, (B, Hq, D), BF16)
    cl = np.array(ctx, dtype=np.int32)
    one = oracle.decode(q, kp, vp, BF16, tables, cl, 0.2, n_threads=1)
    many = oracle.decode(q, kp, vp, BF16, tables, cl, 0.2, n_threads=4)
    assert np.array_equal(one, many)
    oracle.decode(q, kp, vp, BF16, tables, cl, 0.2, n_threads=threads)    # restore the pool size
    assert oracle.max_threads() == threads
