"""Paged decode attention on the GPU against the fp64 oracle (through the C ABI)."""

import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200 import workloads as W
from pa_testlib import (ATOL, TORCH_DT, assert_attention_close, bits, device_inputs, device_step,
                        host_bits, oracle_step, sample_rows)

pytestmark = pytest.mark.gpu


def _both_kernels():
    """Run a test body under each decode kernel the planner can pick."""
    return ["auto", "simt"]


@pytest.fixture(params=_both_kernels())
def kernel_choice(request, monkeypatch):
    if request.param == "simt":
        monkeypatch.setenv("PA_DECODE_KERNEL", "simt")
    else:
        monkeypatch.delenv("PA_DECODE_KERNEL", raising=False)
    return request.param


# -- the tiny fp32 workload, whole -------------------------------------------------
def test_tiny_fp32_workload_full_parity():
    w = W.make_workload(1)
    out, t = device_step(w, out_dtype=torch.float32)
    ref, kc, vc = oracle_step(w)
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    assert_attention_close(out, ref, w.dtype, "tiny-fp32")
    assert torch.equal(bits(t["k_cache"]).cpu(), host_bits(kc))
    assert torch.equal(bits(t["v_cache"]).cpu(), host_bits(vc))


# -- reduced copies of the four large workloads, every output ---------------------
@pytest.mark.parametrize("which", [2, 3, 4, 5])
@pytest.mark.parametrize("out_f32", [True, False])
def test_shrunk_workloads_full_parity(which, out_f32, kernel_choice):
    w = W.shrink_workload(which, seed=100 + which)
    out, t = device_step(w, out_dtype=torch.float32 if out_f32 else None)
    ref, kc, vc = oracle_step(w)
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    assert_attention_close(out, ref, w.dtype, w.name)
    assert torch.equal(bits(t["k_cache"]).cpu(), host_bits(kc))
    assert torch.equal(bits(t["v_cache"]).cpu(), host_bits(vc))


# -- both load schedules of the CUDA-core kernel on the 16-bit and fp32 MHA shapes ----
@pytest.mark.parametrize("prefetch", ["0", "1"])
@pytest.mark.parametrize("which", [1, 2])
def test_cuda_core_load_schedules_agree_with_the_oracle(which, prefetch, monkeypatch):
    """The CUDA-core kernel with and without the next tile's loads in flight
    (the default differs by shape and pool type; both must be exact)."""
    monkeypatch.setenv("PA_SIMT_PREFETCH", prefetch)
    w = W.make_workload(1) if which == 1 else W.shrink_workload(which, seed=300 + which)
    out, t = device_step(w, out_dtype=torch.float32)
    ref, _, _ = oracle_step(w)
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    assert_attention_close(out, ref, w.dtype, f"{w.name} prefetch={prefetch}")


# -- every supported shape, ragged lengths across partition boundaries ------------
SHAPES = [(dt, D, bs, G) for dt in (W.F32, W.F16, W.BF16) for D in (64, 128) for bs in (16, 32)
          for G in (1, 2, 4, 8, 16)]


@pytest.mark.parametrize("dtype,D,bs,G", SHAPES)
def test_every_supported_shape(dtype, D, bs, G, kernel_choice):
    rng = np.random.default_rng(D * 7 + bs * 3 + G + dtype)
    Hkv = 2
    ctx = [1, bs - 1, bs, bs + 1, 2 * bs + 3, 37, 129, 200]
    nb = sum((c + bs - 1) // bs for c in ctx) + 5
    w = W.build_decode_case("shape-sweep", dtype, B=len(ctx), Hq=Hkv * G, Hkv=Hkv, D=D,
                            block_size=bs, num_blocks=nb, context_lens=ctx,
                            seed=int(rng.integers(1 << 30)))
    for psize in (0, bs, 2 * bs):
        out, t = device_step(w, out_dtype=torch.float32, partition_size=psize)
        ref, _, _ = oracle_step(w)
        torch.cuda.synchronize()
        assert int(t["err"].item()) == 0
        assert_attention_close(out, ref, dtype, f"psize={psize}")


@pytest.mark.parametrize("ctx", [[511, 512, 513], [1024, 1025, 1], [1535, 7, 2049]])
def test_default_partition_boundaries(ctx, kernel_choice):
    nb = sum((c + 15) // 16 for c in ctx) + 3
    w = W.build_decode_case("boundaries", W.BF16, B=len(ctx), Hq=32, Hkv=8, D=128,
                            block_size=16, num_blocks=nb, context_lens=ctx, seed=sum(ctx))
    out, t = device_step(w, out_dtype=torch.float32)
    ref, _, _ = oracle_step(w)
    assert int(t["err"].item()) == 0
    assert_attention_close(out, ref, w.dtype, str(ctx))


# -- closed forms and invariances, on the device -----------------------------------
def test_one_token_is_the_v_row_exactly(kernel_choice):
    w = W.build_decode_case("one-token", W.BF16, B=5, Hq=16, Hkv=2, D=128, block_size=16,
                            num_blocks=9, context_lens=[1] * 5, seed=3)
    out, t = device_step(w, out_dtype=torch.float32)
    nv = torch.from_numpy(W.storage_to_float64(w.new_value, w.dtype)).float()
    exp = nv.repeat_interleave(8, dim=1)        # query head hq reads KV head hq // 8
    assert torch.equal(out.cpu(), exp)


def test_relabelled_blocks_give_identical_bits(kernel_choice):
    w = W.shrink_workload(3, seed=77)
    out1, _ = device_step(w, out_dtype=torch.float32)
    rng = np.random.default_rng(1)
    pi = rng.permutation(w.num_blocks)
    w2 = W.shrink_workload(3, seed=77)
    for name in ("k_cache", "v_cache"):
        src = getattr(w2, name)
        dst = np.empty_like(src)
        dst[pi] = src
        setattr(w2, name, dst)
    w2.block_tables = np.where(w2.block_tables >= 0, pi[np.maximum(w2.block_tables, 0)],
                               -1).astype(np.int32)
    w2.slot_mapping = pi[w2.slot_mapping // w2.block_size] * w2.block_size + \
        w2.slot_mapping % w2.block_size
    out2, _ = device_step(w2, out_dtype=torch.float32)
    assert torch.equal(out1, out2)


def test_split_partials_match_the_oracle_partials(kernel_choice):
    ctx = [1300, 700, 40, 1537]
    nb = sum((c + 31) // 32 for c in ctx) + 2
    w = W.build_decode_case("partials", W.BF16, B=4, Hq=16, Hkv=2, D=128, block_size=32,
                            num_blocks=nb, context_lens=ctx, seed=9, k_boost_frac=0.05)
    psize = 256
    out, t = device_step(w, out_dtype=torch.float32, partition_size=psize)
    torch.cuda.synchronize()
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.reshape_and_cache(kc, vc, w.new_key, w.new_value, w.slot_mapping, w.dtype)
    o_ref, m_ref, l_ref, acc_ref = oracle.decode_partitioned(
        w.q, kc, vc, w.dtype, w.block_tables, w.context_lens, w.scale, psize)
    assert_attention_close(out, o_ref, w.dtype, "merged")
    B, Hq, D, P = w.B, w.Hq, w.D, m_ref.shape[2]
    rows = B * Hq * P
    up = lambda x: (x + 255) // 256 * 256
    ws = t["workspace"].cpu().numpy()
    # workspace layout: acc [B, P, Hq, D], then m and l [B, P, Hq]
    acc = ws[:rows * D * 4].view(np.float32).reshape(B, P, Hq, D).transpose(0, 2, 1, 3)
    m2 = ws[up(rows * D * 4):up(rows * D * 4) + rows * 4].view(np.float32).reshape(B, P, Hq)
    m2 = m2.transpose(0, 2, 1)
    l = ws[up(rows * D * 4) + up(rows * 4):][:rows * 4].view(np.float32).reshape(B, P, Hq)
    l = l.transpose(0, 2, 1)
    log2e = 1.0 / math.log(2.0)
    for b in range(B):
        nparts = -(-ctx[b] // psize)
        if nparts == 1:
            continue                                # written straight to the output
        for j in range(nparts):
            np.testing.assert_allclose(m2[b, :, j], m_ref[b, :, j] * log2e, rtol=1e-5, atol=1e-5)
            np.testing.assert_allclose(l[b, :, j], l_ref[b, :, j], rtol=1e-4)
            np.testing.assert_allclose(acc[b, :, j], acc_ref[b, :, j], rtol=1e-4, atol=1e-4)


# -- degenerate and erroneous inputs -----------------------------------------------
def test_empty_context_rows_are_zero_and_unflagged(kernel_choice):
    w = W.build_decode_case("empty", W.F16, B=3, Hq=8, Hkv=8, D=64, block_size=16,
                            num_blocks=8, context_lens=[5, 20, 3], seed=4)
    # no cache ops: attend the ctx-1 cached tokens, and none for sequence 1
    ctx = w.context_lens.copy() - 1
    ctx[1] = 0
    t = device_inputs(w)
    t["context_lens"].copy_(torch.from_numpy(ctx))
    out, t = device_step(w, t=t, out_dtype=torch.float32, do_cache_ops=False)
    ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.dtype, w.block_tables, ctx, w.scale)
    assert int(t["err"].item()) == 0
    assert torch.equal(out[1].cpu(), torch.zeros(8, 64))
    assert_attention_close(out, ref, w.dtype, "empty rows")


def test_empty_batch_is_a_noop():
    q = torch.empty(0, 8, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, 16, 2, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(0, 8, 128, dtype=torch.bfloat16, device="cuda")
    ops.pa_decode(out, q, kc, kc, torch.zeros(0, 1, dtype=torch.int32, device="cuda"),
                  torch.zeros(0, dtype=torch.int32, device="cuda"), 0.1, 0)


def test_bad_block_id_is_flagged_and_contained(kernel_choice):
    w = W.build_decode_case("bad-block", W.BF16, B=3, Hq=16, Hkv=2, D=128, block_size=16,
                            num_blocks=20, context_lens=[40, 40, 40], seed=5)
    t = device_inputs(w)
    t["block_tables"][1, 1] = w.num_blocks + 3        # out of range
    out, t = device_step(w, t=t, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert int(t["err"].item()) & ops.PA_DEV_BAD_BLOCK_ID
    ref, _, _ = oracle_step(w)
    assert torch.isfinite(out).all()
    assert_attention_close(out[[0, 2]], ref[[0, 2]], w.dtype, "untouched sequences")


def test_context_beyond_bound_is_flagged_and_zeroed(kernel_choice):
    w = W.build_decode_case("bad-ctx", W.BF16, B=2, Hq=8, Hkv=8, D=128, block_size=16,
                            num_blocks=10, context_lens=[30, 30], seed=6)
    t = device_inputs(w)
    t["context_lens"][0] = 100                        # > max_context_len (and > table)
    out, t = device_step(w, t=t, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert int(t["err"].item()) & ops.PA_DEV_BAD_CTX
    assert torch.equal(out[0].cpu(), torch.zeros(8, 128))
    ref, _, _ = oracle_step(w)
    assert_attention_close(out[1:], ref[1:], w.dtype, "other sequence")


def test_runs_on_a_side_stream(kernel_choice):
    w = W.shrink_workload(2, seed=8)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        t = device_inputs(w)
        out, t = device_step(w, t=t, out_dtype=torch.float32, stream=s)
    s.synchronize()
    ref, _, _ = oracle_step(w)
    assert_attention_close(out, ref, w.dtype, "side stream")


# -- the named workloads at full size, launched as the benchmark launches them -----
@pytest.fixture(scope="module")
def full_workloads():
    cache = {}

    def get(k):
        if k not in cache:
            cache.clear()
            cache[k] = W.make_workload(k)
        return cache[k]
    return get


@pytest.mark.parametrize("which", [2, 3, 4, 5])
def test_full_size_workload_sampled_parity(which, full_workloads):
    w = full_workloads(which)
    out, t = device_step(w)                            # output in the input type, as timed
    torch.cuda.synchronize()
    assert int(t["err"].item()) == 0
    # pools after the step: bit-exact against the oracle's copy + scatter
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    if len(w.block_mapping):
        oracle.copy_blocks(kc, vc, w.block_mapping, w.dtype)
    oracle.reshape_and_cache(kc, vc, w.new_key, w.new_value, w.slot_mapping, w.dtype)
    for got, exp in ((t["k_cache"], kc), (t["v_cache"], vc)):
        assert torch.equal(bits(got), host_bits(exp).to(got.device))
    del t
    rows = sample_rows(w, 48, seed=which)
    ref = oracle.decode(w.q, kc, vc, w.dtype, w.block_tables, w.context_lens, w.scale, rows=rows)
    got = out[torch.from_numpy(rows[:, 0]).long(), torch.from_numpy(rows[:, 1]).long()]
    assert_attention_close(got, ref, w.dtype, w.name)
    # every output finite (NaN poison never leaks)
    assert torch.isfinite(out.float()).all()


# -- the tensor-core kernel's even split of the work over the SMs -------------------
def _tc_case(ctx, seed, Hq=64, Hkv=8, bs=16):
    nb = sum((c + bs - 1) // bs for c in ctx) + 4
    w = W.build_decode_case("even-split", W.BF16, B=len(ctx), Hq=Hq, Hkv=Hkv, D=128,
                            block_size=bs, num_blocks=nb, context_lens=ctx, seed=seed,
                            k_boost_frac=0.02)
    assert ops.pa_decode_plan(w.kv_dtype, w.B, w.Hq, w.Hkv, w.D, w.block_size,
                              w.max_context_len)[0] == 2
    return w


def _decode_with(w, t, ws, out_dtype=torch.float32, mcl=None):
    out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=out_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.pa_decode(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                  w.scale, mcl or w.max_context_len, 0, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out


@pytest.mark.parametrize("ctx,G,mcl", [
    ([5000, 37, 1, 800, 4096, 33, 64, 3000] + [17] * 20 + [2049, 700], 8, None),  # many pieces
    ([9000, 12, 1], 4, None),                    # one sequence in pieces over ~70 CTAs
    ([1, 1, 1], 8, 4096),                        # fewer tiles than CTAs: empty shares between
    ([40, 1, 70], 4, 8192),                      # pieces with empty shares between them
    ([300 + 37 * i for i in range(150)], 4, None),   # many whole sequences per CTA
    ([0, 900, 0, 0, 17, 0, 2500] + [0, 33] * 12, 8, None),   # empty sequences between pairs
])
@pytest.mark.parametrize("pair_cost", [None, "0", "400"])
def test_even_split_pieces_merge_to_the_oracle(ctx, G, mcl, pair_cost, monkeypatch):
    """Sequences cut into pieces across CTAs (the last piece merges them), whole
    sequences in one CTA, CTAs with nothing to do; the workspace starts full of
    random bytes (tickets of no earlier call), and a second call on the same
    workspace gives the same bits. The split weighs each pair's start: with the
    default weight, with none (equal tile counts), and with a weight of 25
    tiles, under which shares also fall between two pairs' tiles."""
    if pair_cost is not None:
        monkeypatch.setenv("PA_TC_PAIR_COST", pair_cost)
    w = _tc_case([max(c, 1) for c in ctx], seed=len(ctx) * 31 + G, Hq=8 * G, Hkv=8)
    t = device_inputs(w)
    ops.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                             t["slot_mapping"])
    if min(ctx) == 0:           # empty sequences attend nothing (their new token stays unread)
        w.context_lens = np.array(ctx, dtype=w.context_lens.dtype)
        t["context_lens"].copy_(torch.from_numpy(w.context_lens))
    ws = ops.workspace_for(t["q"], t["k_cache"], mcl or w.max_context_len)
    ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8, device="cuda"))
    out1 = _decode_with(w, t, ws, mcl=mcl)
    out2 = _decode_with(w, t, ws, mcl=mcl)
    ref, _, _ = oracle_step(w)
    assert_attention_close(out1, ref, w.dtype, f"even split {len(ctx)} seqs")
    assert torch.equal(out1, out2)
    out3 = _decode_with(w, t, ws, out_dtype=torch.bfloat16, mcl=mcl)   # 16-bit output path
    assert_attention_close(out3, ref, w.dtype, "bf16 out")


def test_pipeline_wait_limit_runs_out_and_the_next_launch_is_correct(monkeypatch):
    """The tensor-core kernel's pipeline waits are bounded. Here one CTA's first
    query load is withheld, so the wait for it can only run out (after 1 ms):
    the launch reports PA_DEV_TIMEOUT (its outputs are unspecified), every CTA
    drains its own copies and products, frees tensor memory and returns; the
    next launch on the same stream, with the normal limit, matches the oracle."""
    w = _tc_case([700, 45, 1300], seed=5)
    t = device_inputs(w)
    ops.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                             t["slot_mapping"])
    ws = ops.workspace_for(t["q"], t["k_cache"], w.max_context_len)
    out = torch.zeros((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("PA_TC_WAIT_NS", "1000000")
    monkeypatch.setenv("PA_TC_TEST_WITHHOLD_Q", "1")
    ops.pa_decode(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                  w.scale, w.max_context_len, 0, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) & 16, "no wait ran out"
    monkeypatch.delenv("PA_TC_WAIT_NS")
    monkeypatch.delenv("PA_TC_TEST_WITHHOLD_Q")
    out = _decode_with(w, t, ws)
    ref, _, _ = oracle_step(w)
    assert_attention_close(out, ref, w.dtype, "after a timed-out launch")


def test_tensor_core_decode_replays_from_a_cuda_graph():
    """A captured call keeps its epoch; every replay must still merge its pieces
    (the merger leaves its ticket at zero for that epoch). Three replays of a
    graph holding the step's scatter and decode, each checked against the oracle."""
    w = _tc_case([5000, 37, 1, 800, 4096, 33, 64, 3000], seed=91)
    t = device_inputs(w)
    ws = ops.workspace_for(t["q"], t["k_cache"], w.max_context_len)
    out = torch.zeros((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                      # warm-up outside capture
        ops.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slot_mapping"], err)
        ops.pa_decode(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                      t["context_lens"], w.scale, w.max_context_len, 0, ws, err)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ops.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                                 t["slot_mapping"], err)
        ops.pa_decode(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                      t["context_lens"], w.scale, w.max_context_len, 0, ws, err)
    ref, _, _ = oracle_step(w)
    for rep in range(3):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert_attention_close(out, ref, w.dtype, f"replay {rep}")
