"""Shared-prefix (cascade) decode on the GPU against the fp64 oracle.

pa_decode_shared_prefix reads each group's shared blocks once for all its
members' queries and each sequence's own blocks once, then merges; its result
must be ordinary attention over every sequence's whole context, which the
oracle computes from the full block tables.
"""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200 import workloads as W
from pa_testlib import assert_attention_close, device_inputs, device_step, oracle_step, sample_rows

pytestmark = pytest.mark.gpu


def _groups_of(w):
    """Group arrays of a shared-prefix workload: its groups, all sharing prefix_blocks."""
    g, c = w.meta["groups"], w.meta["children"]
    pb = w.meta["prefix_blocks"]
    offsets = np.arange(0, g * c + 1, c, dtype=np.int32)
    members = np.arange(g * c, dtype=np.int32)
    shared = np.full(w.B, pb, dtype=np.int32)
    for k in range(g):
        rows = w.block_tables[k * c:(k + 1) * c, :pb]
        assert (rows == rows[0]).all()
    return offsets, members, shared, c, pb


def _run(w, offsets, members, shared, max_group, max_shared, out_dtype=torch.float32,
         partition_size=0, do_cache_ops=True):
    t = device_inputs(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if do_cache_ops:
        device_step(w, t=t, err=err, out_dtype=out_dtype)       # cache ops (and a plain decode)
    out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=out_dtype, device="cuda")
    ws = ops.shared_prefix_workspace_for(t["q"], t["k_cache"], w.max_context_len, max_shared,
                                         partition_size)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ops.pa_decode_shared_prefix(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                t["context_lens"], dev(shared), dev(offsets), dev(members),
                                max_group, max_shared, w.scale, w.max_context_len,
                                partition_size, ws, err)
    torch.cuda.synchronize()
    return out, err, t


@pytest.mark.parametrize("out_f32", [True, False])
def test_shrunk_sampling_workload(out_f32):
    w = W.shrink_workload(5, seed=515)
    offsets, members, shared, c, pb = _groups_of(w)
    out, err, _ = _run(w, offsets, members, shared, c, pb,
                       out_dtype=torch.float32 if out_f32 else torch.bfloat16)
    ref, _, _ = oracle_step(w)
    assert int(err.item()) == 0
    assert_attention_close(out, ref, w.dtype, "cascade")


def _random_groups_case(dtype, G, bs, sizes, shared_blocks, seed, Hkv=2, D=128):
    """Groups of sizes[k] members sharing shared_blocks[k] whole blocks, each member
    with its own tail of 1..3 blocks and a ragged last block."""
    rng = np.random.default_rng(seed)
    B = sum(sizes)
    tails = rng.integers(1, 3 * bs + 1, size=B)
    ctx = np.empty(B, dtype=np.int64)
    i = 0
    for k, n in enumerate(sizes):
        for _ in range(n):
            ctx[i] = shared_blocks[k] * bs + tails[i]
            i += 1
    nb = int(sum((c + bs - 1) // bs for c in ctx)) + 3      # room for an unshared layout too
    w = W.build_decode_case("groups", dtype, B=B, Hq=Hkv * G, Hkv=Hkv, D=D, block_size=bs,
                            num_blocks=nb, context_lens=ctx, seed=seed)
    # rebuild the tables so that each group's members share their leading blocks
    perm = rng.permutation(nb)
    used = 0
    MB = max(int((c + bs - 1) // bs) for c in ctx)
    tables = np.full((B, MB), -1, dtype=np.int32)
    kc = W.nan_fill(w.k_cache.shape, dtype)
    vc = W.nan_fill(w.v_cache.shape, dtype)
    i = 0
    for k, n in enumerate(sizes):
        pre = perm[used:used + shared_blocks[k]]
        used += shared_blocks[k]
        vals = lambda m: W.round_to_storage(rng.standard_normal((m, bs, Hkv, D)).astype(np.float32), dtype)
        kc[pre], vc[pre] = vals(len(pre)), vals(len(pre))
        for _ in range(n):
            own = (int(ctx[i]) - shared_blocks[k] * bs + bs - 1) // bs
            ids = perm[used:used + own]
            used += own
            kc[ids], vc[ids] = vals(own), vals(own)
            tables[i, :shared_blocks[k]] = pre
            tables[i, shared_blocks[k]:shared_blocks[k] + own] = ids
            i += 1
    w.k_cache, w.v_cache, w.block_tables, w.max_blocks = kc, vc, tables, MB
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    members = np.arange(B, dtype=np.int32)
    shared = np.concatenate([[s] * n for s, n in zip(shared_blocks, sizes)]).astype(np.int32)
    return w, offsets, members, shared


@pytest.mark.parametrize("dtype", [W.F16, W.BF16])
@pytest.mark.parametrize("G,bs", [(1, 16), (4, 16), (8, 32), (16, 16), (2, 32)])
def test_random_groups_match_the_oracle(dtype, G, bs):
    sizes = [1, 3, 17, 5, 2] if G <= 4 else [1, 3, 9, 2]
    shared = [0, 2, 21, 1, 9][:len(sizes)]
    w, offsets, members, sh = _random_groups_case(dtype, G, bs, sizes, shared,
                                                  seed=100 * G + bs + dtype)
    for psize in (0, bs * 2):
        out, err, _ = _run(w, offsets, members, sh, max(sizes), max(shared),
                           partition_size=psize, do_cache_ops=False)
        ref, _, _ = oracle_step(w, do_cache_ops=False)
        assert int(err.item()) == 0
        assert_attention_close(out, ref, dtype, f"G={G} bs={bs} psize={psize}")


def test_members_in_any_order_and_a_shared_prefix_longer_than_a_context():
    w, offsets, members, sh = _random_groups_case(W.BF16, 4, 16, [4, 3], [3, 2], seed=77)
    perm = np.random.default_rng(3).permutation(w.B).astype(np.int32)
    # same groups, members listed in another order and groups renumbered
    g_of = np.repeat(np.arange(2), [4, 3])
    members2 = np.concatenate([perm[np.isin(perm, np.where(g_of == 1)[0])],
                               perm[np.isin(perm, np.where(g_of == 0)[0])]]).astype(np.int32)
    offsets2 = np.array([0, 3, 7], dtype=np.int32)
    out, err, _ = _run(w, offsets2, members2, sh, 4, 3, do_cache_ops=False)
    ref, _, _ = oracle_step(w, do_cache_ops=False)
    assert int(err.item()) == 0
    assert_attention_close(out, ref, w.dtype, "reordered")
    # a sequence that claims more shared tokens than it holds is a bad context
    bad = sh.copy()
    w.context_lens[0] = 3 * 16 - 5
    bad[:4] = 3
    out, err, _ = _run(w, offsets, members, bad, 4, 3, do_cache_ops=False)
    assert int(err.item()) & ops.PA_DEV_BAD_CTX
    assert torch.equal(out[0].cpu(), torch.zeros_like(out[0].cpu()))


def test_full_size_sampling_workload_sampled_parity():
    w = W.make_workload(5)
    offsets, members, shared, c, pb = _groups_of(w)
    out, err, t = _run(w, offsets, members, shared, c, pb, out_dtype=torch.bfloat16)
    assert int(err.item()) == 0
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc, vc, w.block_mapping, w.dtype)
    oracle.reshape_and_cache(kc, vc, w.new_key, w.new_value, w.slot_mapping, w.dtype)
    rows = sample_rows(w, 48, seed=5)
    ref = oracle.decode(w.q, kc, vc, w.dtype, w.block_tables, w.context_lens, w.scale, rows=rows)
    got = out[torch.from_numpy(rows[:, 0]).long(), torch.from_numpy(rows[:, 1]).long()]
    assert_attention_close(got, ref, w.dtype, w.name)
    assert torch.isfinite(out.float()).all()


def _codes_like(pool, dtype, rng):
    """An FP8 code pool with the same filled rows as a 16-bit pool."""
    filled = ~np.isnan(W.storage_to_float64(pool, dtype)).any(axis=-1)
    codes = np.full(pool.shape, 0x7F, dtype=np.uint8)
    codes[filled] = W.random_e4m3_codes(rng, (int(filled.sum()), pool.shape[-1]))
    return codes


@pytest.mark.parametrize("k8,v8", [(True, True), (True, False), (False, True)])
def test_shared_prefix_over_fp8_and_mixed_pools(k8, v8):
    """Parallel sampling over an FP8 cache (and the mixed one): the pools after
    the step's cache ops, with codes in the FP8 pools, decoded with the shared
    prefix read once per group; the oracle decodes the same pools plainly."""
    rng = np.random.default_rng(70 + 2 * k8 + v8)
    w = W.shrink_workload(5, seed=517)
    offsets, members, shared, c, pb = _groups_of(w)
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc, vc, w.block_mapping, w.dtype)
    oracle.reshape_and_cache(kc, vc, w.new_key, w.new_value, w.slot_mapping, w.dtype)
    kp = _codes_like(kc, w.dtype, rng) if k8 else kc
    vp = _codes_like(vc, w.dtype, rng) if v8 else vc
    ks, vs = float(np.float32(0.4)), float(np.float32(0.9))
    t = device_inputs(w)
    el = lambda a, fp8: (torch.from_numpy(a).cuda() if fp8
                         else torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda())
    tk, tv = el(kp, k8), el(vp, v8)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ws = ops.shared_prefix_workspace_for(t["q"], tk, w.max_context_len, pb)
    ref = oracle.decode_mixed(w.q, w.dtype, kp, oracle.FP8 if k8 else w.dtype, ks, vp,
                              oracle.FP8 if v8 else w.dtype, vs, w.block_tables, w.context_lens,
                              w.scale)
    for out_dtype in (torch.float32, torch.bfloat16):
        out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=out_dtype, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ops.pa_decode_shared_prefix_kv(out, t["q"], tk, tv, ks, vs, t["block_tables"],
                                       t["context_lens"], dev(shared), dev(offsets), dev(members),
                                       c, pb, w.scale, w.max_context_len, 0, ws, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert_attention_close(out, ref, w.dtype, f"k8={k8} v8={v8} {out_dtype}")
