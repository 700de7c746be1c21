"""The seeded workload generator: shapes, layouts, poison, step semantics."""

import json
import os

import numpy as np

import oracle
from paged_kv_cache_418_b200 import workloads as W


def _nan_rows(pool, dtype):
    return np.isnan(W.storage_to_float64(pool, dtype)).all(axis=(-1, -2))


def test_kv_bytes_match_llama2_7b_figures(golden_dir):
    """16 KiB per token per layer, 512 KiB over 32 layers, 1 GiB for 2048 tokens."""
    g = json.load(open(os.path.join(golden_dir, "llama2_7b_kv_sizes.json")))
    assert g["num_heads"] * g["head_dim"] == g["kv_dim_per_layer"]
    per_layer = W.kv_bytes_for([1], g["num_heads"], g["head_dim"], g["bytes_per_element_fp16"])
    assert per_layer == g["kv_bytes_per_token_per_layer"]
    assert per_layer * g["num_layers"] == g["kv_bytes_per_token_all_layers"]
    req = W.kv_bytes_for([g["context_tokens"]], g["num_heads"], g["head_dim"], 2) * g["num_layers"]
    assert req == g["kv_bytes_per_request"]


def test_tiny_workload_layout():
    w = W.make_workload(1)
    assert (w.B, w.Hq, w.Hkv, w.D, w.block_size, w.num_blocks) == (4, 4, 4, 64, 16, 64)
    assert list(w.context_lens) == [1, 15, 16, 33] and w.scale == 0.125
    bs = w.block_size
    # the step's tokens go to row ctx-1: rows 0, 14, 15, and row 0 of the third block
    assert [int(s) % bs for s in w.slot_mapping] == [0, 14, 15, 0]
    for b, n in enumerate(w.context_lens):
        nblk = (int(n) + bs - 1) // bs
        assert (w.block_tables[b, :nblk] >= 0).all() and (w.block_tables[b, nblk:] == -1).all()
        assert w.slot_mapping[b] // bs == w.block_tables[b, (int(n) - 1) // bs]
    used = set(int(x) for x in w.block_tables.ravel() if x >= 0)
    assert len(used) == sum((int(n) + bs - 1) // bs for n in w.context_lens)
    nan = _nan_rows(w.k_cache, w.dtype)
    for blk in range(w.num_blocks):
        if blk not in used:
            assert nan[blk].all()
    for b, n in enumerate(w.context_lens):
        s = int(w.slot_mapping[b])
        assert nan[s // bs, s % bs]                       # the slot to be written is poison
        g = oracle.gather(w.k_cache, w.dtype, w.block_tables[b], int(n) - 1)
        assert not np.isnan(g).any()                      # everything cached is real


def test_workloads_are_deterministic():
    a, b = W.make_workload(1), W.make_workload(1)
    for f in ("q", "k_cache", "v_cache", "block_tables", "slot_mapping", "new_key"):
        x, y = getattr(a, f), getattr(b, f)
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8))
    c = W.make_workload(1, seed=5)
    assert not np.array_equal(a.q, c.q)


def test_shared_prefix_step_semantics():
    w = W.shrink_workload(5, seed=3)
    groups, children = w.meta["groups"], w.meta["children"]
    bs, pre = w.block_size, w.meta["pre_tables"]
    assert w.B == groups * children and len(w.block_mapping) >= groups
    for g in range(groups):
        b0, b1 = g * children, g * children + 1
        plen = w.meta["parent_len"][g]
        assert w.context_lens[b0] == plen + 1 and w.context_lens[b1] == plen + 1
        # before the step children 0 and 1 share the partial block; child 0 copies it
        part = plen // bs
        assert pre[b0, part] == pre[b1, part]
        src, dst = pre[b0, part], w.block_tables[b0, part]
        assert [src, dst] in w.block_mapping.tolist()
        assert w.block_tables[b1, part] == src                       # child 1 writes in place
        assert w.slot_mapping[b1] == src * bs + plen % bs
        assert w.slot_mapping[b0] == dst * bs + plen % bs
        # the full prefix blocks are shared by every child of the group
        for c in range(children):
            assert np.array_equal(pre[b0 + c, :part], pre[b0, :part])
    # every child's cached rows are real values before the step, after the copies
    k, v = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(k, v, w.block_mapping, w.dtype)
    for b in range(w.B):
        n = int(w.context_lens[b]) - 1
        assert not np.isnan(oracle.gather(k, w.dtype, w.block_tables[b], n)).any()
        assert not np.isnan(oracle.gather(v, w.dtype, w.block_tables[b], n)).any()


def test_shrunk_shapes():
    for k in (2, 3, 4):
        w = W.shrink_workload(k, seed=1)
        full = {2: (32, 32, 128, 16, W.F16), 3: (64, 8, 128, 16, W.BF16),
                4: (64, 8, 128, 32, W.BF16)}[k]
        assert (w.Hq, w.Hkv, w.D, w.block_size, w.dtype) == full
        assert w.kv_bytes() == int(w.context_lens.sum()) * 2 * w.Hkv * w.D * 2


def _cached_rows(w, pool):
    """[tokens, Hkv, D] rows of every sequence's first ctx - 1 tokens (the cached part)."""
    bs = w.block_size
    out = []
    for b in range(w.B):
        n = int(w.context_lens[b]) - 1
        for t in range(n):
            out.append(pool[w.block_tables[b, t // bs], t % bs])
    return np.stack(out)


def test_length_recipes():
    # bounds are about 5 standard errors of 48 draws wide
    w2 = W.make_workload(2, batch=48)
    assert w2.context_lens.min() >= 128 and w2.context_lens.max() <= 2048
    assert 680 < float(w2.context_lens.mean()) < 1500               # U[128, 2048]: mean 1088
    w3 = W.make_workload(3, batch=48)
    assert w3.context_lens.min() >= 16 and w3.context_lens.max() <= 8192
    assert 450 < float(np.median(w3.context_lens)) < 2200             # LogNormal(ln 1200, 0.8)


def test_one_percent_of_k_rows_are_scaled_by_eight():
    w = W.make_workload(4, batch=1)
    assert list(w.context_lens) == [32768]
    k = W.storage_to_float64(_cached_rows(w, w.k_cache), w.dtype)    # [tokens, Hkv, D]
    norm = np.sqrt((k * k).sum(-1)).ravel()
    big = norm > 4.0 * np.median(norm)                                # N(0,1)·8 rows stand out
    n = norm.size
    assert abs(int(big.sum()) - 0.01 * n) < 5 * np.sqrt(0.01 * n)     # binomial, 5 sigma
    # a scaled row is exactly 8 times representable bf16 values (exact in bf16)
    rows = k.reshape(-1, w.D)[big]
    assert np.array_equal(W.storage_to_float64(W.round_to_storage(
        (rows / 8).astype(np.float32), w.dtype), w.dtype) * 8, rows)


def test_fp8_pool_codes_follow_the_recipe():
    w = W.make_workload(6, batch=4)
    assert w.fp8 and w.kv_dtype == W.FP8
    for pool in (w.k_cache, w.v_cache):
        codes = _cached_rows(w, pool).ravel()
        e = (codes >> 3) & 15
        assert e.min() >= 3 and e.max() <= 10                          # exponent field clipped
        assert not np.isin(codes, [0x7F, 0xFF]).any()                  # no NaN in cached data
        assert 0.4 < float((codes >> 7).mean()) < 0.6                  # both signs
