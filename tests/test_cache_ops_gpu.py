"""reshape_and_cache and copy_blocks on the GPU: bit-exact against the oracle."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200 import workloads as W
from pa_testlib import bits, device_inputs, host_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,Hkv,D,bs", [(W.F32, 4, 64, 16), (W.F16, 32, 128, 16),
                                            (W.BF16, 8, 128, 32), (W.BF16, 1, 64, 16)])
def test_reshape_and_cache_bit_exact(dtype, Hkv, D, bs):
    rng = np.random.default_rng(Hkv + D + bs)
    nb, T = 40, 57
    kc, vc = W.nan_fill((nb, bs, Hkv, D), dtype), W.nan_fill((nb, bs, Hkv, D), dtype)
    key = W.round_to_storage(rng.standard_normal((T, Hkv, D)).astype(np.float32), dtype)
    val = W.round_to_storage(rng.standard_normal((T, Hkv, D)).astype(np.float32), dtype)
    slots = rng.choice(nb * bs, size=T, replace=False).astype(np.int64)
    slots[::7] = -1                                       # padding tokens

    def dev(a):
        if a.dtype == np.uint16:                          # bf16 bit patterns
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(a).cuda()

    dk, dv = dev(kc), dev(vc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.pa_reshape_and_cache(dev(key), dev(val), dk, dv, torch.from_numpy(slots).cuda(), err)
    oracle.reshape_and_cache(kc, vc, key, val, slots, dtype)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(bits(dk).cpu(), host_bits(kc))
    assert torch.equal(bits(dv).cpu(), host_bits(vc))


def test_reshape_and_cache_out_of_range_slot_is_flagged_not_written():
    w = W.make_workload(1)
    t = device_inputs(w)
    before = bits(t["k_cache"]).clone()
    sm = t["slot_mapping"].clone()
    sm[2] = w.num_blocks * w.block_size                  # one past the pool
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"], sm, err)
    torch.cuda.synchronize()
    assert int(err.item()) == ops.PA_DEV_BAD_SLOT
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    good = np.array([0, 1, 3])
    oracle.reshape_and_cache(kc, vc, w.new_key[good], w.new_value[good], w.slot_mapping[good],
                             w.dtype)
    assert torch.equal(bits(t["k_cache"]).cpu(), host_bits(kc))
    assert not torch.equal(bits(t["k_cache"]), before)


@pytest.mark.parametrize("which", [1, 5])
def test_copy_blocks_bit_exact(which):
    w = W.make_workload(which) if which == 1 else W.shrink_workload(5, seed=11)
    t = device_inputs(w)
    if which == 1:                                        # tiny workload has no CoW: make some
        free = sorted(set(range(w.num_blocks)) - set(w.block_tables.ravel().tolist()))
        pairs = np.array([[int(w.block_tables[3, 0]), free[0]], [int(w.block_tables[1, 0]), free[1]]],
                         dtype=np.int64)
    else:
        pairs = w.block_mapping
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.pa_copy_blocks(t["k_cache"], t["v_cache"], torch.from_numpy(pairs).cuda(), err)
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc, vc, pairs, w.dtype)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and len(pairs) > 0
    assert torch.equal(bits(t["k_cache"]).cpu(), host_bits(kc))
    assert torch.equal(bits(t["v_cache"]).cpu(), host_bits(vc))


def test_copy_blocks_bad_pair_is_flagged_and_skipped():
    w = W.shrink_workload(5, seed=12)
    t = device_inputs(w)
    pairs = np.concatenate([w.block_mapping, [[0, w.num_blocks]]]).astype(np.int64)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.pa_copy_blocks(t["k_cache"], t["v_cache"], torch.from_numpy(pairs).cuda(), err)
    torch.cuda.synchronize()
    assert int(err.item()) == ops.PA_DEV_BAD_PAIR
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc, vc, w.block_mapping, w.dtype)
    assert torch.equal(bits(t["k_cache"]).cpu(), host_bits(kc))


def test_many_pairs_and_tokens():
    """More pairs than a grid's y/z extent (65535) would allow, and a long token list."""
    rng = np.random.default_rng(2)
    nb, bs, Hkv, D = 4096, 16, 1, 64
    kc = W.round_to_storage(rng.standard_normal((nb, bs, Hkv, D)).astype(np.float32), W.F16)
    vc = W.round_to_storage(rng.standard_normal((nb, bs, Hkv, D)).astype(np.float32), W.F16)
    perm = rng.permutation(nb)
    pairs = np.stack([perm[:2000], perm[2000:4000]], axis=1).astype(np.int64)
    dk, dv = torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda()
    ops.pa_copy_blocks(dk, dv, torch.from_numpy(pairs).cuda())
    oracle.copy_blocks(kc, vc, pairs, W.F16)
    T = 60000                                             # < num_blocks * bs slots
    key = W.round_to_storage(rng.standard_normal((T, Hkv, D)).astype(np.float32), W.F16)
    slots = rng.choice(nb * bs, size=T, replace=False).astype(np.int64)
    ops.pa_reshape_and_cache(torch.from_numpy(key).cuda(), torch.from_numpy(key).cuda(), dk, dv,
                             torch.from_numpy(slots).cuda())
    oracle.reshape_and_cache(kc, vc, key, key, slots, W.F16)
    torch.cuda.synchronize()
    assert torch.equal(bits(dk).cpu(), host_bits(kc)) and torch.equal(bits(dv).cpu(), host_bits(vc))
