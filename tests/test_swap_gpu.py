"""swap_blocks on the GPU: whole blocks between the device pool and a pool in
page-locked host memory, bit-exact against the oracle's block copy."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200 import workloads as W
from pa_testlib import bits, host_bits

pytestmark = pytest.mark.gpu


def _pool(rng, nb, bs, hkv, d, dtype):
    if dtype == W.FP8:
        return W.random_e4m3_codes(rng, (nb, bs, hkv, d))
    return W.round_to_storage(rng.standard_normal((nb, bs, hkv, d)).astype(np.float32), dtype)


def _torch(a, device):
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a)
    return t.pin_memory() if device == "pinned" else t.to(device)


@pytest.mark.parametrize("dtype,Hkv,D,bs", [(W.F16, 32, 128, 16), (W.BF16, 8, 128, 32),
                                            (W.F32, 2, 64, 16), (W.FP8, 8, 128, 16)])
def test_swap_out_then_in_is_bit_exact(dtype, Hkv, D, bs):
    rng = np.random.default_rng(Hkv + D + bs + dtype)
    nd, nh = 48, 24                                   # device and host pool blocks
    dk, dv = _pool(rng, nd, bs, Hkv, D, dtype), _pool(rng, nd, bs, Hkv, D, dtype)
    hk, hv = _pool(rng, nh, bs, Hkv, D, dtype), _pool(rng, nh, bs, Hkv, D, dtype)
    out_pairs = np.stack([rng.choice(nd, 10, replace=False), rng.choice(nh, 10, replace=False)],
                         axis=1).astype(np.int64)
    in_pairs = np.stack([out_pairs[:6, 1], rng.choice(nd, 6, replace=False)],
                        axis=1).astype(np.int64)
    tdk, tdv = _torch(dk, "cuda"), _torch(dv, "cuda")
    thk, thv = _torch(hk, "pinned"), _torch(hv, "pinned")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # swap out: device -> host
    ops.pa_swap_blocks(thk, thv, tdk, tdv, torch.from_numpy(out_pairs).cuda(), err)
    torch.cuda.synchronize()
    oracle.swap_blocks(hk, hv, dk, dv, out_pairs)
    assert torch.equal(bits(thk), host_bits(hk)) and torch.equal(bits(thv), host_bits(hv))
    # swap in: host -> other device blocks
    ops.pa_swap_blocks(tdk, tdv, thk, thv, torch.from_numpy(in_pairs).cuda(), err)
    torch.cuda.synchronize()
    oracle.swap_blocks(dk, dv, hk, hv, in_pairs)
    assert int(err.item()) == 0
    assert torch.equal(bits(tdk).cpu(), host_bits(dk)) and torch.equal(bits(tdv).cpu(), host_bits(dv))


def test_swap_mapping_in_host_memory_and_bad_pairs():
    rng = np.random.default_rng(9)
    dk, dv = _pool(rng, 16, 16, 4, 64, W.BF16), _pool(rng, 16, 16, 4, 64, W.BF16)
    hk, hv = _pool(rng, 8, 16, 4, 64, W.BF16), _pool(rng, 8, 16, 4, 64, W.BF16)
    pairs = np.array([[3, 0], [15, 7], [16, 1], [2, 8], [-1, 2], [5, 3]], dtype=np.int64)
    tdk, tdv = _torch(dk, "cuda"), _torch(dv, "cuda")
    thk, thv = _torch(hk, "pinned"), _torch(hv, "pinned")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.pa_swap_blocks(thk, thv, tdk, tdv, torch.from_numpy(pairs).pin_memory(), err)
    torch.cuda.synchronize()
    assert int(err.item()) == ops.PA_DEV_BAD_PAIR
    good = pairs[[0, 1, 5]]
    oracle.swap_blocks(hk, hv, dk, dv, good)
    assert torch.equal(bits(thk), host_bits(hk)) and torch.equal(bits(thv), host_bits(hv))


def test_swap_of_nothing_and_host_errors():
    t = torch.zeros((4, 16, 2, 64), dtype=torch.float16, device="cuda")
    ops.pa_swap_blocks(t, t, t, t, torch.zeros((0, 2), dtype=torch.int64, device="cuda"))
    with pytest.raises(ops.PAError) as e:
        ops.pa_swap_blocks(t, t, t[..., :48].contiguous(), t, torch.zeros((1, 2), dtype=torch.int64,
                                                                         device="cuda"))
    assert e.value.status == 4           # head size 48 is not supported
