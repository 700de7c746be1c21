"""pa_decode_static: decode for callers that cannot allocate device memory.

Callers such as a plugin inside an engine that owns all device memory get
only their input and output buffers and may not allocate a workspace; this
entry point uses a scratch array built into the library instead. The test
calls it through the C ABI twice in a row (different sizes, both needing the
split pass, so the shared scratch is reused with the first call's leftovers
in it) and checks each result against pa_decode given a freshly allocated
workspace: the two run the same plan and the same kernels on the same inputs,
so the outputs must agree bit for bit; each is also checked against the
oracle at the parity tolerance of the other tests. This file is collected
last so that a failure here stops a -x run only after every other test has
run.
"""

import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200 import workloads as W
from pa_testlib import ATOL, device_inputs, oracle_step

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cases():
    # GQA bf16 with 512-token partitions (tensor-core path) and fp16 MHA with
    # contexts past one default partition (CUDA-core path)
    a = W.build_decode_case("static-gqa", W.BF16, B=3, Hq=32, Hkv=4, D=128, block_size=32,
                            num_blocks=200, context_lens=[1900, 700, 33], seed=41,
                            partition_size=512, k_boost_frac=0.01)
    b = W.build_decode_case("static-mha", W.F16, B=5, Hq=8, Hkv=8, D=128, block_size=16,
                            num_blocks=400, context_lens=[1200, 513, 5, 999, 1600], seed=42)
    return [a, b]


def _run(w, static: bool):
    t = device_inputs(w)
    out = torch.full((w.B, w.Hq, w.D), float("nan"), dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    # the step's new tokens first: decode attends them
    ops.pa_reshape_and_cache(t["new_key"], t["new_value"], t["k_cache"], t["v_cache"],
                             t["slot_mapping"], err)
    if static:
        ops.pa_decode_static(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                             t["context_lens"], w.scale, w.max_context_len, w.partition_size, err)
    else:
        ws = ops.workspace_for(t["q"], t["k_cache"], w.max_context_len, w.partition_size)
        assert ws is not None                    # both cases really use scratch
        ops.pa_decode(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                      t["context_lens"], w.scale, w.max_context_len, w.partition_size, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    o = out.cpu().numpy()
    assert np.isfinite(o).all(), w.name
    return o


def test_static_scratch_matches_workspace_entry_point_on_two_calls_in_a_row():
    cases = _cases()
    expected = [_run(w, static=False) for w in cases]
    for w, ref in zip(cases, expected):              # two calls in a row on the shared array
        got = _run(w, static=True)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), w.name
        oracle, _, _ = oracle_step(w)
        err = float(np.abs(got.astype(np.float64) - oracle).max())
        assert err <= ATOL[w.dtype], (w.name, err)


CHILD = r'''
import ctypes, sys
import numpy as np
import torch
from cuda.bindings import driver as cu
sys.path.insert(0, "tests")
from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200 import workloads as W
from pa_testlib import device_inputs

w = W.build_decode_case("ctx", W.BF16, B=2, Hq=32, Hkv=4, D=128, block_size=16,
                        num_blocks=120, context_lens=[1300, 40], seed=7, partition_size=512)
t = device_inputs(w)
def run(static):
    out = torch.zeros((w.B, w.Hq, w.D), dtype=torch.float32, device="cuda")
    if static:
        ops.pa_decode_static(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                             t["context_lens"], w.scale, w.max_context_len, w.partition_size)
    else:
        ws = ops.workspace_for(t["q"], t["k_cache"], w.max_context_len, w.partition_size)
        ops.pa_decode(out, t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                      t["context_lens"], w.scale, w.max_context_len, w.partition_size, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy()
ref = run(False)
first = run(True)                      # the primary context's address is found here
# a second context on the same device, current on this thread: host side only,
# an empty batch launches nothing but makes the library look the scratch up there
err, dev = cu.cuDeviceGet(0)
assert err == cu.CUresult.CUDA_SUCCESS, err
err, ctx2 = cu.cuCtxCreate(0, dev)
assert err == cu.CUresult.CUDA_SUCCESS, err
rc = ops.LIB.pa_decode_static(None, 2, None, None, None, 2, None, 1, None, 0, 32, 4, 128, 16,
                              1, 0.1, 0, 0, None, None)
err2, = cu.cuCtxPopCurrent()[:1]
err3, = cu.cuCtxDestroy(ctx2)[:1]
assert rc == 0, rc
assert err2 == cu.CUresult.CUDA_SUCCESS and err3 == cu.CUresult.CUDA_SUCCESS, (err2, err3)
again = run(True)                      # back in the primary context: its own address again
assert np.array_equal(first.view(np.uint32), ref.view(np.uint32))
assert np.array_equal(again.view(np.uint32), ref.view(np.uint32))
print("OK")
'''


def test_a_second_context_does_not_change_the_primary_contexts_scratch():
    """The scratch's device address belongs to one CUDA context: a call made
    while another context is current must not leave that context's address
    behind for later calls in the first one. Host side only in the second
    context (an empty batch), in a child process so its contexts end with it."""
    pytest.importorskip("cuda.bindings")
    r = subprocess.run([sys.executable, "-c", CHILD], capture_output=True, text=True, cwd=ROOT,
                       timeout=600, env=dict(os.environ, PYTHONPATH=ROOT))
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), (r.stdout[-2000:],
                                                                   r.stderr[-2000:])


def test_sizes_beyond_the_scratch_are_rejected_before_launch():
    # 64 sequences x 64 heads (no grouping: the CUDA-core split pass) x 128
    # partitions of 512 tokens needs ~270 MB of partials
    q = torch.zeros(64, 64, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, 16, 64, 128, dtype=torch.bfloat16, device="cuda")
    tables = torch.zeros(64, 4096, dtype=torch.int32, device="cuda")
    lens = torch.ones(64, dtype=torch.int32, device="cuda")
    out = torch.zeros(64, 64, 128, dtype=torch.bfloat16, device="cuda")
    assert ops.pa_decode_plan(ops.PA_BF16, 64, 64, 64, 128, 16, 65536, 512)[:2] == (1, 128)
    assert ops.pa_workspace_size(64, 64, 64, 128, 65536, 512) > ops.PA_STATIC_SCRATCH_BYTES
    with pytest.raises(ops.PAError) as e:
        ops.pa_decode_static(out, q, kc, kc, tables, lens, 0.1, 65536, 512)
    assert e.value.status == 5
