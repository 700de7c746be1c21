"""pa_decode_static: decode for callers that cannot allocate device memory.

Callers such as a plugin inside an engine that owns all device memory get
only their input and output buffers and may not allocate a workspace; this
entry point uses a scratch array built into the library instead. The test
calls it through the C ABI twice in a row (different sizes, both needing the
split pass, so the shared scratch is reused with the first call's leftovers
in it) and checks each result against pa_decode given a freshly allocated
workspace, within the parity tolerance of the other tests. This file is
collected last so that a failure here stops a -x run only after every other
test has run.
"""

import numpy as np
import pytest
import torch

from paged_kv_cache_418_b200 import ops
from paged_kv_cache_418_b200 import workloads as W
from pa_testlib import ATOL, device_inputs

pytestmark = pytest.mark.gpu


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
        err = float(np.abs(got.astype(np.float64) - ref).max())
        assert np.isfinite(got).all() and err <= ATOL[w.dtype], (w.name, err)


def test_sizes_beyond_the_scratch_are_rejected_before_launch():
    # 64 sequences x 64 heads x 128 partitions of 512 tokens needs ~270 MB of partials
    q = torch.zeros(64, 64, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, 16, 8, 128, dtype=torch.bfloat16, device="cuda")
    tables = torch.zeros(64, 4096, dtype=torch.int32, device="cuda")
    lens = torch.ones(64, dtype=torch.int32, device="cuda")
    out = torch.zeros(64, 64, 128, dtype=torch.bfloat16, device="cuda")
    assert ops.pa_workspace_size(64, 64, 8, 128, 65536, 512) > ops.PA_STATIC_SCRATCH_BYTES
    with pytest.raises(ops.PAError) as e:
        ops.pa_decode_static(out, q, kc, kc, tables, lens, 0.1, 65536, 512)
    assert e.value.status == 5
