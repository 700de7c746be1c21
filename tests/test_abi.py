"""The C-ABI library on a machine without a GPU: it loads, it exports every
function include/pa.h declares, and its host-side logic (argument checks,
launch planning, workspace sizing) behaves as documented. Nothing here
launches a kernel: every call below returns before any CUDA call."""

import ctypes
import os
import re

import pytest

from paged_kv_cache_418_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(pa_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("pa_decode", "pa_reshape_and_cache", "pa_copy_blocks", "pa_workspace_size",
              "pa_status_string", "pa_decode_plan"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(ops.LIB_PATH)
    for n in _declared_functions():
        assert hasattr(lib, n), n
        assert hasattr(ops, n), n           # the binding keeps the same names


def test_binding_scratch_size_matches_the_header():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    m = re.search(r"#define PA_STATIC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", src)
    assert m, "PA_STATIC_SCRATCH_BYTES not found in include/pa.h"
    a, b, c = (int(x) for x in m.groups())
    assert ops.PA_STATIC_SCRATCH_BYTES == a * b * c


def test_status_strings():
    assert ops.pa_status_string(0) == "ok"
    for s in range(1, 8):
        assert ops.pa_status_string(s) not in ("ok", "unknown status")
    assert ops.pa_status_string(99) == "unknown status"


def test_workspace_and_plan():
    # short contexts: one pass, no workspace
    assert ops.pa_workspace_size(64, 32, 32, 128, 512, 0) == 0
    assert ops.pa_decode_plan(1, 64, 32, 32, 128, 16, 512)[1:] == (1, 512)
    # long contexts on the CUDA-core kernel: 512-token partitions; workspace =
    # acc + m + l (fp32, 256 B aligned)
    k, P, psize = ops.pa_decode_plan(0, 8, 64, 8, 128, 32, 32768, 512)
    assert (k, P, psize) == (1, 64, 512)
    rows = 8 * 64 * 64
    up = lambda x: (x + 255) // 256 * 256
    assert ops.pa_workspace_size(8, 64, 8, 128, 32768, 512) == up(rows * 128 * 4) + 2 * up(rows * 4)
    # the tensor-core kernel splits the work over the SMs itself: no fixed partitions
    assert ops.pa_decode_plan(2, 8, 64, 8, 128, 32, 32768, 512) == (2, 1, 32768)
    # ... and needs its piece slots (2 per SM: 148 without a device) and tickets even
    # for short contexts
    assert ops.pa_workspace_size(8, 64, 8, 128, 100, 0) == \
        up(296 * 32 * 128 * 4) + 2 * up(296 * 32 * 4) + up(8 * 2 * 8)
    assert ops.pa_workspace_size(64, 32, 32, 128, 2048, 0) > 0
    assert ops.pa_decode_plan(1, 64, 32, 32, 128, 16, 2048)[1:] == (4, 512)
    assert ops.pa_workspace_size(0, 32, 32, 128, 2048, 0) == 0


@pytest.mark.parametrize("args,status", [
    (dict(D=96), 4), (dict(block_size=8), 4), (dict(Hq=24, Hkv=8), 4), (dict(Hq=30, Hkv=8), 4),
    (dict(dtype=5), 3), (dict(out_dtype=1, dtype=2), 3), (dict(partition_size=100), 2),
    (dict(B=-1), 2),
])
def test_decode_rejects_bad_arguments_before_launch(args, status):
    base = dict(out_dtype=0, dtype=2, B=2, Hq=8, Hkv=2, D=128, block_size=16, num_blocks=4,
                partition_size=0)
    base.update(args)
    rc = ops.LIB.pa_decode(16, base["out_dtype"], 16, 16, 16, base["dtype"], 16, 1, 16,
                           base["B"], base["Hq"], base["Hkv"], base["D"], base["block_size"],
                           base["num_blocks"], 0.1, 16, base["partition_size"], None, 0, None,
                           None)
    assert rc == status


def test_null_alignment_and_workspace_checks():
    L = ops.LIB
    # NULL query
    assert L.pa_decode(16, 0, None, 16, 16, 2, 16, 1, 16, 2, 8, 2, 128, 16, 4, 0.1, 16, 0,
                       None, 0, None, None) == 1
    # misaligned pool
    assert L.pa_decode(16, 0, 16, 24, 16, 2, 16, 1, 16, 2, 8, 2, 128, 16, 4, 0.1, 16, 0,
                       None, 0, None, None) == 7
    # split needed (max_context_len 4096) but no workspace
    assert L.pa_decode(16, 0, 16, 16, 16, 2, 16, 256, 16, 2, 8, 2, 128, 16, 4, 0.1, 4096, 0,
                       None, 0, None, None) == 5
    # B == 0 is a no-op
    assert L.pa_decode(None, 0, None, None, None, 2, None, 1, None, 0, 8, 2, 128, 16, 4, 0.1, 0,
                       0, None, 0, None, None) == 0
    assert L.pa_reshape_and_cache(16, 16, 16, 16, 2, 16, 0, 8, 128, 16, 4, None, None) == 0
    assert L.pa_reshape_and_cache(None, 16, 16, 16, 2, 16, 3, 8, 128, 16, 4, None, None) == 1
    assert L.pa_copy_blocks(16, 16, 2, 16, 0, 8, 128, 16, 4, None, None) == 0
    assert L.pa_copy_blocks(16, 16, 2, 16, -1, 8, 128, 16, 4, None, None) == 2
    assert L.pa_copy_blocks(16, 16, 7, 16, 1, 8, 128, 16, 4, None, None) == 3


def test_fp8_swap_prefill_and_shared_prefix_host_checks():
    L = ops.LIB
    # FP8 decode: bad query type, bad scale, NULL pool, B == 0 no-op
    assert L.pa_decode_fp8(16, 0, 16, 7, 16, 16, 1.0, 1.0, 16, 1, 16, 2, 8, 2, 128, 16, 4, 0.1,
                           16, 0, None, 0, None, None) == 3
    assert L.pa_decode_fp8(16, 0, 16, 1, 16, 16, 0.0, 1.0, 16, 1, 16, 2, 8, 2, 128, 16, 4, 0.1,
                           16, 0, None, 0, None, None) == 2
    assert L.pa_decode_fp8(16, 0, 16, 1, None, 16, 1.0, 1.0, 16, 1, 16, 2, 8, 2, 128, 16, 4, 0.1,
                           16, 0, None, 0, None, None) == 1
    assert L.pa_decode_fp8(None, 0, None, 1, None, None, 1.0, 1.0, None, 1, None, 0, 8, 2, 128,
                           16, 4, 0.1, 0, 0, None, 0, None, None) == 0
    # FP8 scatter: NaN scale, unsupported head size, misaligned source
    assert L.pa_reshape_and_cache_fp8(16, 16, 1, 16, 16, float("nan"), 1.0, 16, 2, 8, 128, 16, 4,
                                      None, None) == 2
    assert L.pa_reshape_and_cache_fp8(16, 16, 1, 16, 16, 1.0, 1.0, 16, 2, 8, 96, 16, 4,
                                      None, None) == 4
    assert L.pa_reshape_and_cache_fp8(24, 16, 1, 16, 16, 1.0, 1.0, 16, 2, 8, 128, 16, 4,
                                      None, None) == 7
    # swap: FP8 pools are allowed; an unknown type and negative pairs are not
    assert L.pa_swap_blocks(16, 16, 16, 16, 3, 16, 0, 8, 128, 16, 4, 4, None, None) == 0
    assert L.pa_swap_blocks(16, 16, 16, 16, 4, 16, 1, 8, 128, 16, 4, 4, None, None) == 3
    assert L.pa_swap_blocks(16, 16, 16, 16, 2, 16, -1, 8, 128, 16, 4, 4, None, None) == 2
    assert L.pa_swap_blocks(16, 16, None, 16, 2, 16, 1, 8, 128, 16, 4, 4, None, None) == 1
    # prefill: f32 and D = 64 are not on the tensor-core kernel; NULL start offsets
    assert L.pa_prefill(16, 0, 16, 16, 16, 0, 16, 1, 16, 16, 1, 4, 4, 8, 2, 128, 16, 4, 0.1, 16,
                        None, None) == 4
    assert L.pa_prefill(16, 0, 16, 16, 16, 2, 16, 1, 16, 16, 1, 4, 4, 8, 2, 64, 16, 4, 0.1, 16,
                        None, None) == 4
    assert L.pa_prefill(16, 0, 16, 16, 16, 2, 16, 1, 16, None, 1, 4, 4, 8, 2, 128, 16, 4, 0.1,
                        16, None, None) == 1
    assert L.pa_prefill(None, 0, None, None, None, 2, None, 1, None, None, 0, 0, 0, 8, 2, 128, 16,
                        4, 0.1, 16, None, None) == 0
    # shared prefix: more shared blocks than a table holds; NULL group arrays; no workspace
    assert L.pa_decode_shared_prefix(16, 0, 16, 16, 16, 2, 16, 4, 16, 16, 1, 16, 16, 2, 5, 2, 8,
                                     2, 128, 16, 4, 0.1, 64, 0, None, 0, None, None) == 2
    assert L.pa_decode_shared_prefix(16, 0, 16, 16, 16, 2, 16, 4, 16, 16, 1, None, 16, 2, 2, 2, 8,
                                     2, 128, 16, 4, 0.1, 64, 0, None, 0, None, None) == 1
    assert L.pa_decode_shared_prefix(16, 0, 16, 16, 16, 2, 16, 4, 16, 16, 1, 16, 16, 2, 2, 2, 8,
                                     2, 128, 16, 4, 0.1, 64, 0, None, 0, None, None) == 5


def test_shared_prefix_workspace_and_fp8_plan():
    # slots: one per 128-token tile of the largest shared prefix + the suffix partitions
    up = lambda x: (x + 255) // 256 * 256
    B, Hq, D = 256, 32, 128
    n = ops.pa_shared_prefix_workspace_size(B, Hq, 8, D, 1547, 0, 16, 64)
    P = 1024 // 128 + 4
    rows = B * Hq * P
    # + the tensor-core suffix pass's piece slots (2 per SM, 148 here) and tickets
    tc = up(296 * 16 * D * 4) + 2 * up(296 * 16 * 4) + up(B * 2 * 8)
    assert n == up(rows * D * 4) + 2 * up(rows * 4) + tc
    assert ops.pa_shared_prefix_workspace_size(B, Hq, 8, D, 1547, 0, 16, 0) == \
        ops.pa_workspace_size(B, Hq, 8, D, 1547, 0)
    # FP8 pools plan the tensor-core kernel on its GQA shapes (16-bit query), the
    # CUDA-core kernel elsewhere
    assert ops.pa_decode_plan(ops.PA_FP8_E4M3, 8, 64, 8, 128, 16, 4096)[0] == 2
    assert ops.pa_decode_plan(ops.PA_FP8_E4M3, 8, 32, 32, 128, 16, 4096)[0] == 1
