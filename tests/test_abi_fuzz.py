"""Host-side robustness of the C ABI. For every entry point a consistent
argument list (fake but aligned device addresses) passes every host check and
reaches the launch, which fails with PA_ERR_CUDA because no device is visible;
thousands of copies with one to three arguments replaced by random sizes,
dtypes, scales or pointers (NULL, unaligned, never mapped) return a documented
pa_status and never crash, so no entry point reads through a caller pointer
on the host. Runs in a child process with CUDA_VISIBLE_DEVICES="", so nothing
can be launched. CPU only."""

from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import ctypes, random, sys
from paged_kv_cache_418_b200 import ops
L = ops.LIB
rng = random.Random(1234)
ptrs = [None, 16, 0x1000, 0x1001, 0x1008, 0x7f0000000000, 0x7f0000000004]
ints = [-7, -1, 0, 1, 2, 3, 4, 5, 8, 16, 24, 32, 64, 96, 128, 512, 4096, 1 << 20, 1 << 30]
floats = [float("nan"), float("inf"), -1.0, 0.0, 0.08838834764831845, 1.0]
sizes = [0, 1, 255, 1 << 20, 1 << 40]
A = [0x10000 * i for i in range(1, 16)]                 # distinct aligned fake addresses
# a consistent argument list per entry point (every check passes; only the launch
# can fail, and no device is visible)
BASE = {
    "pa_decode": [A[0], 2, A[1], A[2], A[3], 2, A[4], 64, A[5], 4, 32, 8, 128, 16, 256, 0.088,
                  1024, 0, A[6], 1 << 30, A[7], None],
    "pa_decode_static": [A[0], 2, A[1], A[2], A[3], 2, A[4], 64, A[5], 4, 32, 8, 128, 16, 256,
                         0.088, 1024, 0, A[7], None],
    "pa_decode_fp8": [A[0], 1, A[1], 1, A[2], A[3], 0.3, 0.7, A[4], 64, A[5], 4, 32, 32, 128, 16,
                      256, 0.088, 1024, 0, A[6], 1 << 30, A[7], None],
    "pa_reshape_and_cache": [A[0], A[1], A[2], A[3], 2, A[4], 4, 8, 128, 16, 256, A[7], None],
    "pa_reshape_and_cache_fp8": [A[0], A[1], 1, A[2], A[3], 0.3, 0.7, A[4], 4, 8, 128, 16, 256,
                                 A[7], None],
    "pa_copy_blocks": [A[0], A[1], 2, A[2], 3, 8, 128, 16, 256, A[7], None],
    "pa_swap_blocks": [A[0], A[1], A[2], A[3], 2, A[4], 3, 8, 128, 16, 256, 64, A[7], None],
    "pa_decode_shared_prefix": [A[0], 2, A[1], A[2], A[3], 2, A[4], 64, A[5], A[8], 2, A[9],
                                A[10], 16, 8, 32, 32, 8, 128, 16, 1024, 0.088, 1024, 0, A[6],
                                1 << 30, A[7], None],
    "pa_decode_kv": [A[0], 2, A[1], 2, A[2], 3, 0.3, A[3], 2, 1.0, A[4], 64, A[5], 4, 32, 8, 128,
                     16, 256, 0.088, 1024, 0, A[6], 1 << 30, A[7], None],
    "pa_reshape_and_cache_kv": [A[0], A[1], 2, A[2], 3, 0.3, A[3], 2, 1.0, A[4], 4, 8, 128, 16,
                                256, A[7], None],
    "pa_decode_shared_prefix_kv": [A[0], 2, A[1], 2, A[2], 3, 0.3, A[3], 3, 0.7, A[4], 64, A[5],
                                   A[8], 2, A[9], A[10], 16, 8, 32, 32, 8, 128, 16, 1024, 0.088,
                                   1024, 0, A[6], 1 << 30, A[7], None],
    "pa_prefill_kv": [A[0], 2, A[1], 2, A[2], 3, 0.3, A[3], 3, 0.7, A[4], 64, A[5], A[8], 2, 64, 32,
                      64, 8, 128, 16, 1024, 0.088, 1024, A[7], None],
    "pa_prefill": [A[0], 2, A[1], A[2], A[3], 2, A[4], 64, A[5], A[8], 2, 64, 32, 64, 8, 128, 16,
                   1024, 0.088, 1024, A[7], None],
}
def pick(t):
    if t is ctypes.c_void_p:
        return rng.choice(ptrs)
    if t is ctypes.c_float or t is ctypes.c_double:
        return rng.choice(floats)
    if t is ctypes.c_size_t:
        return rng.choice(sizes)
    return rng.choice(ints)
seen = {}
for name, base in BASE.items():
    fn = getattr(L, name)
    assert len(base) == len(fn.argtypes), name
    r0 = fn(*base)
    if r0 != 6:                                          # valid input reaches the launch
        print("BASE", name, r0)
        sys.exit(1)
    for _ in range(3000):
        args = list(base)
        for i in rng.sample(range(len(args)), rng.choice([1, 1, 2, 3])):
            args[i] = pick(fn.argtypes[i])
        r = fn(*args)
        if not 0 <= r <= 7:
            print("BAD", name, r, args)
            sys.exit(1)
        seen.setdefault(name, set()).add(r)
for name in ("pa_workspace_size", "pa_shared_prefix_workspace_size"):
    fn = getattr(L, name)
    for _ in range(3000):
        fn(*[pick(t) for t in fn.argtypes])
print("OK", {k: sorted(v) for k, v in seen.items()})
'''


@pytest.mark.skipif(torch.cuda.is_available(), reason="host-only check; run where no GPU is visible")
def test_random_arguments_never_crash_the_host_side():
    r = subprocess.run([sys.executable, "-c", CHILD], capture_output=True, text=True, cwd=ROOT,
                       timeout=600,
                       env=dict(os.environ, CUDA_VISIBLE_DEVICES="", PYTHONPATH=ROOT))
    assert r.returncode == 0, (r.returncode, r.stdout[-2000:], r.stderr[-2000:])
    assert r.stdout.strip().splitlines()[-1].startswith("OK"), r.stdout
