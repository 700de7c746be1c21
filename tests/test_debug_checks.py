"""Debug-mode precondition checks of the binding (host only): the cache ops'
caller errors that the library leaves unchecked on the device — two tokens on
one slot, a copy destination named twice or also used as a source — are
rejected before any launch. CPU only."""

from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch

from paged_kv_cache_418_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_slot_mapping_check():
    ops.check_slot_mapping(torch.tensor([3, -1, 7, -1, 0], dtype=torch.int64))   # padding may repeat
    with pytest.raises(ValueError, match="same slot"):
        ops.check_slot_mapping(torch.tensor([3, 5, 3], dtype=torch.int64))


def test_block_mapping_check():
    ops.check_block_mapping(torch.tensor([[1, 4], [2, 5]], dtype=torch.int64))
    with pytest.raises(ValueError, match="named twice"):
        ops.check_block_mapping(torch.tensor([[1, 4], [2, 4]], dtype=torch.int64))
    with pytest.raises(ValueError, match="also a source"):
        ops.check_block_mapping(torch.tensor([[1, 4], [4, 6]], dtype=torch.int64))
    # between two pools the same id on both sides is fine, duplicate destinations are not
    ops.check_block_mapping(torch.tensor([[4, 4], [6, 1]], dtype=torch.int64), same_pool=False)
    with pytest.raises(ValueError, match="named twice"):
        ops.check_block_mapping(torch.tensor([[4, 1], [6, 1]], dtype=torch.int64), same_pool=False)


def test_debug_mode_rejects_before_the_library_is_called():
    kc = torch.zeros(8, 4, 2, 16, dtype=torch.float16)
    vc = torch.zeros_like(kc)
    new = torch.zeros(3, 2, 16, dtype=torch.float16)
    was = ops.DEBUG
    ops.set_debug(True)
    try:
        with pytest.raises(ValueError):
            ops.pa_reshape_and_cache(new, new, kc, vc, torch.tensor([1, 1, 2], dtype=torch.int64))
        with pytest.raises(ValueError):
            ops.pa_reshape_and_cache_fp8(new, new, kc.view(torch.uint8)[..., :16], vc.view(torch.uint8)[..., :16],
                                         1.0, 1.0, torch.tensor([0, 5, 5], dtype=torch.int64))
        with pytest.raises(ValueError):
            ops.pa_copy_blocks(kc, vc, torch.tensor([[0, 3], [3, 5]], dtype=torch.int64))
        with pytest.raises(ValueError):
            ops.pa_swap_blocks(kc, vc, kc, vc, torch.tensor([[0, 3], [1, 3]], dtype=torch.int64))
    finally:
        ops.set_debug(was)


def test_debug_mode_from_the_environment():
    code = "from paged_kv_cache_418_b200 import ops; print(ops.DEBUG)"
    for val, want in (("1", "True"), ("0", "False")):
        r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                           env=dict(os.environ, PA_DEBUG=val, PYTHONPATH=ROOT), cwd=ROOT,
                           timeout=300)
        assert r.returncode == 0, r.stderr
        assert r.stdout.strip().endswith(want)
