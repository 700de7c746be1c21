"""Host block manager: the exercise page's worked example plus invariants."""

import json
import os

import numpy as np
import pytest

import oracle
from paged_kv_cache_418_b200.block_manager import BlockManager


def test_worked_example_from_exercise_page(golden_dir):
    """The asserts of test_paged_attention_manager ("17. vLLM PagedAttention", Step 4)."""
    g = json.load(open(os.path.join(golden_dir, "block_manager_worked_example.json")))
    bm = BlockManager(g["num_blocks"], g["block_size"])
    seq = bm.allocate_prefill(1, g["prompt_len"])
    assert len(seq.block_table) == g["after_prefill"]["table_len"]
    assert bm.num_free() == g["after_prefill"]["free"]
    bm.append_token(1)                                   # length 7
    assert len(seq.block_table) == g["after_decode_to_len_7"]["table_len"]
    bm.append_token(1)                                   # length 8
    bm.append_token(1)                                   # length 9: crosses a block boundary
    assert seq.seq_len == 9
    assert len(seq.block_table) == g["after_decode_to_len_9"]["table_len"]
    assert bm.num_free() == g["after_decode_to_len_9"]["free"]
    # the page's pool is [num_blocks, block_size, head_dim]: one KV head here
    pool = np.zeros((g["num_blocks"], g["block_size"], 1, g["head_dim"]), dtype=np.float32)
    pool[seq.block_table[0], 0, 0, 0] = g["marker"]["value"]
    cache = oracle.gather(pool, oracle.F32, np.array(seq.block_table), seq.seq_len)[:, 0, :]
    assert list(cache.shape) == g["marker"]["gathered_shape"]
    r, c = g["marker"]["read_at"]
    assert cache[r, c] == g["marker"]["value"]
    bm.check_invariants()


def test_oom_is_runtime_error_and_allocates_nothing():
    bm = BlockManager(3, 4)
    bm.allocate_prefill(0, 8)
    with pytest.raises(RuntimeError, match="OOM"):
        bm.allocate_prefill(1, 5)            # needs 2, 1 free
    assert bm.num_free() == 1 and 1 not in bm.seqs
    bm.allocate_prefill(1, 4)
    with pytest.raises(RuntimeError, match="OOM"):
        bm.append_token(1)                   # length 5 needs a second block
    assert bm.seqs[1].seq_len == 4
    bm.check_invariants()


def test_block_size_one_allocates_every_token():
    """The exercise's `seq_len % block_size == 1` test never fires for bs=1."""
    bm = BlockManager(8, 1)
    bm.allocate_prefill(0, 2)
    for n in range(3, 7):
        slot, cow = bm.append_token(0)
        assert cow is None and len(bm.seqs[0].block_table) == n
        assert slot == bm.seqs[0].block_table[-1]
    bm.check_invariants()


def test_slots_follow_table_and_offset():
    bm = BlockManager(16, 4, free_order=[5, 9, 2, 7] + [i for i in range(16) if i not in (5, 9, 2, 7)])
    bm.allocate_prefill(0, 5)                 # blocks 5, 9; next pos 5 -> block 9 row 1
    slot, _ = bm.append_token(0)
    assert slot == 9 * 4 + 1
    for _ in range(2):
        bm.append_token(0)                    # positions 6, 7
    slot, _ = bm.append_token(0)              # position 8 -> new block 2, row 0
    assert slot == 2 * 4 + 0 and bm.seqs[0].block_table == [5, 9, 2]


def test_fork_shares_then_copy_on_write():
    bm = BlockManager(10, 4)
    bm.allocate_prefill(0, 6)                 # [0, 1], block 1 half full
    bm.fork(0, 1)
    bm.fork(0, 2)
    assert bm.ref_count[0] == 3 and bm.ref_count[1] == 3
    slot, cow = bm.append_token(1)            # writes into shared block 1 -> copy
    assert cow == (1, 2) and bm.seqs[1].block_table == [0, 2] and slot == 2 * 4 + 2
    assert bm.ref_count[1] == 2 and bm.ref_count[2] == 1
    slot, cow = bm.append_token(2)
    assert cow == (1, 3)
    slot, cow = bm.append_token(0)            # last holder writes in place
    assert cow is None and slot == 1 * 4 + 2 and bm.ref_count[1] == 1
    bm.check_invariants()
    for s in (0, 1, 2):
        bm.free(s)
    assert bm.num_free() == 10 and sum(bm.ref_count) == 0
    bm.check_invariants()


def test_full_block_boundary_fork_allocates_new_block_not_cow():
    bm = BlockManager(6, 4)
    bm.allocate_prefill(0, 8)                 # two full blocks
    bm.fork(0, 1)
    slot, cow = bm.append_token(1)
    assert cow is None and len(bm.seqs[1].block_table) == 3
    bm.check_invariants()


def test_random_lifecycle_keeps_invariants():
    rng = np.random.default_rng(7)
    bm = BlockManager(64, 4, rng.permutation(64))
    live = []
    nxt = 0
    for _ in range(400):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not live:
                bm.allocate_prefill(nxt, int(rng.integers(0, 13)))
                live.append(nxt)
                nxt += 1
            elif op == 1:
                bm.append_token(live[int(rng.integers(len(live)))])
            elif op == 2:
                bm.fork(live[int(rng.integers(len(live)))], nxt)
                live.append(nxt)
                nxt += 1
            else:
                s = live.pop(int(rng.integers(len(live))))
                bm.free(s)
        except RuntimeError:
            pass
        bm.check_invariants()
    for s in live:
        bm.free(s)
    assert bm.num_free() == 64
