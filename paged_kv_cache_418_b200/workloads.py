"""Seeded synthetic workloads for paged decode attention.

This module only makes inputs: paged K/V pools, block tables, context
lengths, query vectors, the new tokens of one decode step with their slot
mapping, and the copy-on-write pairs of that step. It holds none of the
attention arithmetic. Both the CPU oracle (in the tests) and the CUDA path
consume exactly the arrays it returns.

Value recipe (all workloads)
  * One ``numpy.random.Generator(PCG64(seed))`` per workload; draws happen in
    a fixed order: layout (lengths, free-list shuffle), then the query, then
    each sequence's cached K and V rows, then the step's new K and V rows.
  * Values are N(0, 1) drawn in float32 and rounded to nearest-even into the
    storage type (f32, f16 or bf16). Both sides read these rounded values.
  * Pool slots that hold no token (free blocks, the unused tail of each
    sequence's last block, and the slots the step is about to write) are
    NaN, so a kernel that reads outside what it should shows it in its output.
  * Unused block-table entries are -1.
  * FP8 pools (E4M3 codes, one byte each) are drawn as bit fields, not by
    quantising anything: sign ~ U{0,1}, exponent field ~ round(N(7, 1))
    clipped to [3, 10], fraction ~ U{0..7}, so cached values lie in
    [2^-4, 16) in magnitude, around 1, before the pool's scale (like the
    N(0, 1) values of the 16-bit pools). Empty slots hold the NaN code 0x7F. The new K/V rows of the step
    stay N(0, 1) in the query's type: reshape_and_cache_fp8 quantises them.

Layout recipe
  * Physical blocks come from a ``BlockManager`` whose free list is a seeded
    permutation of the pool, so tables are non-contiguous, as in the block
    table example of "五十三：vLLM-PagedAttention" section 8 (logical 0 -> 17,
    1 -> 42, 2 -> 8).
  * Each sequence is prefilled with ``ctx - 1`` tokens; the step appends one
    token per sequence (``reshape_and_cache`` input) and decode then attends
    over all ``ctx`` tokens, the new one included.

The five named workloads mirror the decode batches the pages talk about: a
tiny fp32 case, a Llama-2-7B-shaped batch (32 heads x 128, fp16, the KV size
arithmetic of "vLLM 与 LLM 推理部署实战" section 1), a Llama-3-70B-shaped GQA
batch (64 query heads over 8 KV heads), a long-context batch that needs the
split-context pass, and parallel sampling over a shared prefix ("五十三" section
17; copy-on-write of "vLLM 与 LLM 推理部署实战" section 2.2).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence as Seq

import numpy as np

from .block_manager import BlockManager

F32, F16, BF16, FP8 = 0, 1, 2, 3
DTYPE_NAMES = {F32: "f32", F16: "f16", BF16: "bf16", FP8: "fp8e4m3"}
ESIZE = {F32: 4, F16: 2, BF16: 2, FP8: 1}
_STORAGE = {F32: np.float32, F16: np.float16, BF16: np.uint16, FP8: np.uint8}
_NAN_BITS = {F16: 0x7E00, BF16: 0x7FC0, FP8: 0x7F}


def round_to_storage(x: np.ndarray, dtype: int) -> np.ndarray:
    """Round float32 values to nearest-even in the storage type.

    bf16 is returned as its raw 16-bit pattern (numpy has no bf16 type).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == F32:
        return x
    if dtype == F16:
        return x.astype(np.float16)
    import torch  # library rounding; bf16 has no numpy type

    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def storage_to_float64(a: np.ndarray, dtype: int) -> np.ndarray:
    """Exact widening of stored values (any storage type) to float64."""
    if dtype == BF16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def nan_fill(shape, dtype: int) -> np.ndarray:
    if dtype == F32:
        return np.full(shape, np.nan, dtype=np.float32)
    if dtype == FP8:
        return np.full(shape, _NAN_BITS[FP8], dtype=np.uint8)
    return np.full(shape, _NAN_BITS[dtype], dtype=np.uint16).view(_STORAGE[dtype])


def random_e4m3_codes(rng: np.random.Generator, shape, lo: int = 3, hi: int = 10) -> np.ndarray:
    """E4M3 codes drawn field by field (see the module notes); never NaN.

    The exponent field lies in [lo, hi]; lo=0, hi=15 reaches every finite code.
    """
    sign = rng.integers(0, 2, size=shape, dtype=np.uint8)
    ex = np.clip(np.rint(rng.standard_normal(size=shape, dtype=np.float32) + np.float32(7.0)),
                 lo, hi).astype(np.uint8)
    frac = rng.integers(0, 8, size=shape, dtype=np.uint8)
    frac = np.where((ex == 15) & (frac == 7), np.uint8(6), frac)
    return ((sign << 7) | (ex << 3) | frac).astype(np.uint8)


@dataclass
class Workload:
    """One decode step's worth of inputs (host arrays in storage types)."""

    name: str
    dtype: int
    B: int
    Hq: int
    Hkv: int
    D: int
    block_size: int
    num_blocks: int
    max_blocks: int
    scale: float
    partition_size: int
    q: np.ndarray               # [B, Hq, D]
    k_cache: np.ndarray         # [num_blocks, block_size, Hkv, D], state before the step
    v_cache: np.ndarray
    block_tables: np.ndarray    # [B, max_blocks] int32, -1 = unused
    context_lens: np.ndarray    # [B] int32, after the step's append
    new_key: np.ndarray         # [T, Hkv, D]
    new_value: np.ndarray
    slot_mapping: np.ndarray    # [T] int64
    block_mapping: np.ndarray   # [P, 2] int64 (src, dst) copy-on-write pairs
    seed: int = 0
    meta: Dict = field(default_factory=dict)
    kv_dtype: int = -1          # K pool element type: dtype, or FP8 (codes times k_scale)
    k_scale: float = 1.0
    v_scale: float = 1.0
    v_dtype: int = -1           # V pool element type (default: the K pool's)

    def __post_init__(self):
        if self.kv_dtype < 0:
            self.kv_dtype = self.dtype
        if self.v_dtype < 0:
            self.v_dtype = self.kv_dtype

    @property
    def fp8(self) -> bool:
        """Some pool holds FP8 codes."""
        return self.kv_dtype == FP8 or self.v_dtype == FP8

    @property
    def mixed(self) -> bool:
        """The K and V pools hold different element types."""
        return self.kv_dtype != self.v_dtype

    @property
    def esize(self) -> int:
        """Bytes per cached K/V element (the average of the two pools)."""
        return (ESIZE[self.kv_dtype] + ESIZE[self.v_dtype]) // 2

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.B else 0

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one decode pass must read (attended tokens only)."""
        tokens = int(np.asarray(self.context_lens, dtype=np.int64).sum())
        return tokens * self.Hkv * self.D * (ESIZE[self.kv_dtype] + ESIZE[self.v_dtype])

    def unique_kv_bytes(self) -> int:
        """K+V bytes of the distinct physical slots attended (shared blocks once)."""
        bs = self.block_size
        slots = set()
        for b in range(self.B):
            n = int(self.context_lens[b])
            for i in range((n + bs - 1) // bs):
                slots.add((int(self.block_tables[b, i]), min(bs, n - i * bs)))
        rows = sum(r for _, r in slots)
        return rows * self.Hkv * self.D * (ESIZE[self.kv_dtype] + ESIZE[self.v_dtype])


def kv_bytes_for(context_lens, Hkv: int, D: int, esize: int) -> int:
    """K and V bytes of ``sum(context_lens)`` tokens: 2 * Hkv * D * esize each.

    For the Llama-2-7B shape (32 heads x 128, fp16) this is 16 KiB per token
    per layer, the figure given in section 1 of "vLLM 与 LLM 推理部署实战".
    """
    return int(np.asarray(context_lens, dtype=np.int64).sum()) * 2 * Hkv * D * esize


# --------------------------------------------------------------------------
# generic builder: every sequence prefilled, then one appended token each
# --------------------------------------------------------------------------
def _fill_rows(pool: np.ndarray, table_row: np.ndarray, bs: int, first: int,
               rows: np.ndarray) -> None:
    """Write logical token rows [first, first+len(rows)) of one sequence."""
    if len(rows) == 0:
        return
    t = np.arange(first, first + len(rows))
    pool[table_row[t // bs], t % bs] = rows


def build_decode_case(name: str, dtype: int, B: int, Hq: int, Hkv: int, D: int,
                      block_size: int, num_blocks: int, context_lens: Seq[int],
                      seed: int, rng: Optional[np.random.Generator] = None,
                      max_blocks: Optional[int] = None, scale: Optional[float] = None,
                      partition_size: int = 0, shuffle: bool = True,
                      k_boost_frac: float = 0.0, k_boost: float = 8.0,
                      kv_fp8: bool = False, k_scale: float = 0.3,
                      v_scale: float = 0.7, v_fp8: Optional[bool] = None) -> Workload:
    """Independent sequences, each prefilled with ctx-1 tokens plus one append.

    kv_fp8: the pools hold E4M3 codes (value = code * k_scale / v_scale,
    scales rounded to float32); the query and the new rows keep ``dtype``.
    v_fp8 (default kv_fp8) sets the V pool apart: kv_fp8=True, v_fp8=False
    is an FP8 K pool beside a V pool of ``dtype``.
    """
    v_fp8 = kv_fp8 if v_fp8 is None else bool(v_fp8)
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    rng = rng if rng is not None else np.random.Generator(np.random.PCG64(seed))
    ctx = np.asarray(context_lens, dtype=np.int64)
    if len(ctx) != B or (ctx < 1).any():
        raise ValueError("need B context lengths, each >= 1")
    order = rng.permutation(num_blocks) if shuffle else np.arange(num_blocks)
    bm = BlockManager(num_blocks, block_size, order)
    slots = np.empty(B, dtype=np.int64)
    if shuffle:
        for b in range(B):
            bm.allocate_prefill(b, int(ctx[b]) - 1)
        for b in range(B):
            slot, cow = bm.append_token(b)
            assert cow is None
            slots[b] = slot
    else:
        # contiguous layout: each sequence's blocks, the appended token's
        # included, are one run of consecutive physical ids
        for b in range(B):
            bm.allocate_prefill(b, int(ctx[b]) - 1)
            slot, cow = bm.append_token(b)
            assert cow is None
            slots[b] = slot
    need = max(len(bm.seqs[b].block_table) for b in range(B))
    MB = need if max_blocks is None else int(max_blocks)
    if MB < need:
        raise ValueError("max_blocks too small for the context lengths")
    tables = np.full((B, MB), -1, dtype=np.int32)
    for b in range(B):
        tb = bm.seqs[b].block_table
        tables[b, :len(tb)] = tb

    st = _STORAGE[dtype]
    kdt = FP8 if kv_fp8 else dtype
    vdt = FP8 if v_fp8 else dtype
    q = round_to_storage(rng.standard_normal((B, Hq, D), dtype=np.float32), dtype).view(st)
    kc = nan_fill((num_blocks, block_size, Hkv, D), kdt)
    vc = nan_fill((num_blocks, block_size, Hkv, D), vdt)
    for b in range(B):
        n = int(ctx[b]) - 1
        if kv_fp8:
            _fill_rows(kc, tables[b], block_size, 0, random_e4m3_codes(rng, (n, Hkv, D)))
        else:
            k = rng.standard_normal((n, Hkv, D), dtype=np.float32)
            if k_boost_frac > 0.0:
                k *= np.where(rng.random((n, Hkv, 1)) < k_boost_frac, np.float32(k_boost),
                              np.float32(1.0))
            _fill_rows(kc, tables[b], block_size, 0, round_to_storage(k, dtype).view(st))
        if v_fp8:
            _fill_rows(vc, tables[b], block_size, 0, random_e4m3_codes(rng, (n, Hkv, D)))
        else:
            v = rng.standard_normal((n, Hkv, D), dtype=np.float32)
            _fill_rows(vc, tables[b], block_size, 0, round_to_storage(v, dtype).view(st))
    nk = round_to_storage(rng.standard_normal((B, Hkv, D), dtype=np.float32), dtype).view(st)
    nv = round_to_storage(rng.standard_normal((B, Hkv, D), dtype=np.float32), dtype).view(st)
    return Workload(
        name=name, dtype=dtype, B=B, Hq=Hq, Hkv=Hkv, D=D, block_size=block_size,
        num_blocks=num_blocks, max_blocks=MB,
        scale=float(1.0 / math.sqrt(D)) if scale is None else float(scale),
        partition_size=int(partition_size), q=q, k_cache=kc, v_cache=vc,
        block_tables=tables, context_lens=ctx.astype(np.int32), new_key=nk, new_value=nv,
        slot_mapping=slots, block_mapping=np.zeros((0, 2), dtype=np.int64), seed=seed,
        kv_dtype=kdt, k_scale=float(np.float32(k_scale)) if kv_fp8 else 1.0,
        v_scale=float(np.float32(v_scale)) if v_fp8 else 1.0, v_dtype=vdt)


# --------------------------------------------------------------------------
# shared-prefix parallel sampling (fork + copy-on-write)
# --------------------------------------------------------------------------
def build_shared_prefix_case(name: str, dtype: int, groups: int, children: int,
                             prefix_blocks: int, Hq: int, Hkv: int, D: int,
                             block_size: int, num_blocks: int, max_suffix: int,
                             seed: int, pinned_children: int = 2) -> Workload:
    """Groups of sequences forked from one parent each (parallel sampling).

    Each parent holds ``prefix_blocks`` full blocks plus a partial block of
    r ~ U[1, block_size-1] tokens; its children share all of them (refcount =
    children). Children 0..pinned_children-1 keep no private suffix; the others
    get L ~ U[0, max_suffix] tokens, appended round-robin through the block
    manager, so their first append copies the shared partial block. In the
    measured step every child appends one token: child 0 copies the partial
    block (one copy-on-write pair per group) and child 1, then its sole owner,
    writes into it in place.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    bs = block_size
    order = rng.permutation(num_blocks)
    bm = BlockManager(num_blocks, bs, order)
    parent_len = []
    sid = 0
    child_ids: List[List[int]] = []
    for g in range(groups):
        r = int(rng.integers(1, bs))
        plen = prefix_blocks * bs + r
        parent_len.append(plen)
        pid = 10_000_000 + g
        bm.allocate_prefill(pid, plen)
        ids = []
        for c in range(children):
            bm.fork(pid, sid)
            ids.append(sid)
            sid += 1
        child_ids.append(ids)
    parent_tables = [list(bm.seqs[10_000_000 + g].block_table) for g in range(groups)]
    for g in range(groups):
        bm.free(10_000_000 + g)
    suffix = np.zeros((groups, children), dtype=np.int64)
    for g in range(groups):
        for c in range(pinned_children, children):
            suffix[g, c] = int(rng.integers(0, max_suffix + 1))
    for step in range(int(suffix.max()) if suffix.size else 0):
        for g in range(groups):
            for c in range(children):
                if suffix[g, c] > step:
                    bm.append_token(child_ids[g][c])
    B = groups * children
    slots = np.empty(B, dtype=np.int64)
    pairs = []
    for g in range(groups):
        for c in range(children):
            slot, cow = bm.append_token(child_ids[g][c])
            slots[g * children + c] = slot
            if cow is not None:
                pairs.append(cow)
    bm.check_invariants()
    ctx = np.array([bm.seqs[child_ids[g][c]].seq_len for g in range(groups)
                    for c in range(children)], dtype=np.int64)
    MB = max(len(bm.seqs[i].block_table) for ids in child_ids for i in ids)
    tables = np.full((B, MB), -1, dtype=np.int32)
    for g in range(groups):
        for c in range(children):
            tb = bm.seqs[child_ids[g][c]].block_table
            tables[g * children + c, :len(tb)] = tb
    # the step's copy-on-write happens on the device: before the step, child 0
    # of each group still points at the shared partial block
    pre_tables = tables.copy()
    for (src, dst) in pairs:
        pre_tables[pre_tables == dst] = src

    st = _STORAGE[dtype]
    q = round_to_storage(rng.standard_normal((B, Hq, D), dtype=np.float32), dtype).view(st)
    kc = nan_fill((num_blocks, bs, Hkv, D), dtype)
    vc = nan_fill((num_blocks, bs, Hkv, D), dtype)
    for g in range(groups):
        plen = parent_len[g]
        pk = round_to_storage(rng.standard_normal((plen, Hkv, D), dtype=np.float32), dtype).view(st)
        pv = round_to_storage(rng.standard_normal((plen, Hkv, D), dtype=np.float32), dtype).view(st)
        ptab = np.asarray(parent_tables[g], dtype=np.int64)
        _fill_rows(kc, ptab, bs, 0, pk)
        _fill_rows(vc, ptab, bs, 0, pv)
        tail0 = prefix_blocks * bs
        for c in range(children):
            b = g * children + c
            n = int(suffix[g, c])
            row = pre_tables[b]
            if row[prefix_blocks] != ptab[prefix_blocks]:
                # this child copied the partial block earlier: same prefix rows
                _fill_rows(kc, row, bs, tail0, pk[tail0:])
                _fill_rows(vc, row, bs, tail0, pv[tail0:])
            sk = rng.standard_normal((n, Hkv, D), dtype=np.float32)
            sv = rng.standard_normal((n, Hkv, D), dtype=np.float32)
            _fill_rows(kc, row, bs, plen, round_to_storage(sk, dtype).view(st))
            _fill_rows(vc, row, bs, plen, round_to_storage(sv, dtype).view(st))
    nk = round_to_storage(rng.standard_normal((B, Hkv, D), dtype=np.float32), dtype).view(st)
    nv = round_to_storage(rng.standard_normal((B, Hkv, D), dtype=np.float32), dtype).view(st)
    return Workload(
        name=name, dtype=dtype, B=B, Hq=Hq, Hkv=Hkv, D=D, block_size=bs,
        num_blocks=num_blocks, max_blocks=MB, scale=float(1.0 / math.sqrt(D)),
        partition_size=0, q=q, k_cache=kc, v_cache=vc, block_tables=tables,
        context_lens=ctx.astype(np.int32), new_key=nk, new_value=nv, slot_mapping=slots,
        block_mapping=np.asarray(pairs, dtype=np.int64).reshape(-1, 2), seed=seed,
        meta={"groups": groups, "children": children, "suffix": suffix,
              "parent_len": parent_len, "pre_tables": pre_tables,
              "prefix_blocks": prefix_blocks})


# --------------------------------------------------------------------------
# chunked prefill: a chunk of new tokens per sequence, already in the cache
# --------------------------------------------------------------------------
@dataclass
class PrefillCase:
    """Inputs of one prefill attention call (host arrays in storage types)."""

    name: str
    dtype: int
    B: int
    Hq: int
    Hkv: int
    D: int
    block_size: int
    num_blocks: int
    max_blocks: int
    scale: float
    q: np.ndarray               # [T, Hq, D] new tokens, packed by sequence
    k_cache: np.ndarray         # [num_blocks, block_size, Hkv, D], new tokens included
    v_cache: np.ndarray
    block_tables: np.ndarray    # [B, max_blocks] int32
    context_lens: np.ndarray    # [B] int32, prior + new
    query_start: np.ndarray     # [B + 1] int32
    seed: int = 0

    @property
    def T(self) -> int:
        return int(self.query_start[-1])

    @property
    def max_query_len(self) -> int:
        return int(np.diff(self.query_start).max()) if self.B else 0

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.B else 0

    def attention_flops(self) -> int:
        """4 * D flops per (query head, attended key): the QK and PV products."""
        n = np.diff(self.query_start)
        prior = self.context_lens - n
        keys = sum(int(n[b]) * int(prior[b]) + int(n[b]) * (int(n[b]) + 1) // 2
                   for b in range(self.B))
        return 4 * self.D * self.Hq * keys


def build_prefill_case(name: str, dtype: int, Hq: int, Hkv: int, D: int, block_size: int,
                       prior_lens: Seq[int], new_lens: Seq[int], seed: int,
                       extra_blocks: int = 3) -> PrefillCase:
    """Sequences with prior_lens[b] cached tokens and a chunk of new_lens[b] tokens
    whose K/V rows are already in the pool (written by reshape_and_cache)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    prior = np.asarray(prior_lens, dtype=np.int64)
    new = np.asarray(new_lens, dtype=np.int64)
    B = len(prior)
    ctx = prior + new
    bs = block_size
    num_blocks = int(sum((c + bs - 1) // bs for c in ctx)) + extra_blocks
    bm = BlockManager(num_blocks, bs, rng.permutation(num_blocks))
    for b in range(B):
        bm.allocate_prefill(b, int(ctx[b]))
    MB = max(1, max(len(bm.seqs[b].block_table) for b in range(B)))
    tables = np.full((B, MB), -1, dtype=np.int32)
    for b in range(B):
        tb = bm.seqs[b].block_table
        tables[b, :len(tb)] = tb
    st = _STORAGE[dtype]
    T = int(new.sum())
    q = round_to_storage(rng.standard_normal((T, Hq, D), dtype=np.float32), dtype).view(st)
    kc = nan_fill((num_blocks, bs, Hkv, D), dtype)
    vc = nan_fill((num_blocks, bs, Hkv, D), dtype)
    for b in range(B):
        n = int(ctx[b])
        k = round_to_storage(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype).view(st)
        v = round_to_storage(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype).view(st)
        _fill_rows(kc, tables[b], bs, 0, k)
        _fill_rows(vc, tables[b], bs, 0, v)
    qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    return PrefillCase(name=name, dtype=dtype, B=B, Hq=Hq, Hkv=Hkv, D=D, block_size=bs,
                       num_blocks=num_blocks, max_blocks=MB, scale=float(1.0 / math.sqrt(D)),
                       q=q, k_cache=kc, v_cache=vc, block_tables=tables,
                       context_lens=ctx.astype(np.int32), query_start=qs, seed=seed)


def prefill_to_torch(c: PrefillCase, device="cpu") -> Dict[str, "object"]:
    import torch

    def el(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if c.dtype == BF16:
            t = t.view(torch.int16).view(torch.bfloat16)
        return t.to(device)

    ix = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return {"q": el(c.q), "k_cache": el(c.k_cache), "v_cache": el(c.v_cache),
            "block_tables": ix(c.block_tables), "context_lens": ix(c.context_lens),
            "query_start": ix(c.query_start)}


# --------------------------------------------------------------------------
# the five named workloads
# --------------------------------------------------------------------------
WORKLOADS = {
    1: "tiny-fp32",
    2: "llama2-7b-fp16",
    3: "llama3-70b-gqa-bf16",
    4: "long-context-splitk-bf16",
    5: "shared-prefix-sampling-bf16",
    6: "llama2-7b-fp8kv",
    7: "llama2-7b-fp8k-bf16v",
    8: "llama3-70b-gqa-fp8kv",
}
WORKLOAD_IDS = {v: k for k, v in WORKLOADS.items()}


def make_workload(which, seed: Optional[int] = None, batch: Optional[int] = None,
                  contiguous: bool = False) -> Workload:
    """Build workload ``which`` (1..6 or its name); seed defaults to 1000 + id.

    ``batch`` (profiling runs) keeps every distribution and shape but uses that
    many sequences (groups of 16 for the shared-prefix workload) and a pool
    scaled down with them.

    ``contiguous`` (workloads 2, 3 and 6, full size) gives every sequence one
    run of consecutive physical blocks instead of ids popped from a shuffled
    free list: the same lengths and bytes, with paging reduced to an identity
    table (for measuring what non-contiguous blocks cost).
    """
    if contiguous:
        k = WORKLOAD_IDS[which] if isinstance(which, str) else int(which)
        if k not in (2, 3, 6) or batch is not None:
            raise ValueError("contiguous layouts are built for workloads 2, 3 and 6 at full size")
        return _make_contiguous(k, 1000 + k if seed is None else int(seed))
    k = WORKLOAD_IDS[which] if isinstance(which, str) else int(which)
    seed = 1000 + k if seed is None else int(seed)
    name = WORKLOADS[k] if batch is None else f"{WORKLOADS[k]}-b{int(batch)}"
    if batch is not None and k in (2, 3, 4, 5, 6, 7, 8):
        return _make_batch(k, name, seed, int(batch))
    if k == 1:
        return build_decode_case(name, F32, B=4, Hq=4, Hkv=4, D=64, block_size=16,
                                 num_blocks=64, context_lens=[1, 15, 16, 33], seed=seed,
                                 scale=1.0 / 8.0)
    rng = np.random.Generator(np.random.PCG64(seed))
    if k == 2:
        ctx = rng.integers(128, 2049, size=64)
        return build_decode_case(name, F16, B=64, Hq=32, Hkv=32, D=128, block_size=16,
                                 num_blocks=8192, context_lens=ctx, seed=seed, rng=rng,
                                 max_blocks=128)
    if k == 3:
        ln = rng.lognormal(mean=math.log(1200.0), sigma=0.8, size=128)
        ctx = np.clip(np.rint(ln), 16, 8192).astype(np.int64)
        return build_decode_case(name, BF16, B=128, Hq=64, Hkv=8, D=128, block_size=16,
                                 num_blocks=65536, context_lens=ctx, seed=seed, rng=rng,
                                 max_blocks=512)
    if k == 4:
        return build_decode_case(name, BF16, B=8, Hq=64, Hkv=8, D=128, block_size=32,
                                 num_blocks=16384, context_lens=[32768] * 8, seed=seed,
                                 rng=rng, max_blocks=1024, partition_size=512,
                                 k_boost_frac=0.01)
    if k == 5:
        return build_shared_prefix_case(name, BF16, groups=16, children=16,
                                        prefix_blocks=64, Hq=32, Hkv=8, D=128,
                                        block_size=16, num_blocks=8192, max_suffix=512,
                                        seed=seed)
    if k == 6:
        # the Llama-2-7B batch with an FP8 E4M3 cache: half the bytes per token
        ctx = rng.integers(128, 2049, size=64)
        return build_decode_case(name, F16, B=64, Hq=32, Hkv=32, D=128, block_size=16,
                                 num_blocks=8192, context_lens=ctx, seed=seed, rng=rng,
                                 max_blocks=128, kv_fp8=True)
    if k == 7:
        # the same batch with the explainer's mixed cache: K in FP8, V and query in bf16
        ctx = rng.integers(128, 2049, size=64)
        return build_decode_case(name, BF16, B=64, Hq=32, Hkv=32, D=128, block_size=16,
                                 num_blocks=8192, context_lens=ctx, seed=seed, rng=rng,
                                 max_blocks=128, kv_fp8=True, v_fp8=False)
    if k == 8:
        # the Llama-3-70B-shaped GQA batch with an FP8 E4M3 cache (bf16 query)
        ln = rng.lognormal(mean=math.log(1200.0), sigma=0.8, size=128)
        ctx = np.clip(np.rint(ln), 16, 8192).astype(np.int64)
        return build_decode_case(name, BF16, B=128, Hq=64, Hkv=8, D=128, block_size=16,
                                 num_blocks=65536, context_lens=ctx, seed=seed, rng=rng,
                                 max_blocks=512, kv_fp8=True)
    raise KeyError(which)


def _make_contiguous(k: int, seed: int) -> Workload:
    rng = np.random.Generator(np.random.PCG64(seed))
    name = WORKLOADS[k] + "-contiguous"
    if k in (2, 6):
        ctx = rng.integers(128, 2049, size=64)
        return build_decode_case(name, F16, B=64, Hq=32, Hkv=32, D=128, block_size=16,
                                 num_blocks=8192, context_lens=ctx, seed=seed, rng=rng,
                                 max_blocks=128, kv_fp8=k == 6, shuffle=False)
    ln = rng.lognormal(mean=math.log(1200.0), sigma=0.8, size=128)
    ctx = np.clip(np.rint(ln), 16, 8192).astype(np.int64)
    return build_decode_case(name, BF16, B=128, Hq=64, Hkv=8, D=128, block_size=16,
                             num_blocks=65536, context_lens=ctx, seed=seed, rng=rng,
                             max_blocks=512, shuffle=False)


def _make_batch(k: int, name: str, seed: int, B: int) -> Workload:
    rng = np.random.Generator(np.random.PCG64(seed))
    if k in (2, 6, 7):
        ctx = rng.integers(128, 2049, size=B)
        return build_decode_case(name, BF16 if k == 7 else F16, B=B, Hq=32, Hkv=32, D=128,
                                 block_size=16, num_blocks=B * 128, context_lens=ctx, seed=seed,
                                 rng=rng, max_blocks=128, kv_fp8=k in (6, 7), v_fp8=k == 6)
    if k in (3, 8):
        ln = rng.lognormal(mean=math.log(1200.0), sigma=0.8, size=B)
        ctx = np.clip(np.rint(ln), 16, 8192).astype(np.int64)
        return build_decode_case(name, BF16, B=B, Hq=64, Hkv=8, D=128, block_size=16,
                                 num_blocks=max(512, 2 * int(sum((c + 15) // 16 for c in ctx))),
                                 context_lens=ctx, seed=seed, rng=rng, max_blocks=512,
                                 kv_fp8=k == 8)
    if k == 4:
        return build_decode_case(name, BF16, B=B, Hq=64, Hkv=8, D=128, block_size=32,
                                 num_blocks=B * 2048, context_lens=[32768] * B, seed=seed,
                                 rng=rng, max_blocks=1024, partition_size=512,
                                 k_boost_frac=0.01)
    return build_shared_prefix_case(name, BF16, groups=B, children=16, prefix_blocks=64,
                                    Hq=32, Hkv=8, D=128, block_size=16,
                                    num_blocks=max(1024, 512 * B), max_suffix=512, seed=seed)


def shrink_workload(which, seed: int, B: Optional[int] = None, max_ctx: Optional[int] = None):
    """A reduced copy of a named workload's shape for fast parity tests.

    Same dtype, heads, head size, block size and length distribution family;
    fewer sequences and a shorter length cap, a pool just large enough.
    """
    k = WORKLOAD_IDS[which] if isinstance(which, str) else int(which)
    rng = np.random.Generator(np.random.PCG64(seed))
    if k == 2:
        B = B or 6
        hi = max_ctx or 300
        ctx = rng.integers(1, hi + 1, size=B)
        nb = int(sum((c + 15) // 16 for c in ctx)) + 7
        return build_decode_case("llama2-7b-fp16-small", F16, B=B, Hq=32, Hkv=32, D=128,
                                 block_size=16, num_blocks=nb, context_lens=ctx, seed=seed,
                                 rng=rng)
    if k == 3:
        B = B or 6
        hi = max_ctx or 700
        ln = rng.lognormal(mean=math.log(hi / 3.0), sigma=0.8, size=B)
        ctx = np.clip(np.rint(ln), 1, hi).astype(np.int64)
        nb = int(sum((c + 15) // 16 for c in ctx)) + 5
        return build_decode_case("llama3-70b-gqa-bf16-small", BF16, B=B, Hq=64, Hkv=8, D=128,
                                 block_size=16, num_blocks=nb, context_lens=ctx, seed=seed,
                                 rng=rng)
    if k == 4:
        B = B or 2
        n = max_ctx or 1500
        nb = B * ((n + 31) // 32) + 3
        return build_decode_case("long-context-splitk-bf16-small", BF16, B=B, Hq=64, Hkv=8,
                                 D=128, block_size=32, num_blocks=nb, context_lens=[n] * B,
                                 seed=seed, rng=rng, partition_size=512, k_boost_frac=0.01)
    if k == 5:
        return build_shared_prefix_case("shared-prefix-sampling-bf16-small", BF16, groups=2,
                                        children=4, prefix_blocks=4, Hq=32, Hkv=8, D=128,
                                        block_size=16, num_blocks=96, max_suffix=40,
                                        seed=seed)
    if k in (6, 7):
        B = B or 6
        hi = max_ctx or 300
        ctx = rng.integers(1, hi + 1, size=B)
        nb = int(sum((c + 15) // 16 for c in ctx)) + 7
        return build_decode_case(WORKLOADS[k] + "-small", F16 if k == 6 else BF16, B=B, Hq=32,
                                 Hkv=32, D=128, block_size=16, num_blocks=nb, context_lens=ctx,
                                 seed=seed, rng=rng, kv_fp8=True, v_fp8=k == 6)
    if k == 8:
        B = B or 6
        hi = max_ctx or 700
        ln = rng.lognormal(mean=math.log(hi / 3.0), sigma=0.8, size=B)
        ctx = np.clip(np.rint(ln), 1, hi).astype(np.int64)
        nb = int(sum((c + 15) // 16 for c in ctx)) + 5
        return build_decode_case("llama3-70b-gqa-fp8kv-small", BF16, B=B, Hq=64, Hkv=8, D=128,
                                 block_size=16, num_blocks=nb, context_lens=ctx, seed=seed,
                                 rng=rng, kv_fp8=True)
    raise KeyError(which)


def to_torch(w: Workload, device="cpu") -> Dict[str, "object"]:
    """Device (or host) torch tensors for every array of a workload.

    Element data keep their storage type (bf16 raw bits are viewed as
    ``torch.bfloat16``). No arithmetic happens here.
    """
    import torch

    tdt = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}[w.dtype]

    def el(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if t.dtype == torch.uint8:                 # FP8 codes stay bytes
            return t.to(device)
        if w.dtype == BF16:
            t = t.view(torch.int16).view(torch.bfloat16) if t.dtype != torch.bfloat16 else t
        return t.to(device)

    def ix(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    return {
        "q": el(w.q), "k_cache": el(w.k_cache), "v_cache": el(w.v_cache),
        "new_key": el(w.new_key), "new_value": el(w.new_value),
        "block_tables": ix(w.block_tables), "context_lens": ix(w.context_lens),
        "slot_mapping": ix(w.slot_mapping), "block_mapping": ix(w.block_mapping),
        "torch_dtype": tdt,
    }
