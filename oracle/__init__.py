"""fp64 CPU oracle (ctypes over ``oracle.c``). TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use this package. It imports nothing from the CUDA package
and the CUDA package imports nothing from it; what both see is the arrays the
seeded workload generator produces.

Every function takes host numpy arrays in their storage types (float32,
float16, uint16 bit patterns for bf16, uint8 codes for FP8 E4M3 pools) plus a
dtype code: 0 = f32, 1 = f16, 2 = bf16, 3 = fp8 (E4M3 codes, read times the
pool's scale). What each one computes, and the passage it follows, is in
the header comment of ``oracle.c``. Parity status: every function is pinned by
the ``tests/test_oracle.py`` checks (library routines, closed forms,
invariances, the pages' worked examples); none is "parity unpinned".
"""

from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_STAMP = _LIB + ".src-sha256"
_lib = None

F32, F16, BF16, FP8 = 0, 1, 2, 3
_ERRORS = {1: "bad argument", 2: "block id out of range", 3: "slot out of range",
           4: "copy pair out of range", 5: "out of memory"}


class OracleError(RuntimeError):
    pass


def _src_hash() -> str:
    with open(_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (fp64, no fast-math, no FMA contraction)."""
    h = _src_hash()
    if not force and os.path.exists(_LIB) and os.path.exists(_STAMP):
        with open(_STAMP) as f:
            if f.read().strip() == h:
                return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    with open(_STAMP, "w") as f:
        f.write(h)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I, D, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_longlong
        lib.oracle_gather.argtypes = [P, P, I, P, I, I, I, I, I]
        lib.oracle_decode.argtypes = [P, P, P, P, I, P, I, P, I, I, I, I, I, I, D, P, I, I]
        lib.oracle_decode_partitioned.argtypes = [P, P, P, P, P, P, P, I, P, I, P, I, I, I, I,
                                                  I, I, D, I, I]
        lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I, I]
        lib.oracle_copy_blocks.argtypes = [P, P, P, I, I, I, I, I, I]
        lib.oracle_widen.argtypes = [P, P, LL, I]
        lib.oracle_max_threads.argtypes = []
        lib.oracle_decode_kv.argtypes = [P, P, I, P, P, I, D, D, P, I, P, I, I, I, I, I, I, D,
                                         P, I, I]
        lib.oracle_reshape_and_cache_fp8.argtypes = [P, P, P, P, I, ctypes.c_float,
                                                     ctypes.c_float, P, I, I, I, I, I]
        lib.oracle_fp8_encode.argtypes = [P, P, LL]
        lib.oracle_swap_blocks.argtypes = [P, P, P, P, P, I, ctypes.c_size_t, I, I]
        lib.oracle_prefill.argtypes = [P, P, P, P, I, P, I, P, P, I, I, I, I, I, I, D, I]
        lib.oracle_decode_mixed.argtypes = [P, P, I, P, I, D, P, I, D, P, I, P, I, I, I, I, I,
                                            I, D, P, I, I]
        lib.oracle_prefill_mixed.argtypes = [P, P, I, P, I, D, P, I, D, P, I, P, P, I, I, I, I,
                                             I, I, D, I]
        lib.oracle_reshape_and_cache_mixed.argtypes = [P, P, P, P, I, I, I, ctypes.c_float,
                                                       ctypes.c_float, P, I, I, I, I, I]
        for fn in ("oracle_gather", "oracle_decode", "oracle_decode_partitioned",
                   "oracle_reshape_and_cache", "oracle_copy_blocks", "oracle_widen",
                   "oracle_max_threads", "oracle_decode_kv", "oracle_reshape_and_cache_fp8",
                   "oracle_fp8_encode", "oracle_swap_blocks", "oracle_prefill",
                   "oracle_decode_mixed", "oracle_prefill_mixed",
                   "oracle_reshape_and_cache_mixed"):
            getattr(lib, fn).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int) -> None:
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"error {rc}"))


def _c(a, dt=None):
    return np.ascontiguousarray(a if dt is None else np.asarray(a, dtype=dt))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def widen(a: np.ndarray, dtype: int) -> np.ndarray:
    """Exact float64 values of stored f32 / f16 / bf16 elements or E4M3 codes."""
    a = _c(a)
    out = np.empty(a.shape, dtype=np.float64)
    _check(_load().oracle_widen(_ptr(out), _ptr(a), a.size, dtype))
    return out


def gather(pool: np.ndarray, dtype: int, table_row: np.ndarray, ctx: int) -> np.ndarray:
    """Contiguous [ctx, Hkv, D] float64 rows of one sequence (all KV heads)."""
    pool = _c(pool)
    nb, bs, hkv, d = pool.shape
    tr = _c(table_row, np.int32)
    out = np.empty((ctx, hkv, d), dtype=np.float64)
    _check(_load().oracle_gather(_ptr(out), _ptr(pool), dtype, _ptr(tr), int(ctx), hkv, d, bs, nb))
    return out


def decode(q, k_cache, v_cache, dtype: int, block_tables, context_lens, scale: float,
           rows=None, n_threads: int = 0) -> np.ndarray:
    """Attention outputs in float64: [B, Hq, D], or [len(rows), D] for (b, hq) rows."""
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    bt, cl = _c(block_tables, np.int32), _c(context_lens, np.int32)
    B, Hq, D = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    assert d2 == D and v_cache.shape == k_cache.shape and bt.shape[0] == B
    if rows is None:
        out = np.empty((B, Hq, D), dtype=np.float64)
        rp, nr = None, 0
    else:
        rows = _c(rows, np.int32).reshape(-1, 2)
        out = np.empty((rows.shape[0], D), dtype=np.float64)
        rp, nr = _ptr(rows), rows.shape[0]
    _check(_load().oracle_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), dtype,
                                 _ptr(bt), bt.shape[1], _ptr(cl), B, Hq, hkv, D, bs, nb,
                                 float(scale), rp, nr, int(n_threads)))
    return out


def decode_partitioned(q, k_cache, v_cache, dtype: int, block_tables, context_lens,
                       scale: float, partition_size: int, n_threads: int = 0
                       ) -> Tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """(out [B,Hq,D], m [B,Hq,P], l [B,Hq,P], acc [B,Hq,P,D]) in float64."""
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    bt, cl = _c(block_tables, np.int32), _c(context_lens, np.int32)
    B, Hq, D = q.shape
    nb, bs, hkv, _ = k_cache.shape
    maxc = int(cl.max()) if B else 0
    P = (maxc + partition_size - 1) // partition_size
    out = np.empty((B, Hq, D), dtype=np.float64)
    m = np.empty((B, Hq, P), dtype=np.float64)
    l = np.empty((B, Hq, P), dtype=np.float64)
    acc = np.empty((B, Hq, P, D), dtype=np.float64)
    _check(_load().oracle_decode_partitioned(
        _ptr(out), _ptr(m), _ptr(l), _ptr(acc), _ptr(q), _ptr(k_cache), _ptr(v_cache), dtype,
        _ptr(bt), bt.shape[1], _ptr(cl), B, Hq, hkv, D, bs, nb, float(scale),
        int(partition_size), int(n_threads)))
    return out, m, l, acc


def reshape_and_cache(k_cache: np.ndarray, v_cache: np.ndarray, key, value, slot_mapping,
                      dtype: int) -> None:
    """In place on the host pools (must be C-contiguous)."""
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    key, value, sm = _c(key), _c(value), _c(slot_mapping, np.int64)
    nb, bs, hkv, d = k_cache.shape
    _check(_load().oracle_reshape_and_cache(_ptr(k_cache), _ptr(v_cache), _ptr(key), _ptr(value),
                                            _ptr(sm), sm.shape[0], hkv, d, bs, nb, dtype))


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, block_mapping, dtype: int) -> None:
    """In place on the host pools (must be C-contiguous)."""
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    bm = _c(block_mapping, np.int64).reshape(-1, 2)
    nb, bs, hkv, d = k_cache.shape
    _check(_load().oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(bm), bm.shape[0],
                                      hkv, d, bs, nb, dtype))


def decode_kv(q, q_dtype: int, k_cache, v_cache, kv_dtype: int, k_scale: float, v_scale: float,
              block_tables, context_lens, scale: float, rows=None, n_threads: int = 0
              ) -> np.ndarray:
    """Attention with the query in q_dtype and the pools in kv_dtype (FP8 codes are
    read times k_scale / v_scale): [B, Hq, D] float64, or [len(rows), D]."""
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    bt, cl = _c(block_tables, np.int32), _c(context_lens, np.int32)
    B, Hq, D = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    assert d2 == D and v_cache.shape == k_cache.shape and bt.shape[0] == B
    if rows is None:
        out = np.empty((B, Hq, D), dtype=np.float64)
        rp, nr = None, 0
    else:
        rows = _c(rows, np.int32).reshape(-1, 2)
        out = np.empty((rows.shape[0], D), dtype=np.float64)
        rp, nr = _ptr(rows), rows.shape[0]
    _check(_load().oracle_decode_kv(_ptr(out), _ptr(q), q_dtype, _ptr(k_cache), _ptr(v_cache),
                                    kv_dtype, float(k_scale), float(v_scale), _ptr(bt),
                                    bt.shape[1], _ptr(cl), B, Hq, hkv, D, bs, nb, float(scale),
                                    rp, nr, int(n_threads)))
    return out


def fp8_encode(x) -> np.ndarray:
    """E4M3 codes (uint8) of float32 values: nearest even, saturating at +-448."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    _check(_load().oracle_fp8_encode(_ptr(out), _ptr(x), x.size))
    return out


def reshape_and_cache_fp8(k_codes: np.ndarray, v_codes: np.ndarray, key, value, src_dtype: int,
                          k_scale: float, v_scale: float, slot_mapping) -> None:
    """In place on uint8 code pools [NB, bs, Hkv, D]: code = E4M3(float(x) / scale)."""
    assert k_codes.flags.c_contiguous and v_codes.flags.c_contiguous
    assert k_codes.dtype == np.uint8 and v_codes.dtype == np.uint8
    key, value, sm = _c(key), _c(value), _c(slot_mapping, np.int64)
    nb, bs, hkv, d = k_codes.shape
    _check(_load().oracle_reshape_and_cache_fp8(
        _ptr(k_codes), _ptr(v_codes), _ptr(key), _ptr(value), src_dtype, float(k_scale),
        float(v_scale), _ptr(sm), sm.shape[0], hkv, d, bs, nb))


def swap_blocks(dst_k: np.ndarray, dst_v: np.ndarray, src_k: np.ndarray, src_v: np.ndarray,
                block_mapping) -> None:
    """Copy whole blocks src pool -> dst pool for each (src id, dst id) pair, in place."""
    assert dst_k.flags.c_contiguous and dst_v.flags.c_contiguous
    src_k, src_v = _c(src_k), _c(src_v)
    bm = _c(block_mapping, np.int64).reshape(-1, 2)
    blk = src_k[0].nbytes if src_k.shape[0] else 0
    assert dst_k[0].nbytes == blk and dst_k.dtype == src_k.dtype
    _check(_load().oracle_swap_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(src_k), _ptr(src_v),
                                      _ptr(bm), bm.shape[0], blk, src_k.shape[0], dst_k.shape[0]))


def prefill(q, k_cache, v_cache, dtype: int, block_tables, context_lens, query_start,
            scale: float, n_threads: int = 0) -> np.ndarray:
    """Causal prefill attention in float64: [T, Hq, D] for the packed new tokens."""
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    bt, cl, qs = _c(block_tables, np.int32), _c(context_lens, np.int32), _c(query_start, np.int32)
    T, Hq, D = q.shape
    nb, bs, hkv, _ = k_cache.shape
    B = cl.shape[0]
    assert qs.shape[0] == B + 1 and int(qs[-1]) == T
    out = np.empty((T, Hq, D), dtype=np.float64)
    _check(_load().oracle_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), dtype,
                                  _ptr(bt), bt.shape[1], _ptr(cl), _ptr(qs), B, Hq, hkv, D, bs, nb,
                                  float(scale), int(n_threads)))
    return out


def decode_mixed(q, q_dtype: int, k_cache, k_dtype: int, k_scale: float, v_cache, v_dtype: int,
                 v_scale: float, block_tables, context_lens, scale: float, rows=None,
                 n_threads: int = 0) -> np.ndarray:
    """Attention with one element type per pool (e.g. K as FP8 codes times
    k_scale, V as bf16): [B, Hq, D] float64, or [len(rows), D]."""
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    bt, cl = _c(block_tables, np.int32), _c(context_lens, np.int32)
    B, Hq, D = q.shape
    nb, bs, hkv, d2 = k_cache.shape
    assert d2 == D and v_cache.shape == k_cache.shape and bt.shape[0] == B
    if rows is None:
        out = np.empty((B, Hq, D), dtype=np.float64)
        rp, nr = None, 0
    else:
        rows = _c(rows, np.int32).reshape(-1, 2)
        out = np.empty((rows.shape[0], D), dtype=np.float64)
        rp, nr = _ptr(rows), rows.shape[0]
    _check(_load().oracle_decode_mixed(_ptr(out), _ptr(q), q_dtype, _ptr(k_cache), k_dtype,
                                       float(k_scale), _ptr(v_cache), v_dtype, float(v_scale),
                                       _ptr(bt), bt.shape[1], _ptr(cl), B, Hq, hkv, D, bs, nb,
                                       float(scale), rp, nr, int(n_threads)))
    return out


def reshape_and_cache_mixed(k_pool: np.ndarray, v_pool: np.ndarray, key, value, src_dtype: int,
                            k_dtype: int, v_dtype: int, k_scale: float, v_scale: float,
                            slot_mapping) -> None:
    """In place: each pool gets the new rows copied (pool type = src_dtype) or
    quantised to E4M3 codes (pool type FP8, code = E4M3(float(x) / scale))."""
    assert k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
    key, value, sm = _c(key), _c(value), _c(slot_mapping, np.int64)
    nb, bs, hkv, d = k_pool.shape
    assert v_pool.shape == k_pool.shape
    _check(_load().oracle_reshape_and_cache_mixed(
        _ptr(k_pool), _ptr(v_pool), _ptr(key), _ptr(value), src_dtype, k_dtype, v_dtype,
        float(k_scale), float(v_scale), _ptr(sm), sm.shape[0], hkv, d, bs, nb))


def prefill_mixed(q, q_dtype: int, k_cache, k_dtype: int, k_scale: float, v_cache, v_dtype: int,
                  v_scale: float, block_tables, context_lens, query_start, scale: float,
                  n_threads: int = 0) -> np.ndarray:
    """Causal prefill attention with one element type per pool: [T, Hq, D] float64."""
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    bt, cl, qs = _c(block_tables, np.int32), _c(context_lens, np.int32), _c(query_start, np.int32)
    T, Hq, D = q.shape
    nb, bs, hkv, _ = k_cache.shape
    B = cl.shape[0]
    assert qs.shape[0] == B + 1 and int(qs[-1]) == T and v_cache.shape == k_cache.shape
    out = np.empty((T, Hq, D), dtype=np.float64)
    _check(_load().oracle_prefill_mixed(_ptr(out), _ptr(q), q_dtype, _ptr(k_cache), k_dtype,
                                        float(k_scale), _ptr(v_cache), v_dtype, float(v_scale),
                                        _ptr(bt), bt.shape[1], _ptr(cl), _ptr(qs), B, Hq, hkv, D,
                                        bs, nb, float(scale), int(n_threads)))
    return out
