"""ctypes binding of libpa.so (the C ABI declared in include/pa.h).

Argument marshalling only: every function here checks nothing the library does
not check itself (except, in debug mode, the cache ops' caller preconditions),
reads the sizes off torch tensor shapes, passes raw device pointers and the
current CUDA stream, and turns a nonzero status into ``PAError``. All of the computing happens in the CUDA kernels. There is no
fallback: if the library cannot be built or loaded, importing this module
raises.
"""

from __future__ import annotations

import contextlib
import ctypes
import os
from typing import Optional, Tuple

import torch

from . import _build

PA_F32, PA_F16, PA_BF16, PA_FP8_E4M3 = 0, 1, 2, 3
PA_OK = 0
PA_DEV_BAD_BLOCK_ID, PA_DEV_BAD_CTX, PA_DEV_BAD_SLOT, PA_DEV_BAD_PAIR = 1, 2, 4, 8
_TORCH_TO_PA = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16,
                torch.uint8: PA_FP8_E4M3, torch.float8_e4m3fn: PA_FP8_E4M3}


class PAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {pa_status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    path = _build.ensure_built()
    lib = ctypes.CDLL(path)
    P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    IP = ctypes.POINTER(ctypes.c_int)
    lib.pa_workspace_size.argtypes = [I, I, I, I, I, I]
    lib.pa_workspace_size.restype = S
    lib.pa_decode.argtypes = [P, I, P, P, P, I, P, I, P, I, I, I, I, I, I, F, I, I, P, S, P, P]
    lib.pa_decode.restype = I
    lib.pa_reshape_and_cache.argtypes = [P, P, P, P, I, P, I, I, I, I, I, P, P]
    lib.pa_reshape_and_cache.restype = I
    lib.pa_copy_blocks.argtypes = [P, P, I, P, I, I, I, I, I, P, P]
    lib.pa_copy_blocks.restype = I
    lib.pa_status_string.argtypes = [I]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_decode_plan.argtypes = [I, I, I, I, I, I, I, I, IP, IP, IP]
    lib.pa_decode_plan.restype = I
    lib.pa_decode_static.argtypes = [P, I, P, P, P, I, P, I, P, I, I, I, I, I, I, F, I, I, P, P]
    lib.pa_decode_static.restype = I
    lib.pa_decode_fp8.argtypes = [P, I, P, I, P, P, F, F, P, I, P, I, I, I, I, I, I, F, I, I, P, S,
                                  P, P]
    lib.pa_decode_fp8.restype = I
    lib.pa_reshape_and_cache_fp8.argtypes = [P, P, I, P, P, F, F, P, I, I, I, I, I, P, P]
    lib.pa_reshape_and_cache_fp8.restype = I
    lib.pa_swap_blocks.argtypes = [P, P, P, P, I, P, I, I, I, I, I, I, P, P]
    lib.pa_swap_blocks.restype = I
    lib.pa_shared_prefix_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
    lib.pa_shared_prefix_workspace_size.restype = S
    lib.pa_decode_shared_prefix.argtypes = [P, I, P, P, P, I, P, I, P, P, I, P, P, I, I, I, I, I,
                                            I, I, I, F, I, I, P, S, P, P]
    lib.pa_decode_shared_prefix.restype = I
    lib.pa_prefill.argtypes = [P, I, P, P, P, I, P, I, P, P, I, I, I, I, I, I, I, I, F, I, P, P]
    lib.pa_prefill.restype = I
    lib.pa_decode_kv.argtypes = [P, I, P, I, P, I, F, P, I, F, P, I, P, I, I, I, I, I, I, F, I, I,
                                 P, S, P, P]
    lib.pa_decode_kv.restype = I
    lib.pa_reshape_and_cache_kv.argtypes = [P, P, I, P, I, F, P, I, F, P, I, I, I, I, I, P, P]
    lib.pa_reshape_and_cache_kv.restype = I
    lib.pa_decode_shared_prefix_kv.argtypes = [P, I, P, I, P, I, F, P, I, F, P, I, P, P, I, P, P,
                                               I, I, I, I, I, I, I, I, F, I, I, P, S, P, P]
    lib.pa_decode_shared_prefix_kv.restype = I
    lib.pa_prefill_kv.argtypes = [P, I, P, I, P, I, F, P, I, F, P, I, P, P, I, I, I, I, I, I, I, I,
                                  F, I, P, P]
    lib.pa_prefill_kv.restype = I
    return lib


LIB = _load()
LIB_PATH = _build.LIB


# Debug mode (PA_DEBUG=1 in the environment, or set_debug(True)): before each
# cache op the binding reads the mapping back to the host and rejects the
# inputs the library leaves to the caller (two tokens on one slot; a copy
# destination named twice or also used as a source). It costs a device-to-host
# copy and a sync per call, so it is off by default.
DEBUG = os.environ.get("PA_DEBUG", "0") not in ("", "0")


def set_debug(on: bool) -> None:
    global DEBUG
    DEBUG = bool(on)


def check_slot_mapping(slot_mapping: torch.Tensor, fn: str = "pa_reshape_and_cache") -> None:
    """ValueError if two tokens name the same (non-negative) slot."""
    s = slot_mapping.detach().to("cpu", torch.int64).reshape(-1)
    s = s[s >= 0]
    if torch.unique(s).numel() != s.numel():
        raise ValueError(f"{fn}: two tokens name the same slot in slot_mapping")


def check_block_mapping(block_mapping: torch.Tensor, fn: str = "pa_copy_blocks",
                        same_pool: bool = True) -> None:
    """ValueError if a destination block is named twice or, within one pool, is
    also a source of the same call."""
    m = block_mapping.detach().to("cpu", torch.int64).reshape(-1, 2)
    src, dst = m[:, 0], m[:, 1]
    if torch.unique(dst).numel() != dst.numel():
        raise ValueError(f"{fn}: a destination block is named twice")
    if same_pool and bool(torch.isin(dst, src).any()):
        raise ValueError(f"{fn}: a destination block is also a source")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _on_device_of(*tensors):
    """Make the device of the first CUDA tensor current for the call, so the
    default stream (and, for pa_decode_static, the scratch) is that device's."""
    for t in tensors:
        if t is not None and t.is_cuda:
            return torch.cuda.device(t.device)
    return contextlib.nullcontext()


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def pa_dtype(t: torch.Tensor) -> int:
    try:
        return _TORCH_TO_PA[t.dtype]
    except KeyError:
        raise PAError("pa_dtype", 3) from None


def pa_status_string(status: int) -> str:
    return LIB.pa_status_string(int(status)).decode()


def pa_workspace_size(B: int, Hq: int, Hkv: int, D: int, max_context_len: int,
                      partition_size: int = 0) -> int:
    return int(LIB.pa_workspace_size(B, Hq, Hkv, D, max_context_len, partition_size))


def pa_decode_plan(dtype: int, B: int, Hq: int, Hkv: int, D: int, block_size: int,
                   max_context_len: int, partition_size: int = 0) -> Tuple[int, int, int]:
    k, p, t = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    rc = LIB.pa_decode_plan(dtype, B, Hq, Hkv, D, block_size, max_context_len, partition_size,
                            ctypes.byref(k), ctypes.byref(p), ctypes.byref(t))
    if rc:
        raise PAError("pa_decode_plan", rc)
    return k.value, p.value, t.value


def pa_decode(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
              value_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor,
              scale: float, max_context_len: int, partition_size: int = 0,
              workspace: Optional[torch.Tensor] = None, err_flag: Optional[torch.Tensor] = None,
              stream=None) -> None:
    """out [B,Hq,D] <- paged decode attention (see pa_decode in include/pa.h)."""
    B, Hq, D = query.shape
    num_blocks, block_size, Hkv, _ = key_cache.shape
    with _on_device_of(query):
        rc = LIB.pa_decode(
            _ptr(out), pa_dtype(out), _ptr(query), _ptr(key_cache), _ptr(value_cache),
            pa_dtype(key_cache), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
            B, Hq, Hkv, D, block_size, num_blocks, float(scale), int(max_context_len),
            int(partition_size), _ptr(workspace),
            0 if workspace is None else workspace.numel() * workspace.element_size(),
            _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_decode", rc)


# PA_STATIC_SCRATCH_BYTES of include/pa.h (a CPU test checks the two agree)
PA_STATIC_SCRATCH_BYTES = 64 * 1024 * 1024


def pa_decode_static(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                     value_cache: torch.Tensor, block_tables: torch.Tensor,
                     context_lens: torch.Tensor, scale: float, max_context_len: int,
                     partition_size: int = 0, err_flag: Optional[torch.Tensor] = None,
                     stream=None) -> None:
    """pa_decode with the library's own device scratch instead of a workspace
    argument, for callers that cannot allocate device memory (see pa_decode_static
    in include/pa.h: one shared scratch per device, calls must not overlap)."""
    B, Hq, D = query.shape
    num_blocks, block_size, Hkv, _ = key_cache.shape
    with _on_device_of(query):
        rc = LIB.pa_decode_static(
            _ptr(out), pa_dtype(out), _ptr(query), _ptr(key_cache), _ptr(value_cache),
            pa_dtype(key_cache), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
            B, Hq, Hkv, D, block_size, num_blocks, float(scale), int(max_context_len),
            int(partition_size), _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_decode_static", rc)


def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                         value_cache: torch.Tensor, slot_mapping: torch.Tensor,
                         err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """Scatter new K/V rows [T,Hkv,D] into the pools at slot_mapping [T] (int64)."""
    if DEBUG:
        check_slot_mapping(slot_mapping)
    num_blocks, block_size, Hkv, D = key_cache.shape
    T = slot_mapping.shape[0]
    with _on_device_of(key_cache):
        rc = LIB.pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache),
                                      pa_dtype(key_cache), _ptr(slot_mapping), T, Hkv, D,
                                      block_size, num_blocks, _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_reshape_and_cache", rc)


def pa_copy_blocks(key_cache: torch.Tensor, value_cache: torch.Tensor,
                   block_mapping: torch.Tensor, err_flag: Optional[torch.Tensor] = None,
                   stream=None) -> None:
    """Copy whole blocks src -> dst for each (src, dst) row of block_mapping [P,2] (int64)."""
    if DEBUG:
        check_block_mapping(block_mapping)
    num_blocks, block_size, Hkv, D = key_cache.shape
    P = block_mapping.shape[0]
    with _on_device_of(key_cache):
        rc = LIB.pa_copy_blocks(_ptr(key_cache), _ptr(value_cache), pa_dtype(key_cache),
                                _ptr(block_mapping), P, Hkv, D, block_size, num_blocks,
                                _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_copy_blocks", rc)


def pa_decode_fp8(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                  value_cache: torch.Tensor, k_scale: float, v_scale: float,
                  block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                  max_context_len: int, partition_size: int = 0,
                  workspace: Optional[torch.Tensor] = None,
                  err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """out [B,Hq,D] <- paged decode attention over FP8 E4M3 pools (uint8 codes)."""
    B, Hq, D = query.shape
    num_blocks, block_size, Hkv, _ = key_cache.shape
    with _on_device_of(query):
        rc = LIB.pa_decode_fp8(
            _ptr(out), pa_dtype(out), _ptr(query), pa_dtype(query), _ptr(key_cache),
            _ptr(value_cache), float(k_scale), float(v_scale), _ptr(block_tables),
            block_tables.shape[1], _ptr(context_lens), B, Hq, Hkv, D, block_size, num_blocks,
            float(scale), int(max_context_len), int(partition_size), _ptr(workspace),
            0 if workspace is None else workspace.numel() * workspace.element_size(),
            _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_decode_fp8", rc)


def pa_reshape_and_cache_fp8(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                             value_cache: torch.Tensor, k_scale: float, v_scale: float,
                             slot_mapping: torch.Tensor, err_flag: Optional[torch.Tensor] = None,
                             stream=None) -> None:
    """Quantise new K/V rows [T,Hkv,D] to E4M3 codes and scatter them into the pools."""
    if DEBUG:
        check_slot_mapping(slot_mapping, "pa_reshape_and_cache_fp8")
    num_blocks, block_size, Hkv, D = key_cache.shape
    T = slot_mapping.shape[0]
    with _on_device_of(key_cache):
        rc = LIB.pa_reshape_and_cache_fp8(_ptr(key), _ptr(value), pa_dtype(key), _ptr(key_cache),
                                          _ptr(value_cache), float(k_scale), float(v_scale),
                                          _ptr(slot_mapping), T, Hkv, D, block_size, num_blocks,
                                          _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_reshape_and_cache_fp8", rc)


def pa_decode_kv(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                 value_cache: torch.Tensor, k_scale: float, v_scale: float,
                 block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                 max_context_len: int, partition_size: int = 0,
                 workspace: Optional[torch.Tensor] = None,
                 err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """out [B,Hq,D] <- paged decode attention with one element type per pool
    (uint8 = FP8 E4M3 codes read times the pool's scale; see pa_decode_kv)."""
    B, Hq, D = query.shape
    num_blocks, block_size, Hkv, _ = key_cache.shape
    with _on_device_of(query):
        rc = LIB.pa_decode_kv(
            _ptr(out), pa_dtype(out), _ptr(query), pa_dtype(query), _ptr(key_cache),
            pa_dtype(key_cache), float(k_scale), _ptr(value_cache), pa_dtype(value_cache),
            float(v_scale), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), B, Hq,
            Hkv, D, block_size, num_blocks, float(scale), int(max_context_len),
            int(partition_size), _ptr(workspace),
            0 if workspace is None else workspace.numel() * workspace.element_size(),
            _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_decode_kv", rc)


def pa_reshape_and_cache_kv(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                            value_cache: torch.Tensor, k_scale: float, v_scale: float,
                            slot_mapping: torch.Tensor, err_flag: Optional[torch.Tensor] = None,
                            stream=None) -> None:
    """Scatter new K/V rows [T,Hkv,D] into pools of per-pool types (an FP8 pool
    gets E4M3 codes of x / scale, a pool of the rows' type gets them copied)."""
    if DEBUG:
        check_slot_mapping(slot_mapping, "pa_reshape_and_cache_kv")
    num_blocks, block_size, Hkv, D = key_cache.shape
    T = slot_mapping.shape[0]
    with _on_device_of(key_cache):
        rc = LIB.pa_reshape_and_cache_kv(_ptr(key), _ptr(value), pa_dtype(key), _ptr(key_cache),
                                         pa_dtype(key_cache), float(k_scale), _ptr(value_cache),
                                         pa_dtype(value_cache), float(v_scale),
                                         _ptr(slot_mapping), T, Hkv, D, block_size, num_blocks,
                                         _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_reshape_and_cache_kv", rc)


def pa_swap_blocks(dst_key: torch.Tensor, dst_value: torch.Tensor, src_key: torch.Tensor,
                   src_value: torch.Tensor, block_mapping: torch.Tensor,
                   err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """Copy whole blocks src pool -> dst pool ((src id, dst id) rows of block_mapping);
    either pool may be pinned host memory."""
    if DEBUG:
        check_block_mapping(block_mapping, "pa_swap_blocks", same_pool=False)
    src_blocks, block_size, Hkv, D = src_key.shape
    dst_blocks = dst_key.shape[0]
    P = block_mapping.shape[0]
    with _on_device_of(dst_key, src_key):
        rc = LIB.pa_swap_blocks(_ptr(dst_key), _ptr(dst_value), _ptr(src_key), _ptr(src_value),
                                pa_dtype(src_key), _ptr(block_mapping), P, Hkv, D, block_size,
                                src_blocks, dst_blocks, _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_swap_blocks", rc)


def pa_shared_prefix_workspace_size(B: int, Hq: int, Hkv: int, D: int, max_context_len: int,
                                    partition_size: int, block_size: int,
                                    max_shared_blocks: int) -> int:
    return int(LIB.pa_shared_prefix_workspace_size(B, Hq, Hkv, D, max_context_len,
                                                   partition_size, block_size,
                                                   max_shared_blocks))


def pa_decode_shared_prefix(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                            value_cache: torch.Tensor, block_tables: torch.Tensor,
                            context_lens: torch.Tensor, shared_blocks: torch.Tensor,
                            group_offsets: torch.Tensor, group_members: torch.Tensor,
                            max_group_size: int, max_shared_blocks: int, scale: float,
                            max_context_len: int, partition_size: int = 0,
                            workspace: Optional[torch.Tensor] = None,
                            err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """pa_decode for groups of sequences sharing their leading blocks (see
    pa_decode_shared_prefix in include/pa.h): shared blocks read once per group."""
    B, Hq, D = query.shape
    num_blocks, block_size, Hkv, _ = key_cache.shape
    with _on_device_of(query):
        rc = LIB.pa_decode_shared_prefix(
            _ptr(out), pa_dtype(out), _ptr(query), _ptr(key_cache), _ptr(value_cache),
            pa_dtype(key_cache), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
            _ptr(shared_blocks), group_offsets.shape[0] - 1, _ptr(group_offsets), _ptr(group_members),
            int(max_group_size), int(max_shared_blocks), B, Hq, Hkv, D, block_size, num_blocks,
            float(scale), int(max_context_len), int(partition_size), _ptr(workspace),
            0 if workspace is None else workspace.numel() * workspace.element_size(),
            _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_decode_shared_prefix", rc)


def pa_decode_shared_prefix_kv(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                               value_cache: torch.Tensor, k_scale: float, v_scale: float,
                               block_tables: torch.Tensor, context_lens: torch.Tensor,
                               shared_blocks: torch.Tensor, group_offsets: torch.Tensor,
                               group_members: torch.Tensor, max_group_size: int,
                               max_shared_blocks: int, scale: float, max_context_len: int,
                               partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
                               err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """pa_decode_shared_prefix over pools of per-pool types (uint8 = FP8 E4M3 codes
    read times the pool's scale; see pa_decode_shared_prefix_kv in include/pa.h)."""
    B, Hq, D = query.shape
    num_blocks, block_size, Hkv, _ = key_cache.shape
    with _on_device_of(query):
        rc = LIB.pa_decode_shared_prefix_kv(
            _ptr(out), pa_dtype(out), _ptr(query), pa_dtype(query), _ptr(key_cache),
            pa_dtype(key_cache), float(k_scale), _ptr(value_cache), pa_dtype(value_cache),
            float(v_scale), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
            _ptr(shared_blocks), group_offsets.shape[0] - 1, _ptr(group_offsets),
            _ptr(group_members), int(max_group_size), int(max_shared_blocks), B, Hq, Hkv, D,
            block_size, num_blocks, float(scale), int(max_context_len), int(partition_size),
            _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
            _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_decode_shared_prefix_kv", rc)


def pa_prefill(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
               value_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor,
               query_start: torch.Tensor, max_query_len: int, scale: float, max_context_len: int,
               err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """out [T,Hq,D] <- causal paged attention of the new tokens query [T,Hq,D] (see
    pa_prefill in include/pa.h)."""
    T, Hq, D = query.shape
    num_blocks, block_size, Hkv, _ = key_cache.shape
    B = query_start.shape[0] - 1
    with _on_device_of(query):
        rc = LIB.pa_prefill(_ptr(out), pa_dtype(out), _ptr(query), _ptr(key_cache), _ptr(value_cache),
                            pa_dtype(key_cache), _ptr(block_tables), block_tables.shape[1],
                            _ptr(context_lens), _ptr(query_start), B, T, int(max_query_len), Hq, Hkv,
                            D, block_size, num_blocks, float(scale), int(max_context_len),
                            _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_prefill", rc)


def pa_prefill_kv(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                  value_cache: torch.Tensor, k_scale: float, v_scale: float,
                  block_tables: torch.Tensor, context_lens: torch.Tensor,
                  query_start: torch.Tensor, max_query_len: int, scale: float,
                  max_context_len: int, err_flag: Optional[torch.Tensor] = None,
                  stream=None) -> None:
    """pa_prefill over pools of per-pool types (uint8 = FP8 E4M3 codes read times
    the pool's scale; see pa_prefill_kv in include/pa.h)."""
    T, Hq, D = query.shape
    num_blocks, block_size, Hkv, _ = key_cache.shape
    B = query_start.shape[0] - 1
    with _on_device_of(query):
        rc = LIB.pa_prefill_kv(_ptr(out), pa_dtype(out), _ptr(query), pa_dtype(query),
                               _ptr(key_cache), pa_dtype(key_cache), float(k_scale),
                               _ptr(value_cache), pa_dtype(value_cache), float(v_scale),
                               _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                               _ptr(query_start), B, T, int(max_query_len), Hq, Hkv, D,
                               block_size, num_blocks, float(scale), int(max_context_len),
                               _ptr(err_flag), _stream(stream))
    if rc:
        raise PAError("pa_prefill_kv", rc)


def shared_prefix_workspace_for(query: torch.Tensor, key_cache: torch.Tensor,
                                max_context_len: int, max_shared_blocks: int,
                                partition_size: int = 0) -> Optional[torch.Tensor]:
    B, Hq, D = query.shape
    n = pa_shared_prefix_workspace_size(B, Hq, key_cache.shape[2], D, max_context_len,
                                        partition_size, key_cache.shape[1], max_shared_blocks)
    return None if n == 0 else torch.empty(n, dtype=torch.uint8, device=query.device)


def workspace_for(query: torch.Tensor, key_cache: torch.Tensor, max_context_len: int,
                  partition_size: int = 0) -> Optional[torch.Tensor]:
    """A device byte tensor big enough for pa_decode, or None when none is needed."""
    B, Hq, D = query.shape
    n = pa_workspace_size(B, Hq, key_cache.shape[2], D, max_context_len, partition_size)
    return None if n == 0 else torch.empty(n, dtype=torch.uint8, device=query.device)
