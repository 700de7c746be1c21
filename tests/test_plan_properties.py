"""Properties of the host-side launch plan and workspace sizing of the C ABI over
random shapes (CPU only; nothing is launched): the partitions cover every
context exactly once, the workspace holds the partials of every partition (or
the tensor-core kernel's pieces and tickets), and the tensor-core path is
planned only for 16-bit and FP8 pools on the shapes it takes."""

from __future__ import annotations

from hypothesis import given, settings, strategies as st

from paged_kv_cache_418_b200 import ops

DEFAULT_PARTITION = 512


def _up(x: int) -> int:
    return (x + 255) // 256 * 256


shapes = st.tuples(
    st.integers(1, 512),                                   # B
    st.sampled_from([1, 2, 4, 8]),                         # Hkv
    st.sampled_from([1, 2, 4, 8, 16]),                     # G
    st.sampled_from([64, 128]),                            # D
    st.sampled_from([16, 32]),                             # block_size
    st.integers(1, 65536),                                 # max_context_len
    st.integers(0, 64),                                    # partition size in blocks (0 = auto)
    st.sampled_from([ops.PA_F32, ops.PA_F16, ops.PA_BF16, ops.PA_FP8_E4M3]),
)


@settings(max_examples=400, deadline=None)
@given(shapes)
def test_partitions_cover_each_context_once(shape):
    B, Hkv, G, D, bs, mcl, pblocks, dtype = shape
    Hq = Hkv * G
    psize_in = pblocks * bs
    kernel, P, psize = ops.pa_decode_plan(dtype, B, Hq, Hkv, D, bs, mcl, psize_in)
    assert kernel in (1, 2)
    tc_shape = D == 128 and Hkv % 4 == 0 and G in (4, 8)
    if dtype == ops.PA_F32 or not tc_shape:
        assert kernel == 1                    # tcgen05 path: 16-bit or FP8 pools, its shapes
    else:
        assert kernel == 2
    if D != 128:
        assert kernel == 1
    assert P >= 1 and psize > 0 and psize % bs == 0
    want = psize_in or DEFAULT_PARTITION
    if kernel == 2:
        # the tensor-core kernel splits the work evenly over the SMs itself
        assert P == 1 and mcl <= psize < mcl + bs
        return
    if P == 1:
        assert mcl <= psize < mcl + bs          # one pass over the whole (block-rounded) context
        assert mcl <= want
    else:
        assert psize == want
        assert (P - 1) * psize < mcl <= P * psize


SMS = 148        # no device here: the library sizes for a B200's 148 SMs


def _tc_bytes(B, Hq, Hkv):
    """Piece slots (2 per SM) of 4 * G query-head rows and one ticket per
    (sequence, group of 4 KV heads): the tensor-core kernel's scratch."""
    ns, slots = 4 * (Hq // Hkv), 2 * SMS
    return _up(slots * ns * 128 * 4) + 2 * _up(slots * ns * 4) + _up(B * (Hkv // 4) * 8)


@settings(max_examples=400, deadline=None)
@given(shapes)
def test_workspace_holds_every_partial(shape):
    B, Hkv, G, D, bs, mcl, pblocks, _ = shape
    Hq = Hkv * G
    psize_in = pblocks * bs
    # the CUDA-core kernel's partials (its plan for the same shape) ...
    _, P, _ = ops.pa_decode_plan(ops.PA_F32, B, Hq, Hkv, D, bs, mcl, psize_in)
    simt = 0 if P == 1 else _up(B * Hq * P * D * 4) + 2 * _up(B * Hq * P * 4)
    # ... or the tensor-core kernel's pieces and tickets, on the shapes it takes
    tc_shape = D == 128 and Hkv % 4 == 0 and G in (4, 8)
    tc = _tc_bytes(B, Hq, Hkv) if tc_shape else 0
    n = ops.pa_workspace_size(B, Hq, Hkv, D, mcl, psize_in)
    assert n == max(simt, tc)
    for dt in (ops.PA_F16, ops.PA_BF16):
        if ops.pa_decode_plan(dt, B, Hq, Hkv, D, bs, mcl, psize_in)[0] == 2:
            assert tc_shape and n >= tc
