"""Properties of the host-side launch plan and workspace sizing of the C ABI over
random shapes (CPU only; nothing is launched): the partitions cover every
context exactly once, the workspace holds the partials of every partition, and
the tensor-core path is planned only for 16-bit pools."""

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
    if dtype in (ops.PA_F32, ops.PA_FP8_E4M3):
        assert kernel == 1                    # tcgen05 path: 16-bit pools only
    if D != 128:
        assert kernel == 1
    assert P >= 1 and psize > 0 and psize % bs == 0
    want = psize_in or DEFAULT_PARTITION
    if P == 1:
        assert mcl <= psize < mcl + bs          # one pass over the whole (block-rounded) context
        assert mcl <= want
    else:
        assert psize == want
        assert (P - 1) * psize < mcl <= P * psize


@settings(max_examples=400, deadline=None)
@given(shapes)
def test_workspace_holds_every_partial(shape):
    B, Hkv, G, D, bs, mcl, pblocks, _ = shape
    Hq = Hkv * G
    psize_in = pblocks * bs
    _, P, _ = ops.pa_decode_plan(ops.PA_F16, B, Hq, Hkv, D, bs, mcl, psize_in)
    n = ops.pa_workspace_size(B, Hq, Hkv, D, mcl, psize_in)
    if P == 1:
        assert n == 0
    else:
        rows = B * Hq * P
        assert n == _up(rows * D * 4) + 2 * _up(rows * 4)
