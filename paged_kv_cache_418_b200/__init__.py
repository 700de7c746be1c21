"""B200-native paged KV-cache decode attention.

Decode-step attention of one query token per sequence over a KV cache kept in
fixed-size physical blocks and reached through per-sequence block tables,
plus ``reshape_and_cache`` (write each new token's K/V to its slot) and
``copy_blocks`` (copy-on-write of a shared block). Beside the decode step:
FP8 (E4M3) pools with per-pool scales, ``swap_blocks`` between device and
host pools, a shared-prefix decode that streams a group's common blocks once
for the whole group, and paged (chunked) prefill with a causal mask.

Modules:
  ops            thin ctypes binding of the C-ABI library ``libpa.so``
                 (same names as ``include/pa.h``); loads or builds the CUDA
                 library and fails loudly if it cannot.
  block_manager  host-side free list / block tables / refcounts / CoW.
  workloads      seeded synthetic inputs (no attention arithmetic).

Importing the package does not load the CUDA library; ``ops`` does.
"""

__version__ = "0.1.0"
