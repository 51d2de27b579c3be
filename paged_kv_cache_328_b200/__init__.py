"""B200-native paged KV-cache decode attention (sm_100a).

The hot path is a C-ABI shared library, ``libpagedkv.so`` (declared in
``include/pagedkv.h``), built in-tree by ``paged_kv_cache_328_b200.build``:

* ``paged_attn_decode``  single-query decode attention over a block-table-paged
                         KV cache, with split-context partitions merged by
                         log-sum-exp;
* ``kv_cache_append``    per-token K/V append into slots;
* ``kv_block_copy``      copy-on-write block copies;
* ``paged_kv_gather``    contiguous copy of one sequence (indexing checks);
* ``kv_blocks_to_host`` / ``kv_blocks_from_host``  block-granular swaps;
* ``BlockManager``       the native host-side block bookkeeping.

This package is the thin Python binding (argument marshalling only) plus the
seeded synthetic input generator in ``workloads``.  Nothing here computes on the
CPU: without the built library every call raises.
"""

from ._lib import (  # noqa: F401
    BlockManager,
    PagedKVError,
    abi_version,
    alloc_workspace,
    check_copy_pairs,
    check_slots,
    get_device_error,
    gqa_partition_tokens,
    gqa_workspace_size,
    kv_block_copy,
    kv_blocks_from_host,
    kv_blocks_to_host,
    kv_cache_append,
    load,
    paged_attn_decode,
    paged_attn_multi_query,
    paged_kv_gather,
    partition_tokens,
    selftest_wait_timeout,
    set_debug_checks,
    strerror,
    tune_partition_tokens,
    workspace_size,
)
