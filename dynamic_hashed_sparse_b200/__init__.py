"""B200 dynamic hashed embedding engine: IDMap + EmbeddingBlocks, lookup-or-
insert + sum-pooling forward, coalesced sparse-gradient + fused optimizer
backward, all in the CUDA kernels of libdhs.so (C ABI: include/dhs.h).

This package is the thin Python binding of that library.
"""
from ._binding import (  # noqa: F401
    DhsError,
    OPT_CODES,
    PHASES,
    Table,
    TorchAllocator,
    dhs_pack_keys,
    dhs_status_str,
    embbag_backward_update,
    embbag_backward_update_noalloc,
    NOALLOC_MAX_KEYS,
    embbag_forward,
    embbag_forward_ex,
    embbag_backward_update_ex,
    POOL_MODES,
    ROW_DTYPES,
    ht_counters,
    ht_create,
    ht_destroy,
    ht_export,
    ht_get_rows,
    ht_lookup,
    ht_lookup_or_insert,
    ht_phase_times,
    ht_reserve,
    ht_set_hooks,
    ht_evict,
    ht_live_rows,
    ht_row_stride,
    ht_set_phase_timing,
    ht_size,
    ht_sync,
    ht_shard_route,
    ht_shard_pool,
    ht_shard_grads,
    lib,
)
from .sharded import NcclExchange, ShardedTable, run_lockstep  # noqa: F401,E402
