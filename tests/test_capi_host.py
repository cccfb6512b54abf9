"""C-ABI library checks that need no GPU: it loads, exports every function
include/dhs.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes as C
import os
import re

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "dhs.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+char\s*\*|dhs_status|int64_t|void)\s+(\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_path_calls():
    names = declared_functions()
    for required in ("ht_create", "ht_destroy", "ht_lookup_or_insert", "embbag_forward",
                     "embbag_backward_update", "ht_size", "ht_export", "dhs_status_str",
                     "dhs_pack_keys"):
        assert required in names


def test_library_exports_every_declared_symbol():
    from dynamic_hashed_sparse_b200 import lib
    L = lib()
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings():
    from dynamic_hashed_sparse_b200 import dhs_status_str
    assert dhs_status_str(0) == "ok"
    assert dhs_status_str(5) == "key not found"
    assert dhs_status_str(99) == "unknown status"


def test_host_side_argument_errors_return_before_cuda():
    from dynamic_hashed_sparse_b200 import lib
    L = lib()
    out = C.c_void_p()
    # dim not a multiple of 4, dim too large, bad optimizer, block_rows not a power of two
    assert L.ht_create(6, 0, 0, 0, None, None, C.byref(out)) == 1
    assert L.ht_create(1024, 0, 0, 0, None, None, C.byref(out)) == 1
    assert L.ht_create(16, 9, 0, 0, None, None, C.byref(out)) == 1
    assert L.ht_create(16, 0, 1000, 0, None, None, C.byref(out)) == 1
    assert L.ht_create(16, 0, 0, 1 << 40, None, None, C.byref(out)) == 1
    assert L.ht_create(16, 0, 0, 0, None, None, None) == 1
    # NULL table handle
    assert L.ht_lookup_or_insert(None, None, 0, None, None) == 1
    assert L.embbag_forward(None, None, 0, None, 0, None, None) == 1
    assert L.embbag_backward_update(None, None, 0, None, 0, None, C.c_float(0.1), None) == 1
    assert L.embbag_forward_ex(None, None, 0, None, 0, None, 0, None, None) == 1
    assert L.embbag_backward_update_ex(None, None, 0, None, 0, None, 1, None, C.c_float(0.1), None) == 1
    assert L.ht_sync(None) == 1
    assert L.ht_set_hooks(None, 2, 1) == 1
    n = C.c_int64()
    assert L.ht_evict(None, 3, C.byref(n), None) == 1
    assert L.ht_live_rows(None, C.byref(n)) == 1
    assert L.ht_row_stride(None) == -1
    # sharded engine calls
    counts = (C.c_int64 * 4)()
    assert L.ht_shard_route(None, None, 0, 4, None, None, counts, None) == 1
    assert L.ht_shard_pool(None, None, None, 0, None, 0, None, 0, None, None) == 1
    assert L.ht_shard_grads(None, None, None, 0, 0, None, None, 0, None, None, None) == 1
    # negative sizes
    assert L.dhs_pack_keys(None, None, -1, None, None) == 1
    assert L.dhs_pack_keys(None, None, 0, None, None) == 0
