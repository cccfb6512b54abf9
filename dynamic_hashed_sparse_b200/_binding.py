"""ctypes binding of libdhs.so, with the C ABI's names (include/dhs.h).

Argument marshalling only: each function checks devices, dtypes and shapes,
allocates the output tensor where the C call writes one, and passes raw
pointers plus the CUDA stream.  Every step of the hashed embedding path runs
in the library's kernels.  There is no fallback: if libdhs.so cannot be built
or loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes as C
import os
import re
from typing import Optional, Tuple

import numpy as np
import torch

from . import build as _build

STATUS = {
    0: "ok", 1: "invalid argument", 2: "out of device memory", 3: "CUDA error",
    4: "table full", 5: "key not found", 6: "unsupported", 7: "internal wait bound exceeded",
}
OPT_CODES = {"sgd": 0, "adagrad": 1, "adam": 2, "adagrad_rowwise": 3}
POOL_MODES = {"sum": 0, "mean": 1, "divide": 2}  # "divide": backward only (sharded owners)
ROW_DTYPES = {"f32": 0, "bf16": 1}
PHASES = ("fwd_probe_pool", "fwd_assign", "bwd_probe", "bwd_sort", "bwd_seg_update",
          "lookup_or_insert", "idmap_growth", "fwd_probe", "bwd_combine")


class DhsError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {STATUS.get(status, status)} (status {status})")
        self.status = status


def _load() -> C.CDLL:
    if not _build.up_to_date():
        _build.build()
    path = _build.LIB
    if not os.path.exists(path):
        raise ImportError(f"libdhs.so is missing at {path}; build it with "
                          "`python -m dynamic_hashed_sparse_b200.build`")
    L = C.CDLL(path)
    vp, i64, i32, f32 = C.c_void_p, C.c_int64, C.c_int32, C.c_float
    sig = {
        "dhs_status_str": (C.c_char_p, [C.c_int]),
        "dhs_pack_keys": (C.c_int, [vp, vp, i64, vp, vp]),
        "ht_create": (C.c_int, [i32, C.c_int, i64, i64, vp, vp, C.POINTER(vp)]),
        "ht_create_ex": (C.c_int, [i32, C.c_int, C.c_int, i64, i64, vp, vp, C.POINTER(vp)]),
        "ht_destroy": (C.c_int, [vp]),
        "ht_reserve": (C.c_int, [vp, i64, vp]),
        "ht_lookup_or_insert": (C.c_int, [vp, vp, i64, vp, vp]),
        "ht_lookup": (C.c_int, [vp, vp, i64, vp, vp]),
        "embbag_forward": (C.c_int, [vp, vp, i64, vp, i64, vp, vp]),
        "embbag_backward_update": (C.c_int, [vp, vp, i64, vp, i64, vp, f32, vp]),
        "embbag_forward_ex": (C.c_int, [vp, vp, i64, vp, i64, vp, C.c_int, vp, vp]),
        "embbag_backward_update_ex": (C.c_int, [vp, vp, i64, vp, i64, vp, C.c_int, vp, f32, vp]),
        "embbag_backward_update_noalloc": (C.c_int, [vp, vp, i64, vp, i64, vp, f32, vp]),
        "ht_get_rows": (C.c_int, [vp, vp, i64, vp, vp]),
        "ht_set_hooks": (C.c_int, [vp, i64, C.c_int]),
        "ht_evict": (C.c_int, [vp, i64, C.POINTER(i64), vp]),
        "ht_live_rows": (C.c_int, [vp, C.POINTER(i64)]),
        "ht_row_stride": (i64, [vp]),
        "ht_sync": (C.c_int, [vp]),
        "ht_size": (C.c_int, [vp, C.POINTER(i64)]),
        "ht_export": (C.c_int, [vp, vp, vp]),
        "ht_counters": (C.c_int, [vp, vp]),
        "ht_set_phase_timing": (C.c_int, [vp, C.c_int]),
        "ht_phase_times": (C.c_int, [vp, vp, vp, C.c_int]),
        "ht_shard_route": (C.c_int, [vp, vp, i64, i32, vp, vp, vp, vp]),
        "ht_shard_pool": (C.c_int, [vp, vp, vp, i64, vp, i64, vp, C.c_int, vp, vp]),
        "ht_shard_grads": (C.c_int, [vp, vp, vp, i64, i64, vp, vp, C.c_int, vp, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_lib = _load()


def lib() -> C.CDLL:
    return _lib


class _OptParams(C.Structure):
    _fields_ = [("eps", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float)]


# dhs_allocator: alloc(bytes, stream, ctx) -> device pointer or NULL;
# free(ptr, bytes, stream, ctx)
ALLOC_FN = C.CFUNCTYPE(C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p)
FREE_FN = C.CFUNCTYPE(None, C.c_void_p, C.c_size_t, C.c_void_p, C.c_void_p)


class _Allocator(C.Structure):
    _fields_ = [("alloc", ALLOC_FN), ("free", FREE_FN), ("ctx", C.c_void_p)]


class TorchAllocator:
    """A dhs_allocator backed by torch's caching allocator, counting its calls
    (alloc_calls, free_calls, live_bytes).  The ctypes callbacks are kept
    alive by this object, which must outlive every table created with it."""

    def __init__(self, device=None):
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.alloc_calls = 0
        self.free_calls = 0
        self.live_bytes = 0
        self._sizes = {}

        def _alloc(nbytes, stream, ctx):
            try:
                p = torch.cuda.caching_allocator_alloc(int(nbytes), self.device, int(stream or 0))
            except RuntimeError:
                return None
            self.alloc_calls += 1
            self.live_bytes += int(nbytes)
            self._sizes[int(p)] = int(nbytes)
            return int(p)

        def _free(ptr, nbytes, stream, ctx):
            if ptr:
                self.free_calls += 1
                self.live_bytes -= self._sizes.pop(int(ptr), 0)
                torch.cuda.caching_allocator_delete(int(ptr))

        self._c_alloc = ALLOC_FN(_alloc)
        self._c_free = FREE_FN(_free)
        self.struct = _Allocator(self._c_alloc, self._c_free, None)


def _check(fn: str, rc: int):
    if rc != 0:
        raise DhsError(fn, rc)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, dtype, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


class Table:
    """Handle of one library-owned table (IDMap + EmbeddingBlocks)."""

    def __init__(self, handle: int, dim: int, optimizer: str, device: torch.device, weights: str = "f32"):
        self.handle = handle
        self.dim = dim
        self.optimizer = optimizer
        self.device = device
        self.weights = weights
        self.stride = int(_lib.ht_row_stride(handle))  # floats per exported row

    def close(self):
        if self.handle:
            _lib.ht_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def dhs_status_str(status: int) -> str:
    return _lib.dhs_status_str(status).decode()


def dhs_pack_keys(table_ids: torch.Tensor, ids: torch.Tensor, out: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    _dev(table_ids, torch.int32, "table_ids")
    _dev(ids, torch.int64, "ids")
    n = ids.numel()
    if table_ids.numel() != n:
        raise ValueError("table_ids and ids differ in length")
    out = torch.empty(n, dtype=torch.int64, device=ids.device) if out is None else _dev(out, torch.int64, "out")
    _check("dhs_pack_keys", _lib.dhs_pack_keys(table_ids.data_ptr(), ids.data_ptr(), n, out.data_ptr(),
                                               _stream(stream)))
    return out


def ht_create(dim: int, optimizer: str = "sgd", block_rows: int = 0, max_rows: int = 0,
              eps: float = 1e-8, beta1: float = 0.9, beta2: float = 0.999,
              device=None, allocator: Optional[TorchAllocator] = None, weights: str = "f32") -> Table:
    """A new table; weights "f32" or "bf16" (bf16 weights, fp32 optimizer
    state: ht_create_ex)."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    p = _OptParams(eps, beta1, beta2)
    h = C.c_void_p()
    with torch.cuda.device(device):
        rc = _lib.ht_create_ex(int(dim), OPT_CODES[optimizer], ROW_DTYPES[weights], int(block_rows),
                               int(max_rows), C.byref(p),
                               C.byref(allocator.struct) if allocator is not None else None, C.byref(h))
    _check("ht_create", rc)
    t = Table(h.value, int(dim), optimizer, device, weights)
    t.allocator = allocator  # keeps the callbacks alive as long as the table
    return t


def ht_destroy(t: Table):
    t.close()


def ht_reserve(t: Table, n_keys: int, stream=None):
    _check("ht_reserve", _lib.ht_reserve(t.handle, int(n_keys), _stream(stream)))


def ht_lookup_or_insert(t: Table, keys: torch.Tensor, out: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    _dev(keys, torch.int64, "keys")
    out = torch.empty_like(keys) if out is None else _dev(out, torch.int64, "out")
    _check("ht_lookup_or_insert", _lib.ht_lookup_or_insert(t.handle, keys.data_ptr(), keys.numel(),
                                                           out.data_ptr(), _stream(stream)))
    return out


def ht_lookup(t: Table, keys: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _dev(keys, torch.int64, "keys")
    out = torch.empty_like(keys) if out is None else _dev(out, torch.int64, "out")
    _check("ht_lookup", _lib.ht_lookup(t.handle, keys.data_ptr(), keys.numel(), out.data_ptr(),
                                       _stream(stream)))
    return out


def embbag_forward(t: Table, keys: torch.Tensor, bag_offsets: torch.Tensor,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _dev(keys, torch.int64, "keys")
    _dev(bag_offsets, torch.int64, "bag_offsets")
    nb = bag_offsets.numel() - 1
    if nb < 0:
        raise ValueError("bag_offsets needs n_bags + 1 entries")
    if out is None:
        out = torch.empty((nb, t.dim), dtype=torch.float32, device=keys.device)
    else:
        _dev(out, torch.float32, "out")
        if out.numel() != nb * t.dim:
            raise ValueError("out must hold n_bags * dim floats")
        if out.data_ptr() % 16:
            raise ValueError("out must be 16-byte aligned")
    _check("embbag_forward", _lib.embbag_forward(t.handle, keys.data_ptr(), keys.numel(),
                                                 bag_offsets.data_ptr(), nb, out.data_ptr(),
                                                 _stream(stream)))
    return out


def embbag_backward_update(t: Table, keys: torch.Tensor, bag_offsets: torch.Tensor,
                           grad: torch.Tensor, lr: float, stream=None):
    _dev(keys, torch.int64, "keys")
    _dev(bag_offsets, torch.int64, "bag_offsets")
    _dev(grad, torch.float32, "grad")
    if grad.data_ptr() % 16:
        raise ValueError("grad must be 16-byte aligned")
    nb = bag_offsets.numel() - 1
    if grad.numel() != nb * t.dim:
        raise ValueError("grad must hold n_bags * dim floats")
    _check("embbag_backward_update",
           _lib.embbag_backward_update(t.handle, keys.data_ptr(), keys.numel(), bag_offsets.data_ptr(),
                                       nb, grad.data_ptr(), float(lr), _stream(stream)))


def _header_define(name: str) -> int:
    with open(os.path.join(_build.INCLUDE, "dhs.h")) as f:
        m = re.search(rf"#define\s+{name}\s+(\d+)", f.read())
    if not m:
        raise ImportError(f"{name} is not defined in include/dhs.h")
    return int(m.group(1))


def _psw(per_sample_weights, keys: torch.Tensor) -> int:
    if per_sample_weights is None:
        return 0
    _dev(per_sample_weights, torch.float32, "per_sample_weights")
    if per_sample_weights.numel() != keys.numel():
        raise ValueError("per_sample_weights needs one weight per key")
    return per_sample_weights.data_ptr()


def embbag_forward_ex(t: Table, keys: torch.Tensor, bag_offsets: torch.Tensor,
                      per_sample_weights: Optional[torch.Tensor] = None, mode: str = "sum",
                      out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """EmbeddingBag forward with mode "sum" (optionally weighted per id) or
    "mean"."""
    _dev(keys, torch.int64, "keys")
    _dev(bag_offsets, torch.int64, "bag_offsets")
    nb = bag_offsets.numel() - 1
    if nb < 0:
        raise ValueError("bag_offsets needs n_bags + 1 entries")
    if out is None:
        out = torch.empty((nb, t.dim), dtype=torch.float32, device=keys.device)
    else:
        _dev(out, torch.float32, "out")
        if out.numel() != nb * t.dim:
            raise ValueError("out must hold n_bags * dim floats")
    _check("embbag_forward_ex",
           _lib.embbag_forward_ex(t.handle, keys.data_ptr(), keys.numel(), bag_offsets.data_ptr(), nb,
                                  _psw(per_sample_weights, keys), POOL_MODES[mode], out.data_ptr(),
                                  _stream(stream)))
    return out


def embbag_backward_update_ex(t: Table, keys: torch.Tensor, bag_offsets: torch.Tensor, grad: torch.Tensor,
                              lr: float, per_sample_weights: Optional[torch.Tensor] = None, mode: str = "sum",
                              stream=None):
    """Backward + update for the pooling forms of embbag_forward_ex (same
    weights and mode as the forward)."""
    _dev(keys, torch.int64, "keys")
    _dev(bag_offsets, torch.int64, "bag_offsets")
    _dev(grad, torch.float32, "grad")
    nb = bag_offsets.numel() - 1
    if grad.numel() != nb * t.dim:
        raise ValueError("grad must hold n_bags * dim floats")
    _check("embbag_backward_update_ex",
           _lib.embbag_backward_update_ex(t.handle, keys.data_ptr(), keys.numel(), bag_offsets.data_ptr(), nb,
                                          _psw(per_sample_weights, keys), POOL_MODES[mode], grad.data_ptr(),
                                          float(lr), _stream(stream)))


NOALLOC_MAX_KEYS = _header_define("DHS_NOALLOC_MAX_KEYS")


def embbag_backward_update_noalloc(t: Table, keys: torch.Tensor, bag_offsets: torch.Tensor,
                                   grad: torch.Tensor, lr: float, stream=None):
    """embbag_backward_update for callers that cannot allocate device memory
    during a step: the library uses a fixed device array as scratch (at most
    NOALLOC_MAX_KEYS keys, dim <= 128); it allocates nothing.  Make the first
    call on a device before any stream capture; calls that overlap on the GPU
    race."""
    _dev(keys, torch.int64, "keys")
    _dev(bag_offsets, torch.int64, "bag_offsets")
    _dev(grad, torch.float32, "grad")
    nb = bag_offsets.numel() - 1
    if grad.numel() != nb * t.dim:
        raise ValueError("grad must hold n_bags * dim floats")
    _check("embbag_backward_update_noalloc",
           _lib.embbag_backward_update_noalloc(t.handle, keys.data_ptr(), keys.numel(), bag_offsets.data_ptr(),
                                               nb, grad.data_ptr(), float(lr), _stream(stream)))


def ht_get_rows(t: Table, keys: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _dev(keys, torch.int64, "keys")
    out = torch.empty((keys.numel(), t.stride), dtype=torch.float32, device=keys.device) if out is None \
        else _dev(out, torch.float32, "out")
    _check("ht_get_rows", _lib.ht_get_rows(t.handle, keys.data_ptr(), keys.numel(), out.data_ptr(),
                                           _stream(stream)))
    return out


def ht_set_hooks(t: Table, admit_threshold: int = 1, track_access: bool = False):
    """Feature admission threshold and access tracking (before the first insert)."""
    _check("ht_set_hooks", _lib.ht_set_hooks(t.handle, int(admit_threshold), int(bool(track_access))))


def ht_evict(t: Table, max_idle: int, stream=None) -> int:
    """Evict keys idle for more than max_idle insert calls; returns the rows freed."""
    n = C.c_int64()
    _check("ht_evict", _lib.ht_evict(t.handle, int(max_idle), C.byref(n), _stream(stream)))
    return int(n.value)


def ht_live_rows(t: Table) -> Tuple[int, int]:
    """(rows held by keys, latched status)."""
    n = C.c_int64()
    rc = _lib.ht_live_rows(t.handle, C.byref(n))
    return int(n.value), int(rc)


def ht_row_stride(t: Table) -> int:
    return int(_lib.ht_row_stride(t.handle))


def ht_sync(t: Table) -> int:
    """Wait for the table's work; returns (and clears) the latched device status."""
    return int(_lib.ht_sync(t.handle))


def ht_size(t: Table) -> Tuple[int, int]:
    n = C.c_int64()
    rc = _lib.ht_size(t.handle, C.byref(n))
    return int(n.value), int(rc)


def ht_export(t: Table, rows: bool = True) -> Tuple[np.ndarray, Optional[np.ndarray], int]:
    """(keys by row, rows or None, latched status).  rows=False exports the
    key -> row map only."""
    n, rc = ht_size(t)
    keys = np.empty(n, np.int64)
    r = np.empty((n, t.stride), np.float32) if rows else None
    rc2 = _lib.ht_export(t.handle, keys.ctypes.data, r.ctypes.data if rows else None)
    return keys, r, int(rc or rc2)


def ht_counters(t: Table) -> dict:
    out = np.zeros(14, np.int64)
    _check("ht_counters", _lib.ht_counters(t.handle, out.ctypes.data))
    names = ("rows", "inserted", "unique_updated", "insert_calls", "backward_calls", "slots",
             "blocks", "rehashes", "launches", "last_inserted", "host_waits", "host_wait_ns",
             "allocs", "alloc_ns")
    return {k: int(v) for k, v in zip(names, out)}


def ht_set_phase_timing(t: Table, enable):
    """enable: False / 0 off, True / 1 every phase, 2 the IDMap growth phase only."""
    _check("ht_set_phase_timing", _lib.ht_set_phase_timing(t.handle, int(enable)))


def ht_phase_times(t: Table) -> dict:
    ms = np.zeros(len(PHASES), np.float64)
    cnt = np.zeros(len(PHASES), np.int64)
    _check("ht_phase_times", _lib.ht_phase_times(t.handle, ms.ctypes.data, cnt.ctypes.data, len(PHASES)))
    return {p: (float(m), int(c)) for p, m, c in zip(PHASES, ms, cnt)}


# ---- hash-sharded engine (see the header's section on it) ----

def ht_shard_route(t: Table, keys: torch.Tensor, world: int, stream=None):
    """Group the batch's keys by owner rank: (send_keys int64[n], slot_of
    int32[n], counts list[world]).  Synchronises the stream."""
    _dev(keys, torch.int64, "keys")
    n = keys.numel()
    send = torch.empty(n, dtype=torch.int64, device=keys.device)
    slot = torch.empty(n, dtype=torch.int32, device=keys.device)
    counts = np.zeros(world, np.int64)
    _check("ht_shard_route", _lib.ht_shard_route(t.handle, keys.data_ptr(), n, int(world), send.data_ptr(),
                                                 slot.data_ptr(), counts.ctypes.data, _stream(stream)))
    return send, slot, [int(c) for c in counts]


def ht_shard_pool(t: Table, rows: torch.Tensor, slot_of: torch.Tensor, bag_offsets: torch.Tensor,
                  per_sample_weights: Optional[torch.Tensor] = None, mode: str = "sum",
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Pool the owners' rows (rows[slot_of[i]] is the row of id i)."""
    _dev(rows, torch.float32, "rows")
    _dev(slot_of, torch.int32, "slot_of")
    _dev(bag_offsets, torch.int64, "bag_offsets")
    n = slot_of.numel()
    nb = bag_offsets.numel() - 1
    if rows.numel() != n * t.dim:
        raise ValueError("rows must hold n_keys * dim floats")
    if out is None:
        out = torch.empty((nb, t.dim), dtype=torch.float32, device=rows.device)
    psw = 0
    if per_sample_weights is not None:
        _dev(per_sample_weights, torch.float32, "per_sample_weights")
        if per_sample_weights.numel() != n:
            raise ValueError("per_sample_weights needs one weight per key")
        psw = per_sample_weights.data_ptr()
    _check("ht_shard_pool", _lib.ht_shard_pool(t.handle, rows.data_ptr(), slot_of.data_ptr(), n,
                                               bag_offsets.data_ptr(), nb, psw, POOL_MODES[mode], out.data_ptr(),
                                               _stream(stream)))
    return out


def ht_shard_grads(t: Table, grad: torch.Tensor, bag_offsets: torch.Tensor, slot_of: torch.Tensor,
                   per_sample_weights: Optional[torch.Tensor] = None, mode: str = "sum", stream=None):
    """Per-id gradient rows in routed order (and their factors, or None for
    plain sum pooling): (send_grads float[n, dim], send_fact float[n] or None)."""
    _dev(grad, torch.float32, "grad")
    _dev(bag_offsets, torch.int64, "bag_offsets")
    _dev(slot_of, torch.int32, "slot_of")
    n = slot_of.numel()
    nb = bag_offsets.numel() - 1
    if grad.numel() != nb * t.dim:
        raise ValueError("grad must hold n_bags * dim floats")
    send = torch.empty((n, t.dim), dtype=torch.float32, device=grad.device)
    psw = 0
    if per_sample_weights is not None:
        _dev(per_sample_weights, torch.float32, "per_sample_weights")
        psw = per_sample_weights.data_ptr()
    fact = torch.empty(n, dtype=torch.float32, device=grad.device) if (psw or mode == "mean") else None
    _check("ht_shard_grads", _lib.ht_shard_grads(t.handle, grad.data_ptr(), bag_offsets.data_ptr(), nb, n,
                                                 slot_of.data_ptr(), psw, POOL_MODES[mode], send.data_ptr(),
                                                 fact.data_ptr() if fact is not None else 0, _stream(stream)))
    return send, fact
