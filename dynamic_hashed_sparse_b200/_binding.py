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
from typing import Optional, Tuple

import numpy as np
import torch

from . import build as _build

STATUS = {
    0: "ok", 1: "invalid argument", 2: "out of device memory", 3: "CUDA error",
    4: "table full", 5: "key not found", 6: "unsupported", 7: "internal wait bound exceeded",
}
OPT_CODES = {"sgd": 0, "adagrad": 1, "adam": 2, "adagrad_rowwise": 3}
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
        "ht_destroy": (C.c_int, [vp]),
        "ht_reserve": (C.c_int, [vp, i64, vp]),
        "ht_lookup_or_insert": (C.c_int, [vp, vp, i64, vp, vp]),
        "ht_lookup": (C.c_int, [vp, vp, i64, vp, vp]),
        "embbag_forward": (C.c_int, [vp, vp, i64, vp, i64, vp, vp]),
        "embbag_backward_update": (C.c_int, [vp, vp, i64, vp, i64, vp, f32, vp]),
        "embbag_backward_update_noalloc": (C.c_int, [vp, vp, i64, vp, i64, vp, f32, vp]),
        "ht_get_rows": (C.c_int, [vp, vp, i64, vp, vp]),
        "ht_row_stride": (i64, [vp]),
        "ht_sync": (C.c_int, [vp]),
        "ht_size": (C.c_int, [vp, C.POINTER(i64)]),
        "ht_export": (C.c_int, [vp, vp, vp]),
        "ht_counters": (C.c_int, [vp, vp]),
        "ht_set_phase_timing": (C.c_int, [vp, C.c_int]),
        "ht_phase_times": (C.c_int, [vp, vp, vp, C.c_int]),
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

    def __init__(self, handle: int, dim: int, optimizer: str, device: torch.device):
        self.handle = handle
        self.dim = dim
        self.optimizer = optimizer
        self.device = device
        self.stride = int(_lib.ht_row_stride(handle))

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
              device=None) -> Table:
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    p = _OptParams(eps, beta1, beta2)
    h = C.c_void_p()
    with torch.cuda.device(device):
        rc = _lib.ht_create(int(dim), OPT_CODES[optimizer], int(block_rows), int(max_rows),
                            C.byref(p), None, C.byref(h))
    _check("ht_create", rc)
    return Table(h.value, int(dim), optimizer, device)


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


NOALLOC_MAX_KEYS = 131072


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


def ht_row_stride(t: Table) -> int:
    return int(_lib.ht_row_stride(t.handle))


def ht_sync(t: Table) -> int:
    """Wait for the table's work; returns (and clears) the latched device status."""
    return int(_lib.ht_sync(t.handle))


def ht_size(t: Table) -> Tuple[int, int]:
    n = C.c_int64()
    rc = _lib.ht_size(t.handle, C.byref(n))
    return int(n.value), int(rc)


def ht_export(t: Table) -> Tuple[np.ndarray, np.ndarray, int]:
    n, rc = ht_size(t)
    keys = np.empty(n, np.int64)
    rows = np.empty((n, t.stride), np.float32)
    rc2 = _lib.ht_export(t.handle, keys.ctypes.data, rows.ctypes.data)
    return keys, rows, int(rc or rc2)


def ht_counters(t: Table) -> dict:
    out = np.zeros(14, np.int64)
    _check("ht_counters", _lib.ht_counters(t.handle, out.ctypes.data))
    names = ("rows", "inserted", "unique_updated", "insert_calls", "backward_calls", "slots",
             "blocks", "rehashes", "launches", "last_inserted", "host_waits", "host_wait_ns",
             "allocs", "alloc_ns")
    return {k: int(v) for k, v in zip(names, out)}


def ht_set_phase_timing(t: Table, enable: bool):
    _check("ht_set_phase_timing", _lib.ht_set_phase_timing(t.handle, int(bool(enable))))


def ht_phase_times(t: Table) -> dict:
    ms = np.zeros(len(PHASES), np.float64)
    cnt = np.zeros(len(PHASES), np.int64)
    _check("ht_phase_times", _lib.ht_phase_times(t.handle, ms.ctypes.data, cnt.ctypes.data, len(PHASES)))
    return {p: (float(m), int(c)) for p, m, c in zip(PHASES, ms, cnt)}
