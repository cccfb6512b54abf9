"""ctypes wrapper of oracle/liboracle.so (test infrastructure only).

Each method marshals numpy arrays into the C oracle; every computation happens
in oracle.cpp, whose header states the definitions it follows.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

OPT_CODES = {"sgd": 0, "adagrad": 1, "adam": 2, "adagrad_rowwise": 3}
MODES = {"sum": 0, "mean": 1}
STORAGE = {"f32": 0, "bf16": 1}
_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        i64, i32, f32, vp = C.c_int64, C.c_int32, C.c_float, C.c_void_p
        L.orc_splitmix64_next.restype = C.c_uint64
        L.orc_splitmix64_next.argtypes = [C.POINTER(C.c_uint64)]
        L.orc_init_row.argtypes = [i64, C.c_int, vp]
        L.orc_pack_keys.restype = C.c_int
        L.orc_pack_keys.argtypes = [vp, vp, i64, vp]
        L.orc_create.restype = vp
        L.orc_create.argtypes = [C.c_int, C.c_int, f32, f32, f32]
        L.orc_create_ex.restype = vp
        L.orc_create_ex.argtypes = [C.c_int, C.c_int, f32, f32, f32, C.c_int]
        L.orc_round_bf16.restype = f32
        L.orc_round_bf16.argtypes = [f32]
        L.orc_destroy.argtypes = [vp]
        L.orc_size.restype = i64
        L.orc_size.argtypes = [vp]
        L.orc_stride.restype = i64
        L.orc_stride.argtypes = [vp]
        L.orc_lookup_or_insert.restype = C.c_int
        L.orc_lookup_or_insert.argtypes = [vp, vp, i64, vp]
        L.orc_lookup.argtypes = [vp, vp, i64, vp]
        L.orc_forward.restype = C.c_int
        L.orc_forward.argtypes = [vp, vp, vp, i64, vp]
        L.orc_backward_update.restype = C.c_int
        L.orc_backward_update.argtypes = [vp, vp, vp, i64, vp, f32]
        L.orc_forward_ex.restype = C.c_int
        L.orc_forward_ex.argtypes = [vp, vp, vp, i64, vp, C.c_int, vp]
        L.orc_backward_update_ex.restype = C.c_int
        L.orc_backward_update_ex.argtypes = [vp, vp, vp, i64, vp, C.c_int, vp, f32]
        L.orc_export.argtypes = [vp, vp, vp]
        L.orc_import_rows.argtypes = [vp, vp, i64]
        L.orc_set_hooks.argtypes = [vp, i64, C.c_int]
        L.orc_evict.restype = i64
        L.orc_evict.argtypes = [vp, i64]
        L.orc_live.restype = i64
        L.orc_live.argtypes = [vp]
        L.orc_get_rows.restype = i64
        L.orc_get_rows.argtypes = [vp, vp, i64, vp]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def splitmix64_outputs(seed: int, n: int) -> list:
    s = C.c_uint64(seed & (2**64 - 1))
    return [int(lib().orc_splitmix64_next(C.byref(s))) for _ in range(n)]


def init_row(key: int, dim: int) -> np.ndarray:
    out = np.empty(dim, np.float32)
    lib().orc_init_row(int(key), dim, _p(out))
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    """The oracle's fp32 -> nearest bf16 (widened back to fp32), elementwise."""
    x = np.ascontiguousarray(x, np.float32)
    f = lib().orc_round_bf16
    return np.array([f(float(v)) for v in x.ravel()], np.float32).reshape(x.shape)


def pack_keys(table_ids: np.ndarray, ids: np.ndarray):
    t = np.ascontiguousarray(table_ids, np.int32)
    i = np.ascontiguousarray(ids, np.int64)
    out = np.empty(i.shape[0], np.int64)
    rc = lib().orc_pack_keys(_p(t), _p(i), i.shape[0], _p(out))
    return out, rc


class Oracle:
    """std::unordered_map IDMap + one row vector; sequential loops."""

    def __init__(self, dim: int, optimizer: str = "sgd", eps: float = 1e-8,
                 beta1: float = 0.9, beta2: float = 0.999, storage: str = "f32"):
        self.dim = int(dim)
        self.optimizer = optimizer
        self.storage = storage
        self.h = lib().orc_create_ex(self.dim, OPT_CODES[optimizer], eps, beta1, beta2, STORAGE[storage])
        if not self.h:
            raise ValueError("bad oracle arguments")

    def close(self):
        if self.h:
            lib().orc_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def size(self) -> int:
        """Rows allocated (free rows included)."""
        return int(lib().orc_size(self.h))

    @property
    def live(self) -> int:
        """Keys with a row."""
        return int(lib().orc_live(self.h))

    def set_hooks(self, admit_threshold: int = 1, track_access: bool = False):
        """Admission threshold and access tracking (before the first insert)."""
        lib().orc_set_hooks(self.h, int(admit_threshold), int(bool(track_access)))

    def evict(self, max_idle: int) -> int:
        return int(lib().orc_evict(self.h, int(max_idle)))

    @property
    def stride(self) -> int:
        return int(lib().orc_stride(self.h))

    def lookup_or_insert(self, keys):
        k = np.ascontiguousarray(keys, np.int64)
        out = np.empty(k.shape[0], np.int64)
        rc = lib().orc_lookup_or_insert(self.h, _p(k), k.shape[0], _p(out))
        return out, rc

    def lookup(self, keys):
        k = np.ascontiguousarray(keys, np.int64)
        out = np.empty(k.shape[0], np.int64)
        lib().orc_lookup(self.h, _p(k), k.shape[0], _p(out))
        return out

    def forward(self, keys, bag_offsets, per_sample_weights=None, mode: str = "sum"):
        """EmbeddingBag forward; mode "sum" or "mean"; optional per-sample
        weights (float[n], sum mode only)."""
        k = np.ascontiguousarray(keys, np.int64)
        bo = np.ascontiguousarray(bag_offsets, np.int64)
        nb = bo.shape[0] - 1
        out = np.empty((nb, self.dim), np.float32)
        w = None if per_sample_weights is None else np.ascontiguousarray(per_sample_weights, np.float32)
        rc = lib().orc_forward_ex(self.h, _p(k), _p(bo), nb, _p(w) if w is not None else None,
                                  MODES[mode], _p(out))
        return out, rc

    def backward_update(self, keys, bag_offsets, grad, lr: float, per_sample_weights=None, mode: str = "sum"):
        k = np.ascontiguousarray(keys, np.int64)
        bo = np.ascontiguousarray(bag_offsets, np.int64)
        g = np.ascontiguousarray(grad, np.float32)
        nb = bo.shape[0] - 1
        assert g.shape == (nb, self.dim)
        w = None if per_sample_weights is None else np.ascontiguousarray(per_sample_weights, np.float32)
        return lib().orc_backward_update_ex(self.h, _p(k), _p(bo), nb, _p(w) if w is not None else None,
                                            MODES[mode], _p(g), float(lr))

    def export(self):
        n = self.size
        keys = np.empty(n, np.int64)
        rows = np.empty((n, self.stride), np.float32)
        lib().orc_export(self.h, _p(keys), _p(rows))
        return keys, rows

    def get_rows(self, keys):
        k = np.ascontiguousarray(keys, np.int64)
        out = np.empty((k.shape[0], self.stride), np.float32)
        missing = lib().orc_get_rows(self.h, _p(k), k.shape[0], _p(out))
        return out, int(missing)
