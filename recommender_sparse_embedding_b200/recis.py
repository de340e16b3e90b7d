"""Thin ctypes binding of librecis.so (include/recis.h).

Argument marshalling only: every step of the embedding path runs in the CUDA
library.  Device buffers are torch CUDA tensors (their data pointers are passed
as raw device addresses) and streams are torch CUDA streams.  There is no CPU
fallback: if the library or a GPU is missing, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librecis.so")

OK = 0
ERR_INVALID_ARG, ERR_OOM, ERR_TABLE_FULL, ERR_RESERVED_KEY, ERR_CUDA, ERR_TIMEOUT, ERR_NO_DEVICE = (
    1, 2, 3, 4, 5, 6, 7)
BUCKETIZE, HASH, MOD, TAG, FLOAT = 1, 2, 4, 8, 16
ADAGRAD, ADAM = 0, 1
SUM, MEAN = 0, 1
PLACE_BLOCKS_HOST, PLACE_IDMAP_HOST = 1, 2

# every entry point declared in include/recis.h
EXPORTS = (
    "recis_feature_hash", "recis_feature_status_sync", "recis_table_create",
    "recis_table_destroy", "recis_batch_create", "recis_batch_destroy", "recis_lookup_pooled",
    "recis_backward_update", "recis_table_insert", "recis_table_size", "recis_table_export",
    "recis_table_import", "recis_table_status_sync", "recis_batch_get_unique",
    "recis_profile_enable", "recis_profile_collect", "recis_launch_count",
    "recis_last_error_string", "recis_unique_static", "recis_table_read_rows",
    "recis_debug_set", "recis_plan_tables", "recis_table_reserve", "recis_table_save",
    "recis_table_load", "recis_table_evict", "recis_table_clock", "recis_batch_dedup",
    "recis_partition_keys", "recis_pool_rows", "recis_reduce_grad",
)
DEBUG_SPIN_LIMIT, DEBUG_MAP_LIMIT = 1, 2


class RecisError(RuntimeError):
    def __init__(self, code: int, what: str, detail: str = ""):
        super().__init__(f"{what}: status {code}" + (f" ({detail})" if detail else ""))
        self.code = code


class FeatureOp(ctypes.Structure):
    _fields_ = [
        ("flags", ctypes.c_uint32),
        ("n_bound", ctypes.c_int32),
        ("hash_seed", ctypes.c_uint64),
        ("mod", ctypes.c_uint64),
        ("tag", ctypes.c_uint64),
        ("tag_shift", ctypes.c_int32),
        ("reserved_", ctypes.c_int32),
        ("boundaries", ctypes.c_void_p),
    ]


class TableConfig(ctypes.Structure):
    _fields_ = [
        ("dim", ctypes.c_int32),
        ("optimizer", ctypes.c_int32),
        ("lr", ctypes.c_double),
        ("beta1", ctypes.c_double),
        ("beta2", ctypes.c_double),
        ("eps", ctypes.c_double),
        ("adagrad_init_acc", ctypes.c_double),
        ("init_scale", ctypes.c_double),
        ("init_seed", ctypes.c_uint64),
        ("initial_capacity", ctypes.c_int64),
        ("block_rows", ctypes.c_int64),
        ("max_rows", ctypes.c_int64),
        ("admit_threshold", ctypes.c_int32),
        ("evictable", ctypes.c_int32),
        ("placement", ctypes.c_int32),
        ("reserved_", ctypes.c_int32),
    ]


class FeatureSpec(ctypes.Structure):
    _fields_ = [("table", TableConfig), ("value_bits", ctypes.c_int32),
                ("reserved_", ctypes.c_int32)]


_lib = None
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32


def load(path: str = LIB_PATH):
    """Load librecis.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"librecis.so is not built ({path}); run "
                               "recommender_sparse_embedding_b200.build.build()")
        L = ctypes.CDLL(path)
        sig = {
            "recis_feature_hash": [_vp, _i32, _vp, _vp, _vp, _vp],
            "recis_feature_status_sync": [_vp],
            "recis_table_create": [_vp, _vp, _vp],
            "recis_table_destroy": [_vp],
            "recis_batch_create": [_vp],
            "recis_batch_destroy": [_vp],
            "recis_lookup_pooled": [_vp, _vp, _vp, _i64, _vp, _i32, _i64, _i32, _vp, _vp, _vp],
            "recis_backward_update": [_vp, _vp, _vp, _vp, _vp],
            "recis_table_insert": [_vp, _vp, _vp, _i64, _vp, _vp],
            "recis_table_size": [_vp, _vp, _vp, _vp],
            "recis_table_export": [_vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp],
            "recis_table_import": [_vp, _vp, _vp, _vp, _i64, _i64, _vp],
            "recis_table_status_sync": [_vp, _vp],
            "recis_batch_get_unique": [_vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp],
            "recis_profile_enable": [_i32],
            "recis_profile_collect": [_vp, _vp, _vp, _i32],
            "recis_launch_count": [],
            "recis_last_error_string": [],
            "recis_unique_static": [_vp, _i64, _vp, _vp, _vp, _vp],
            "recis_table_read_rows": [_vp, _vp, _i64, _vp, _vp, _vp, _vp],
            "recis_debug_set": [_i32, _i64],
            "recis_plan_tables": [_vp, _i32, _vp, _vp, _vp, _vp, _vp],
            "recis_table_reserve": [_vp, _i64, _vp],
            "recis_table_save": [_vp, ctypes.c_char_p, _vp],
            "recis_table_load": [_vp, ctypes.c_char_p, _vp],
            "recis_table_evict": [_vp, _i64, _vp, _vp],
            "recis_table_clock": [_vp, _vp],
            "recis_batch_dedup": [_vp, _vp, _i64, _vp, _vp, _vp, _vp],
            "recis_partition_keys": [_vp, _vp, _i64, _i32, ctypes.c_uint64, _vp, _vp, _vp, _vp],
            "recis_pool_rows": [_vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _vp, _vp],
            "recis_reduce_grad": [_vp, _vp, _i32, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.recis_launch_count.restype = ctypes.c_int64
        L.recis_last_error_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(rc: int, what: str):
    if rc != OK:
        detail = load().recis_last_error_string()
        raise RecisError(rc, what, detail.decode() if detail else "")


def _dev(t: Optional[torch.Tensor], dtype=None) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


@dataclass
class Feature:
    """One feature's transform (flags from BUCKETIZE, HASH, MOD, TAG, FLOAT).
    BUCKETIZE | FLOAT: float64 boundaries, and the feature's values are
    float64 bit patterns in the int64 values tensor (x.view(torch.int64))."""
    flags: int = 0
    hash_seed: int = 0
    mod: int = 0
    tag: int = 0
    tag_shift: int = 48
    boundaries: Optional[torch.Tensor] = None  # device int64 (float64 with FLOAT), sorted


def feature_hash(features: Sequence[Feature], values: torch.Tensor, feat_offsets: Sequence[int],
                 keys_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """recis_feature_hash: fused hash/mod/bucketize/tag of all features."""
    L = load()
    F = len(features)
    ops = (FeatureOp * max(F, 1))()
    for f, ft in enumerate(features):
        ops[f].flags = ft.flags
        ops[f].hash_seed = ft.hash_seed & (2**64 - 1)
        ops[f].mod = ft.mod
        ops[f].tag = ft.tag
        ops[f].tag_shift = ft.tag_shift
        if ft.boundaries is not None:
            ops[f].n_bound = ft.boundaries.numel()
            ops[f].boundaries = _dev(ft.boundaries, torch.float64 if ft.flags & FLOAT else torch.int64)
    offs = (ctypes.c_int64 * (F + 1))(*[int(x) for x in feat_offsets])
    if keys_out is None:
        keys_out = torch.empty_like(values)
    _check(L.recis_feature_hash(ops, F, _dev(values, torch.int64), offs,
                                _dev(keys_out, torch.int64), _stream(stream)), "recis_feature_hash")
    return keys_out


def feature_status_sync(stream=None):
    _check(load().recis_feature_status_sync(_stream(stream)), "recis_feature_status_sync")


class Batch:
    """recis_batch_t: per-step scratch of one lookup, reused across steps."""

    def __init__(self):
        h = ctypes.c_void_p()
        _check(load().recis_batch_create(ctypes.byref(h)), "recis_batch_create")
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            load().recis_batch_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def get_unique(self, n_occ: int, capacity: Optional[int] = None, stream=None):
        """(uniq int64[U], inv int32[N], rows int64[U], n_new) of the last lookup."""
        L = load()
        dev = torch.cuda.current_device()
        cap = n_occ if capacity is None else capacity
        uniq = torch.empty(max(cap, 1), dtype=torch.int64, device=dev)
        rows = torch.empty(max(cap, 1), dtype=torch.int64, device=dev)
        inv = torch.empty(max(n_occ, 1), dtype=torch.int32, device=dev)
        U, nn = ctypes.c_int64(), ctypes.c_int64()
        _check(L.recis_batch_get_unique(self.handle, uniq.data_ptr(), inv.data_ptr(),
                                        rows.data_ptr(), cap, ctypes.byref(U), ctypes.byref(nn),
                                        _stream(stream)), "recis_batch_get_unique")
        return uniq[: U.value], inv[:n_occ], rows[: U.value], nn.value


class Table:
    """recis_table_t: one logical (merged) embedding table."""

    def __init__(self, dim: int, optimizer: int, lr: float, beta1: float = 0.9,
                 beta2: float = 0.999, eps: Optional[float] = None, adagrad_init_acc: float = 0.0,
                 init_scale: float = 0.0, init_seed: int = 0, initial_capacity: int = 0,
                 block_rows: int = 0, max_rows: int = 0, admit_threshold: int = 0,
                 evictable: bool = False, placement: int = 0, stream=None):
        if eps is None:
            eps = 1e-10 if optimizer == ADAGRAD else 1e-8
        cfg = TableConfig(dim=dim, optimizer=optimizer, lr=lr, beta1=beta1, beta2=beta2, eps=eps,
                          adagrad_init_acc=adagrad_init_acc, init_scale=init_scale,
                          init_seed=init_seed & (2**64 - 1), initial_capacity=initial_capacity,
                          block_rows=block_rows, max_rows=max_rows,
                          admit_threshold=admit_threshold, evictable=1 if evictable else 0,
                          placement=placement)
        h = ctypes.c_void_p()
        _check(load().recis_table_create(ctypes.byref(cfg), _stream(stream), ctypes.byref(h)),
               "recis_table_create")
        self.handle = h
        self.dim = dim
        self.optimizer = optimizer
        self.s = 1 if optimizer == ADAGRAD else 2

    def close(self):
        if getattr(self, "handle", None):
            load().recis_table_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def lookup_pooled(self, batch: Batch, keys: torch.Tensor, bag_offsets: torch.Tensor, F: int,
                      B: int, combiner: int = SUM, pooled_out: Optional[torch.Tensor] = None,
                      unpooled_out: Optional[torch.Tensor] = None, stream=None):
        _check(load().recis_lookup_pooled(
            self.handle, batch.handle, _dev(keys, torch.int64), keys.numel(),
            _dev(bag_offsets, torch.int64), F, B, combiner, _dev(pooled_out, torch.float32),
            _dev(unpooled_out, torch.float32), _stream(stream)), "recis_lookup_pooled")
        return pooled_out, unpooled_out

    def backward_update(self, batch: Batch, grad_pooled: Optional[torch.Tensor] = None,
                        grad_unpooled: Optional[torch.Tensor] = None, stream=None):
        _check(load().recis_backward_update(self.handle, batch.handle,
                                            _dev(grad_pooled, torch.float32),
                                            _dev(grad_unpooled, torch.float32), _stream(stream)),
               "recis_backward_update")

    def insert(self, batch: Batch, keys: torch.Tensor, rows_out: Optional[torch.Tensor] = None,
               stream=None):
        _check(load().recis_table_insert(self.handle, batch.handle, _dev(keys, torch.int64),
                                         keys.numel(), _dev(rows_out, torch.int64),
                                         _stream(stream)), "recis_table_insert")
        return rows_out

    def evict(self, min_clock: int, stream=None) -> int:
        """recis_table_evict: remove keys last touched before lookup `min_clock`;
        returns the rows freed."""
        n = ctypes.c_int64()
        _check(load().recis_table_evict(self.handle, min_clock, ctypes.byref(n), _stream(stream)),
               "recis_table_evict")
        return n.value

    @property
    def clock(self) -> int:
        c = ctypes.c_int64()
        _check(load().recis_table_clock(self.handle, ctypes.byref(c)), "recis_table_clock")
        return c.value

    def reserve(self, rows: int, stream=None):
        """recis_table_reserve: room for `rows` live rows in total, mapped now."""
        _check(load().recis_table_reserve(self.handle, rows, _stream(stream)), "recis_table_reserve")

    def size(self, stream=None):
        n, st = ctypes.c_int64(), ctypes.c_int64()
        _check(load().recis_table_size(self.handle, ctypes.byref(n), ctypes.byref(st),
                                       _stream(stream)), "recis_table_size")
        return n.value, st.value

    def status_sync(self, stream=None):
        _check(load().recis_table_status_sync(self.handle, _stream(stream)), "recis_table_status_sync")

    def export(self, stream=None):
        """(keys int64[n], emb fp32[n, D], state fp32[n, s*D], step) as numpy arrays."""
        import numpy as np
        n, _ = self.size(stream)
        keys = np.empty(max(n, 1), np.int64)
        emb = np.empty((max(n, 1), self.dim), np.float32)
        st = np.empty((max(n, 1), self.s * self.dim), np.float32)
        n_out, step = ctypes.c_int64(), ctypes.c_int64()
        _check(load().recis_table_export(self.handle, keys.ctypes.data, emb.ctypes.data,
                                         st.ctypes.data, n, ctypes.byref(n_out),
                                         ctypes.byref(step), _stream(stream)), "recis_table_export")
        return keys[:n], emb[:n], st[:n], step.value

    def read_rows(self, rows: torch.Tensor, stream=None):
        """(keys int64[n], emb fp32[n, D], state fp32[n, s*D]) of the given row
        offsets (device int64), gathered on the device."""
        n = rows.numel()
        dev = rows.device
        keys = torch.empty(max(n, 1), dtype=torch.int64, device=dev)
        emb = torch.empty((max(n, 1), self.dim), dtype=torch.float32, device=dev)
        st = torch.empty((max(n, 1), self.s * self.dim), dtype=torch.float32, device=dev)
        _check(load().recis_table_read_rows(self.handle, _dev(rows, torch.int64), n, keys.data_ptr(),
                                            emb.data_ptr(), st.data_ptr(), _stream(stream)),
               "recis_table_read_rows")
        return keys[:n], emb[:n], st[:n]

    def save(self, path: str, stream=None):
        """recis_table_save: the table as a SafeTensors file."""
        _check(load().recis_table_save(self.handle, os.fsencode(path), _stream(stream)),
               "recis_table_save")

    def load_file(self, path: str, stream=None):
        """recis_table_load: append the rows of a SafeTensors file."""
        _check(load().recis_table_load(self.handle, os.fsencode(path), _stream(stream)),
               "recis_table_load")

    def import_rows(self, keys, emb, state=None, step: int = 0, stream=None):
        import numpy as np
        keys = np.ascontiguousarray(keys, np.int64)
        emb = np.ascontiguousarray(emb, np.float32)
        st = None if state is None else np.ascontiguousarray(state, np.float32)
        _check(load().recis_table_import(self.handle, keys.ctypes.data, emb.ctypes.data,
                                         None if st is None else st.ctypes.data, len(keys), step,
                                         _stream(stream)), "recis_table_import")


def unique_static(keys: torch.Tensor, stream=None):
    """recis_unique_static: allocation-free dedup (N <= 262144).

    Returns (uniq int64[N] buffer, inv int32[N], U int64[1]) on the device; the
    first U entries of uniq are the unique keys.  The output tensors are
    allocated here by torch, not by the library."""
    n = keys.numel()
    uniq = torch.empty(max(n, 1), dtype=torch.int64, device=keys.device)
    inv = torch.empty(max(n, 1), dtype=torch.int32, device=keys.device)
    U = torch.empty(1, dtype=torch.int64, device=keys.device)
    _check(load().recis_unique_static(_dev(keys, torch.int64), n, uniq.data_ptr(), inv.data_ptr(),
                                      U.data_ptr(), _stream(stream)), "recis_unique_static")
    return uniq, inv, U


@dataclass
class TablePlan:
    """Result of plan_tables: per feature its logical table, tag and tag shift;
    per logical table its merged configuration (a TableConfig)."""
    table_of: list
    tag_of: list
    tag_shift_of: list
    tables: list


def plan_tables(features) -> TablePlan:
    """recis_plan_tables (host only): merge features whose table attributes
    are equal into logical tables.  features: sequence of (TableConfig,
    value_bits) pairs."""
    F = len(features)
    arr = (FeatureSpec * max(F, 1))()
    for f, (cfg, bits) in enumerate(features):
        arr[f].table = cfg
        arr[f].value_bits = bits
    table_of = (ctypes.c_int32 * max(F, 1))()
    tag_of = (ctypes.c_uint64 * max(F, 1))()
    shift_of = (ctypes.c_int32 * max(F, 1))()
    tabs = (TableConfig * max(F, 1))()
    n = ctypes.c_int32(0)
    _check(load().recis_plan_tables(arr, F, table_of, tag_of, shift_of, tabs, ctypes.byref(n)),
           "recis_plan_tables")
    return TablePlan(list(table_of[:F]), list(tag_of[:F]), list(shift_of[:F]),
                     [tabs[i] for i in range(n.value)])


def table_config(dim: int, optimizer: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
                 eps: Optional[float] = None, adagrad_init_acc: float = 0.0,
                 init_scale: float = 0.0, init_seed: int = 0, initial_capacity: int = 0,
                 block_rows: int = 0, max_rows: int = 0) -> TableConfig:
    """A recis_table_config with the library's usual defaults."""
    if eps is None:
        eps = 1e-10 if optimizer == ADAGRAD else 1e-8
    return TableConfig(dim=dim, optimizer=optimizer, lr=lr, beta1=beta1, beta2=beta2, eps=eps,
                       adagrad_init_acc=adagrad_init_acc, init_scale=init_scale,
                       init_seed=init_seed & (2**64 - 1), initial_capacity=initial_capacity,
                       block_rows=block_rows, max_rows=max_rows)


def debug_set(what: int, value: int):
    """recis_debug_set: test hooks (DEBUG_SPIN_LIMIT, DEBUG_MAP_LIMIT; 0 = default)."""
    _check(load().recis_debug_set(what, value), "recis_debug_set")


def profile_enable(on: bool = True):
    _check(load().recis_profile_enable(1 if on else 0), "recis_profile_enable")


def profile_collect(max_names: int = 64):
    """{kernel name: (launches, total ms)} since the last collect (synchronous)."""
    L = load()
    names = (ctypes.c_char_p * max_names)()
    cnt = (ctypes.c_int64 * max_names)()
    ms = (ctypes.c_double * max_names)()
    n = L.recis_profile_collect(names, cnt, ms, max_names)
    return {names[i].decode(): (cnt[i], ms[i]) for i in range(n)}


def launch_count() -> int:
    return int(load().recis_launch_count())
