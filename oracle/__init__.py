"""CPU oracle of the RecIS dynamic-hash embedding step -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
binding) never does.  It wraps ``liboracle.so`` (built from ``oracle.cpp`` with
``build()``) through ctypes; every function below is argument marshalling only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")

OK, INVALID_ARG, RESERVED_KEY = 0, 1, 2
BUCKETIZE, HASH, MOD, TAG, FLOAT = 1, 2, 4, 8, 16
ADAGRAD, ADAM = 0, 1
SUM, MEAN = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (no fast-math, no FMA contraction)."""
    src = os.path.join(_HERE, "oracle.cpp")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(
        os.path.getmtime(src), os.path.getmtime(os.path.join(_HERE, "oracle.h"))
    ):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math",
             "-shared", "-fPIC", "-o", tmp, src]
        )
        os.replace(tmp, _SO)
    return _SO


class _FeatureOp(ctypes.Structure):
    _fields_ = [
        ("flags", ctypes.c_uint32),
        ("n_bound", ctypes.c_int32),
        ("hash_seed", ctypes.c_uint64),
        ("mod", ctypes.c_uint64),
        ("tag", ctypes.c_uint64),
        ("tag_shift", ctypes.c_int32),
        ("pad_", ctypes.c_int32),
        ("boundaries", ctypes.POINTER(ctypes.c_int64)),
    ]


def _ptr(a: Optional[np.ndarray], ctype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        L.orc_hash64.restype = ctypes.c_uint64
        L.orc_hash64.argtypes = [ctypes.c_uint64]
        L.orc_feature_hash.restype = ctypes.c_int
        L.orc_table_new.restype = ctypes.c_void_p
        L.orc_table_new.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
                                    ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                    ctypes.c_double, ctypes.c_uint64, ctypes.c_double]
        L.orc_table_free.argtypes = [ctypes.c_void_p]
        L.orc_table_clock.restype = ctypes.c_int64
        L.orc_table_clock.argtypes = [ctypes.c_void_p]
        L.orc_table_set_admission.argtypes = [ctypes.c_void_p, ctypes.c_int32]
        L.orc_table_evict.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.orc_lookup.restype = ctypes.c_int
        L.orc_lookup.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64), ctypes.c_int64,
                                 ctypes.POINTER(ctypes.c_int64), ctypes.c_int32, ctypes.c_int64,
                                 ctypes.c_int32, ctypes.POINTER(ctypes.c_float),
                                 ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int64),
                                 ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64),
                                 ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64)]
        L.orc_backward_update.restype = ctypes.c_int
        L.orc_backward_update.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_float),
                                          ctypes.POINTER(ctypes.c_float),
                                          ctypes.POINTER(ctypes.c_double)]
        L.orc_table_size.restype = ctypes.c_int64
        L.orc_table_size.argtypes = [ctypes.c_void_p]
        L.orc_table_step.restype = ctypes.c_int64
        L.orc_table_step.argtypes = [ctypes.c_void_p]
        L.orc_table_export.restype = ctypes.c_int
        L.orc_table_export.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64),
                                       ctypes.POINTER(ctypes.c_float),
                                       ctypes.POINTER(ctypes.c_float)]
        L.orc_table_import.restype = ctypes.c_int
        L.orc_table_import.argtypes = [ctypes.c_void_p, ctypes.c_int64,
                                       ctypes.POINTER(ctypes.c_int64),
                                       ctypes.POINTER(ctypes.c_float),
                                       ctypes.POINTER(ctypes.c_float), ctypes.c_int64]
        _lib = L
    return _lib


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} returned status {code}")
        self.code = code


def hash64(x: int) -> int:
    return int(lib().orc_hash64(ctypes.c_uint64(x & (2**64 - 1))))


@dataclass
class FeatureOp:
    """One feature's transform: flags from {BUCKETIZE, HASH, MOD, TAG, FLOAT}.
    With BUCKETIZE | FLOAT the boundaries are floats and the values are
    float64 bit patterns held in the int64 array."""
    flags: int = 0
    hash_seed: int = 0
    mod: int = 0
    tag: int = 0
    tag_shift: int = 48
    boundaries: Sequence[int] = field(default_factory=list)


def feature_hash(ops: Sequence[FeatureOp], values: np.ndarray, feat_offsets: np.ndarray) -> np.ndarray:
    F = len(ops)
    values = np.ascontiguousarray(values, dtype=np.int64)
    feat_offsets = np.ascontiguousarray(feat_offsets, dtype=np.int64)
    arr = (_FeatureOp * max(F, 1))()
    keep = []
    for f, op in enumerate(ops):
        if op.flags & FLOAT:
            b = np.ascontiguousarray(np.asarray(op.boundaries, dtype=np.float64)).view(np.int64)
        else:
            b = np.ascontiguousarray(np.asarray(op.boundaries, dtype=np.int64))
        keep.append(b)
        arr[f].flags = op.flags
        arr[f].n_bound = len(b)
        arr[f].hash_seed = op.hash_seed & (2**64 - 1)
        arr[f].mod = op.mod
        arr[f].tag = op.tag
        arr[f].tag_shift = op.tag_shift
        arr[f].boundaries = _ptr(b, ctypes.c_int64) if len(b) else None
    out = np.empty_like(values)
    rc = lib().orc_feature_hash(arr, ctypes.c_int32(F), _ptr(values, ctypes.c_int64),
                                _ptr(feat_offsets, ctypes.c_int64), _ptr(out, ctypes.c_int64))
    if rc != OK:
        raise OracleError(rc, "feature_hash")
    return out


@dataclass
class LookupResult:
    pooled: Optional[np.ndarray]
    unpooled: Optional[np.ndarray]
    uniq: np.ndarray
    inv: np.ndarray
    rows: np.ndarray
    n_new: int


class Table:
    """One logical (merged) embedding table of the oracle."""

    def __init__(self, dim: int, optimizer: int, lr: float, beta1: float = 0.9,
                 beta2: float = 0.999, eps: Optional[float] = None,
                 adagrad_init_acc: float = 0.0, init_seed: int = 0,
                 init_scale: Optional[float] = None, admit_threshold: int = 0):
        if eps is None:
            eps = 1e-10 if optimizer == ADAGRAD else 1e-8
        if init_scale is None:
            init_scale = 1.0 / np.sqrt(dim)
        self.dim, self.optimizer = dim, optimizer
        self.s = 1 if optimizer == ADAGRAD else 2
        self._h = lib().orc_table_new(dim, optimizer, lr, beta1, beta2, eps, adagrad_init_acc,
                                      ctypes.c_uint64(init_seed & (2**64 - 1)), init_scale)
        if not self._h:
            raise OracleError(INVALID_ARG, "table_new")
        if admit_threshold:
            lib().orc_table_set_admission(self._h, admit_threshold)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lib is not None:
            _lib.orc_table_free(h)
            self._h = None

    def lookup(self, keys: np.ndarray, bag_offsets: np.ndarray, F: int, B: int,
               combiner: int = SUM, pooled: bool = True, unpooled: bool = False) -> LookupResult:
        keys = np.ascontiguousarray(keys, dtype=np.int64)
        bag_offsets = np.ascontiguousarray(bag_offsets, dtype=np.int64)
        N, D = len(keys), self.dim
        po = np.empty((B, F, D), np.float32) if pooled else None
        uo = np.empty((N, D), np.float32) if unpooled else None
        uniq = np.empty(max(N, 1), np.int64)
        rows = np.empty(max(N, 1), np.int64)
        inv = np.empty(max(N, 1), np.int32)
        U = ctypes.c_int64(0)
        nn = ctypes.c_int64(0)
        rc = lib().orc_lookup(self._h, _ptr(keys, ctypes.c_int64), N,
                              _ptr(bag_offsets, ctypes.c_int64), F, B, combiner,
                              _ptr(po, ctypes.c_float), _ptr(uo, ctypes.c_float),
                              _ptr(uniq, ctypes.c_int64), _ptr(inv, ctypes.c_int32),
                              _ptr(rows, ctypes.c_int64), ctypes.byref(U), ctypes.byref(nn))
        if rc != OK:
            raise OracleError(rc, "lookup")
        return LookupResult(po, uo, uniq[: U.value].copy(), inv[:N].copy(),
                            rows[: U.value].copy(), nn.value)

    def backward_update(self, grad_pooled: Optional[np.ndarray] = None,
                        grad_unpooled: Optional[np.ndarray] = None,
                        return_grad: bool = False, n_unique: int = 0):
        gp = None if grad_pooled is None else np.ascontiguousarray(grad_pooled, np.float32)
        gu = None if grad_unpooled is None else np.ascontiguousarray(grad_unpooled, np.float32)
        gout = np.empty((max(n_unique, 1), self.dim), np.float64) if return_grad else None
        rc = lib().orc_backward_update(self._h, _ptr(gp, ctypes.c_float), _ptr(gu, ctypes.c_float),
                                       _ptr(gout, ctypes.c_double))
        if rc != OK:
            raise OracleError(rc, "backward_update")
        return gout[:n_unique] if return_grad else None

    @property
    def size(self) -> int:
        return int(lib().orc_table_size(self._h))

    @property
    def step(self) -> int:
        return int(lib().orc_table_step(self._h))

    @property
    def clock(self) -> int:
        return int(lib().orc_table_clock(self._h))

    def evict(self, min_clock: int) -> int:
        """Remove rows and candidates last touched before lookup `min_clock`."""
        n = ctypes.c_int64(0)
        rc = lib().orc_table_evict(self._h, ctypes.c_int64(min_clock), ctypes.byref(n))
        if rc != OK:
            raise OracleError(rc, "evict")
        return n.value

    def export(self):
        n, D = self.size, self.dim
        keys = np.empty(max(n, 1), np.int64)
        emb = np.empty((max(n, 1), D), np.float32)
        st = np.empty((max(n, 1), self.s * D), np.float32)
        lib().orc_table_export(self._h, _ptr(keys, ctypes.c_int64), _ptr(emb, ctypes.c_float),
                               _ptr(st, ctypes.c_float))
        return keys[:n].copy(), emb[:n].copy(), st[:n].copy()

    def import_rows(self, keys: np.ndarray, emb: np.ndarray, state: Optional[np.ndarray] = None,
                    step: int = 0):
        keys = np.ascontiguousarray(keys, np.int64)
        emb = np.ascontiguousarray(emb, np.float32)
        st = None if state is None else np.ascontiguousarray(state, np.float32)
        rc = lib().orc_table_import(self._h, len(keys), _ptr(keys, ctypes.c_int64),
                                    _ptr(emb, ctypes.c_float), _ptr(st, ctypes.c_float), step)
        if rc != OK:
            raise OracleError(rc, "import")


class _FeatureAttrs(ctypes.Structure):
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
        ("capacity", ctypes.c_int64),
        ("value_bits", ctypes.c_int32),
        ("pad_", ctypes.c_int32),
    ]


def plan_tables(features):
    """Table merging of the oracle.  features: sequence of dicts with keys dim,
    optimizer, lr, beta1, beta2, eps, adagrad_init_acc, init_scale, init_seed,
    capacity, value_bits.  Returns (table_of, tag_of, shift_of, capacities)."""
    F = len(features)
    arr = (_FeatureAttrs * max(F, 1))()
    for f, a in enumerate(features):
        for k, v in a.items():
            setattr(arr[f], k, v)
    table_of = np.empty(max(F, 1), np.int32)
    tag_of = np.empty(max(F, 1), np.uint64)
    shift_of = np.empty(max(F, 1), np.int32)
    caps = np.empty(max(F, 1), np.int64)
    n = ctypes.c_int32(0)
    rc = lib().orc_plan_tables(arr, F, _ptr(table_of, ctypes.c_int32), _ptr(tag_of, ctypes.c_uint64),
                               _ptr(shift_of, ctypes.c_int32), _ptr(caps, ctypes.c_int64),
                               ctypes.byref(n))
    if rc != OK:
        raise OracleError(rc, "plan_tables")
    return table_of[:F].copy(), tag_of[:F].copy(), shift_of[:F].copy(), caps[: n.value].copy()
