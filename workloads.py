"""Seeded synthetic workloads for the RecIS dynamic-hash embedding step.

This module only draws inputs: feature IDs, bag lengths and upstream
gradients.  It holds none of the embedding step's arithmetic (no feature hash,
no dedup, no pooling, no optimiser), so both the CPU oracle's tests and the CUDA
path can take their inputs from it.

Recipe (one entry of WORKLOADS per workload):
  * IDs: a Zipf(a) rank r in [1, n] (P(r) proportional to r^-a), drawn exactly with
    the rejection-inversion method of Hoermann & Derflinger ("Rejection-inversion
    to generate variates from monotone discrete distributions", ACM TOMACS 1996);
    then mapped to an ID in [0, n) by a per-feature keyed bijection (a 4-round
    Feistel network with cycle walking), so hot ranks land on scattered IDs.
  * Bag lengths per workload: fixed 1 (one-hot), uniform ranges, or geometric.
  * Values are laid out feature-major: all bags of feature 0, then feature 1, ...
    (CSR by feature, then by bag); bag f*B+b is sample b of feature f.
  * Upstream gradients: uniform in [0.5, 1) (no cancellation), or [-1, 1).
  * Seeds: 2025 + workload index, then one stream per batch index.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np

BUCKETIZE, HASH, MOD, TAG, FLOAT = 1, 2, 4, 8, 16
_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)


# --------------------------------------------------------------------------
# Zipf sampler: rejection-inversion (Hoermann & Derflinger 1996)
# --------------------------------------------------------------------------
class Zipf:
    """Exact Zipf(a) on {1..n}, any a > 0, vectorised."""

    def __init__(self, n: int, a: float):
        assert n >= 1 and a > 0
        self.n, self.a = int(n), float(a)
        self._hx1 = self._Hint(1.5) - 1.0
        self._hn = self._Hint(self.n + 0.5)
        self._s = 2.0 - self._Hinv(self._Hint(2.5) - self._h(2.0))

    # h(x) = x^-a; Hint is an antiderivative of h; Hinv its inverse.
    def _h(self, x):
        return np.exp(-self.a * np.log(x))

    def _Hint(self, x):
        lx = np.log(x)
        t = (1.0 - self.a) * lx
        # (exp(t) - 1) / t, continuous at t = 0
        f = np.where(np.abs(t) > 1e-8, np.expm1(t) / np.where(t == 0, 1, t), 1.0 + t / 2.0)
        return f * lx

    def _Hinv(self, y):
        t = y * (1.0 - self.a)
        t = np.maximum(t, -1.0 + 1e-16)
        # log1p(t) / t, continuous at t = 0
        f = np.where(np.abs(t) > 1e-8, np.log1p(t) / np.where(t == 0, 1, t), 1.0 - t / 2.0)
        return np.exp(f * y)

    def sample(self, rng: np.random.Generator, size: int) -> np.ndarray:
        out = np.empty(size, np.int64)
        todo = np.arange(size)
        while todo.size:
            u = self._hn + rng.random(todo.size) * (self._hx1 - self._hn)
            x = self._Hinv(u)
            k = np.clip(np.floor(x + 0.5), 1, self.n)
            ok = (k - x <= self._s) | (u >= self._Hint(k + 0.5) - self._h(k))
            out[todo[ok]] = k[ok].astype(np.int64)
            todo = todo[~ok]
        return out


# --------------------------------------------------------------------------
# keyed bijection of [0, n): Feistel network + cycle walking
# --------------------------------------------------------------------------
def _feistel(x: np.ndarray, half_bits: int, keys: Sequence[int]) -> np.ndarray:
    mask = np.uint64((1 << half_bits) - 1)
    hi = (x >> np.uint64(half_bits)) & mask
    lo = x & mask
    for k in keys:
        # round function: multiply-xorshift mixing keyed per round
        f = (lo * np.uint64(0xD6E8FEB86659FD93) + np.uint64(k)) & _M64
        f ^= f >> np.uint64(29)
        f = (f * np.uint64(0xA0761D6478BD642F)) & _M64
        f ^= f >> np.uint64(32)
        hi, lo = lo, (hi ^ f) & mask
    return (hi << np.uint64(half_bits)) | lo


def scramble(ranks0: np.ndarray, n: int, key: int) -> np.ndarray:
    """Bijection of [0, n) onto itself, keyed by `key` (ranks0 are 0-based)."""
    bits = max(2, int(math.ceil(math.log2(max(n, 2)))))
    bits += bits & 1
    half = bits // 2
    rk = np.random.default_rng(key).integers(0, 2**63, size=4, dtype=np.int64)
    keys = [int(v) for v in rk]
    x = ranks0.astype(np.uint64)
    todo = np.ones(x.shape, bool)
    while True:
        x[todo] = _feistel(x[todo], half, keys)
        todo = x >= np.uint64(n)
        if not todo.any():
            break
    return x.astype(np.int64)


# --------------------------------------------------------------------------
# workload descriptions
# --------------------------------------------------------------------------
@dataclass
class FeatureSpec:
    flags: int
    hash_seed: int = 0
    mod: int = 0
    tag: int = 0
    tag_shift: int = 48
    boundaries: Sequence[int] = field(default_factory=list)


@dataclass
class TableSpec:
    name: str
    features: List[int]        # consecutive feature indices merged into this table
    dim: int
    optimizer: str             # "adagrad" | "adam"
    lr: float
    combiner: str              # "sum" | "mean"
    pooled: bool = True
    unpooled: bool = False
    init_seed: int = 0


@dataclass
class Workload:
    name: str
    index: int
    F: int
    B: int
    n_ids: int                 # ID space per feature (Zipf support)
    zipf_a: float
    length: str                # "one" | "uniform:lo:hi" | "geom:p"
    tables: List[TableSpec]
    features: List[FeatureSpec]
    live_ids: int = 0          # large-table workload: IDs pre-inserted
    fresh_frac: float = 0.0    # fraction of occurrences that are never-seen IDs

    def scaled(self, B: int) -> "Workload":
        """Same recipe with a smaller batch (for parity tests)."""
        w = Workload(**{k: getattr(self, k) for k in self.__dataclass_fields__})
        w.B = B
        return w


def _tagged(F, shift, extra=0):
    return [FeatureSpec(flags=TAG | extra, tag=f, tag_shift=shift) for f in range(F)]


def _hashed(F):
    return [FeatureSpec(flags=HASH | MOD | TAG, hash_seed=0x5EED0000 + 7919 * f,
                        mod=1 << 40, tag=f, tag_shift=40) for f in range(F)]


WORKLOADS = {
    "tiny": Workload("tiny", 0, F=4, B=256, n_ids=10_000, zipf_a=1.1, length="uniform:1:8",
                     tables=[TableSpec("t16", [0, 1, 2, 3], 16, "adagrad", 0.01, "sum",
                                       init_seed=11)],
                     features=_tagged(4, 48)),
    "criteo26": Workload("criteo26", 1, F=26, B=8192, n_ids=10_000_000, zipf_a=1.05, length="one",
                         tables=[TableSpec("t64", list(range(26)), 64, "adam", 1e-3, "sum",
                                           init_seed=12)],
                         features=_hashed(26)),
    "seq8": Workload("seq8", 2, F=8, B=4096, n_ids=100_000_000, zipf_a=1.2,
                     length="uniform:1:100",
                     tables=[TableSpec("t32", [0, 1, 2, 3], 32, "adagrad", 0.01, "mean",
                                       init_seed=13),
                             TableSpec("t64", [4, 5, 6, 7], 64, "adagrad", 0.01, "mean",
                                       init_seed=14)],
                     features=_tagged(8, 48)),
    "longseq": Workload("longseq", 3, F=1, B=512, n_ids=100_000_000, zipf_a=0.9,
                        length="uniform:1000:5000",
                        tables=[TableSpec("t128", [0], 128, "adam", 1e-3, "sum",
                                          pooled=True, unpooled=True, init_seed=15)],
                        features=_tagged(1, 48)),
    "large": Workload("large", 4, F=100, B=65536, n_ids=1 << 48, zipf_a=1.05, length="geom:0.2",
                      tables=[TableSpec("t64", list(range(100)), 64, "adam", 1e-3, "sum",
                                        init_seed=16)],
                      features=_tagged(100, 48), live_ids=50_000_000, fresh_frac=0.05),
}


@dataclass
class Batch:
    values: np.ndarray        # int64 [N], feature-major
    feat_offsets: np.ndarray  # int64 [F+1]
    bag_offsets: np.ndarray   # int64 [F*B+1]
    lengths: np.ndarray       # int64 [F*B]
    fresh_pos: Optional[List[np.ndarray]] = None  # per feature: positions holding fresh IDs

    def table_slice(self, t: TableSpec, B: int):
        """(value range, bag offsets rebased to 0) for the features of table t."""
        f0, f1 = t.features[0], t.features[-1] + 1
        lo, hi = int(self.feat_offsets[f0]), int(self.feat_offsets[f1])
        bo = self.bag_offsets[f0 * B: f1 * B + 1] - lo
        return lo, hi, np.ascontiguousarray(bo)


def _lengths(w: Workload, rng: np.random.Generator) -> np.ndarray:
    nb = w.F * w.B
    if w.length == "one":
        return np.ones(nb, np.int64)
    kind, *args = w.length.split(":")
    if kind == "uniform":
        lo, hi = int(args[0]), int(args[1])
        return rng.integers(lo, hi + 1, size=nb, dtype=np.int64)
    if kind == "geom":
        return rng.geometric(float(args[0]), size=nb).astype(np.int64)
    raise ValueError(w.length)


def make_batch(w: Workload, batch_index: int = 0, seed: Optional[int] = None) -> Batch:
    base = 2025 + w.index if seed is None else seed
    rng = np.random.default_rng([base, batch_index])
    lengths = _lengths(w, rng)
    bag_offsets = np.zeros(w.F * w.B + 1, np.int64)
    np.cumsum(lengths, out=bag_offsets[1:])
    N = int(bag_offsets[-1])
    feat_offsets = bag_offsets[:: w.B].copy()
    values = np.empty(N, np.int64)
    # large-table workload: Zipf over each feature's share of the live set (the
    # pre-inserted IDs of live_ids()), so every non-fresh occurrence is live
    zipf = Zipf(w.live_ids // w.F if w.live_ids else w.n_ids, w.zipf_a)
    fresh_pos = [] if w.fresh_frac > 0 else None
    for f in range(w.F):
        lo, hi = int(feat_offsets[f]), int(feat_offsets[f + 1])
        n = hi - lo
        ranks0 = zipf.sample(rng, n) - 1
        if w.fresh_frac > 0:
            fresh = np.nonzero(rng.random(n) < w.fresh_frac)[0]
            ranks0[fresh] = _fresh_ranks(w, f, batch_index, len(fresh))
            fresh_pos.append(lo + fresh)
        values[lo:hi] = scramble(ranks0, w.n_ids, key=(base << 8) + f)
    return Batch(values, feat_offsets, bag_offsets, lengths, fresh_pos)


def _fresh_ranks(w: Workload, f: int, stream_index: int, count: int) -> np.ndarray:
    """Ranks of never-seen IDs: past the live set, from a counter range of
    feature f and stream index (disjoint for different (f, index) pairs)."""
    assert 0 <= stream_index < 4095 and f < 256 and count < (1 << 28)
    return (w.live_ids + ((stream_index + 1) << 36) + (f << 28)
            + np.arange(count, dtype=np.int64))


def with_fresh_ids(w: Workload, b: Batch, stream_index: int,
                   seed: Optional[int] = None) -> np.ndarray:
    """Values of batch b with every fresh-ID position given a never-seen ID of
    counter range `stream_index` (the rest unchanged): one more step of the
    large-table workload without drawing its Zipf part again."""
    base = 2025 + w.index if seed is None else seed
    vals = b.values.copy()
    for f, pos in enumerate(b.fresh_pos or []):
        ranks0 = _fresh_ranks(w, f, stream_index, len(pos))
        vals[pos] = scramble(ranks0, w.n_ids, key=(base << 8) + f)
    return vals


def live_ids(w: Workload, f: int, count: int, seed: Optional[int] = None) -> np.ndarray:
    """The IDs of ranks 1..count of feature f (the pre-inserted live set:
    count = live_ids // F per feature)."""
    base = 2025 + w.index if seed is None else seed
    return scramble(np.arange(count, dtype=np.int64), w.n_ids, key=(base << 8) + f)


def make_grad(shape, seed: int, signed: bool = False) -> np.ndarray:
    rng = np.random.default_rng([seed, 7])
    g = rng.random(shape, dtype=np.float32)
    return (2.0 * g - 1.0).astype(np.float32) if signed else (0.5 + 0.5 * g).astype(np.float32)
