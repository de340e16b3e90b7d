"""Shared driver of the GPU-vs-oracle parity tests.

Runs the same seeded workload through the CUDA library (through its C ABI) and
through the CPU oracle, step by step, and compares every output: integers
bit-exact, floating point within |gpu - ref| <= 1e-6 + 1e-5 |ref|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import workloads as W

RTOL, ATOL = 1e-5, 1e-6


def close(a, b, what):
    np.testing.assert_allclose(a, b, rtol=RTOL, atol=ATOL, err_msg=what)


def _rfeat(R, f: W.FeatureSpec, dev):
    bnd = None
    if f.boundaries:
        bnd = torch.tensor(list(f.boundaries), dtype=torch.int64, device=dev)
    return R.Feature(flags=f.flags, hash_seed=f.hash_seed, mod=f.mod, tag=f.tag,
                     tag_shift=f.tag_shift, boundaries=bnd)


def _ofeat(f: W.FeatureSpec):
    return O.FeatureOp(flags=f.flags, hash_seed=f.hash_seed, mod=f.mod, tag=f.tag,
                       tag_shift=f.tag_shift, boundaries=list(f.boundaries))


class Pair:
    """One logical table on both sides."""

    def __init__(self, R, spec: W.TableSpec, initial_capacity=0, block_rows=0, init_acc=0.0,
                 admit_threshold=0, evictable=False, placement=0):
        opt_r = R.ADAGRAD if spec.optimizer == "adagrad" else R.ADAM
        opt_o = O.ADAGRAD if spec.optimizer == "adagrad" else O.ADAM
        self.spec = spec
        self.gpu = R.Table(spec.dim, opt_r, spec.lr, init_seed=spec.init_seed,
                           initial_capacity=initial_capacity, block_rows=block_rows,
                           adagrad_init_acc=init_acc, admit_threshold=admit_threshold,
                           evictable=evictable, placement=placement)
        self.ora = O.Table(spec.dim, opt_o, spec.lr, init_seed=spec.init_seed,
                           adagrad_init_acc=init_acc, admit_threshold=admit_threshold)
        self.batch = R.Batch()
        self.combiner_r = R.SUM if spec.combiner == "sum" else R.MEAN
        self.combiner_o = O.SUM if spec.combiner == "sum" else O.MEAN

    def close(self):
        self.gpu.close()
        self.batch.close()


def run_workload(R, w: W.Workload, steps=2, batch_seed=None, check_unique=True, pairs=None,
                 initial_capacity=0, block_rows=0, grad_signed=False, return_pairs=False,
                 admit_threshold=0, evict_every=0, evict_age=1):
    """Steps of workload w on both sides, compared after every step.  With
    evict_every > 0 both sides evict, after every evict_every-th step, the keys
    last touched more than evict_age lookups before the current clock."""
    dev = torch.device("cuda", torch.cuda.current_device())
    if pairs is None:
        pairs = [Pair(R, t, initial_capacity, block_rows, admit_threshold=admit_threshold,
                      evictable=evict_every > 0) for t in w.tables]
    rfeats = [_rfeat(R, f, dev) for f in w.features]
    ofeats = [_ofeat(f) for f in w.features]
    for step in range(steps):
        bt = W.make_batch(w, step, seed=batch_seed)
        vals = torch.from_numpy(bt.values).to(dev)
        keys = R.feature_hash(rfeats, vals, bt.feat_offsets.tolist())
        okeys = O.feature_hash(ofeats, bt.values, bt.feat_offsets)
        gk = keys.cpu().numpy()
        assert np.array_equal(gk, okeys), f"feature hash differs at step {step}"
        for p in pairs:
            t = p.spec
            lo, hi, bo = bt.table_slice(t, w.B)
            Ft = len(t.features)
            N = hi - lo
            D = t.dim
            k_dev = keys[lo:hi]
            bo_dev = torch.from_numpy(bo).to(dev)
            pooled = torch.empty((w.B, Ft, D), dtype=torch.float32, device=dev) if t.pooled else None
            unpooled = torch.empty((N, D), dtype=torch.float32, device=dev) if t.unpooled else None
            p.gpu.lookup_pooled(p.batch, k_dev, bo_dev, Ft, w.B, p.combiner_r, pooled, unpooled)
            r = p.ora.lookup(okeys[lo:hi], bo, Ft, w.B, p.combiner_o, pooled=t.pooled,
                             unpooled=t.unpooled)
            if check_unique:
                uq, inv, rows, n_new = p.batch.get_unique(N)
                assert np.array_equal(uq.cpu().numpy(), r.uniq), f"uniq differs ({t.name}, step {step})"
                assert np.array_equal(inv.cpu().numpy(), r.inv), f"inv differs ({t.name}, step {step})"
                assert np.array_equal(rows.cpu().numpy(), r.rows), f"rows differ ({t.name}, step {step})"
                assert n_new == r.n_new
            if t.pooled:
                close(pooled.cpu().numpy(), r.pooled, f"pooled {t.name} step {step}")
            if t.unpooled:
                close(unpooled.cpu().numpy(), r.unpooled, f"unpooled {t.name} step {step}")
            gseed = 1000 * (step + 1) + w.index
            gp = W.make_grad((w.B, Ft, D), gseed, signed=grad_signed) if t.pooled else None
            gu = W.make_grad((N, D), gseed + 1, signed=grad_signed) if t.unpooled else None
            p.gpu.backward_update(p.batch, None if gp is None else torch.from_numpy(gp).to(dev),
                                  None if gu is None else torch.from_numpy(gu).to(dev))
            p.ora.backward_update(gp, gu)
            p.gpu.status_sync()
            compare_tables(p, f"{t.name} step {step}")
            if evict_every and (step + 1) % evict_every == 0:
                assert p.gpu.clock == p.ora.clock
                cut = p.ora.clock - evict_age + 1
                assert p.gpu.evict(cut) == p.ora.evict(cut)
                compare_tables(p, f"{t.name} after eviction at step {step}")
    if return_pairs:
        return pairs
    for p in pairs:
        p.close()


def compare_tables(p: Pair, what: str):
    gk, ge, gs, gstep = p.gpu.export()
    ok, oe, os_ = p.ora.export()
    assert np.array_equal(gk, ok), f"row keys differ ({what})"
    close(ge, oe, f"emb {what}")
    close(gs, os_, f"state {what}")
    assert gstep == p.ora.step
