"""GPU parity at sizes past the sample-sort dedup (radix-sort path) and at the
full large-table workload.

- A 2.5M-occurrence batch (above the 1.6M sample-sort limit) runs through the
  LSD radix dedup and is compared with the oracle element by element.
- The large-table workload at full size (50M pre-inserted keys, 65536 x 100
  bags of geometric length, 32.8M occurrences) is too large for the oracle,
  so integers are checked by properties that hold at any size (unique keys
  strictly ascending, keys == uniq[inv], pre-inserted keys keep their rows,
  new keys take the next rows in ascending key order) and floating point on
  sampled bags and keys, each recomputed by the oracle from the pages'
  definitions (pooled sum of the sampled bags; one Adam step of sampled keys
  with their gradient summed over all their occurrences in float64).
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity_util import Pair, close, compare_tables

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def R():
    import recommender_sparse_embedding_b200 as R
    from recommender_sparse_embedding_b200 import build
    build.build()
    assert torch.cuda.is_available()
    R.load()
    return R


def test_radix_path_parity(R):
    rng = np.random.default_rng(31)
    B = 1_000_000
    lengths = rng.integers(1, 5, size=B).astype(np.int64)  # ~2.5M occurrences
    bo = np.zeros(B + 1, np.int64)
    np.cumsum(lengths, out=bo[1:])
    N = int(bo[-1])
    assert N > 1_600_000
    keys = rng.integers(0, 1_200_000, size=N).astype(np.int64) * 7919 - 3_000_000_000
    spec = W.TableSpec("t", [0], 8, "adam", 0.01, "sum", pooled=True, init_seed=23)
    p = Pair(R, spec)
    k_dev = torch.from_numpy(keys).to(DEV)
    bo_dev = torch.from_numpy(bo).to(DEV)
    for step in range(2):
        pooled = torch.empty((B, 1, 8), dtype=torch.float32, device=DEV)
        p.gpu.lookup_pooled(p.batch, k_dev, bo_dev, 1, B, R.SUM, pooled)
        r = p.ora.lookup(keys, bo, 1, B, O.SUM)
        uq, inv, rows, n_new = p.batch.get_unique(N)
        assert np.array_equal(uq.cpu().numpy(), r.uniq)
        assert np.array_equal(inv.cpu().numpy(), r.inv)
        assert np.array_equal(rows.cpu().numpy(), r.rows)
        assert n_new == r.n_new
        close(pooled.cpu().numpy(), r.pooled, f"pooled step {step}")
        gp = W.make_grad((B, 1, 8), 70 + step, signed=True)
        p.gpu.backward_update(p.batch, torch.from_numpy(gp).to(DEV))
        p.ora.backward_update(gp)
        p.gpu.status_sync()
        compare_tables(p, f"step {step}")
    p.close()


def test_large_workload_full_size_sampled(R):
    w = W.WORKLOADS["large"]
    spec = w.tables[0]
    D, F, B = spec.dim, w.F, w.B
    rng = np.random.default_rng(77)
    # the live set: ranks 1 .. live_ids/F of every feature, tagged, ascending
    per = w.live_ids // F
    live = np.concatenate([(np.int64(w.features[f].tag) << np.int64(48)) | W.live_ids(w, f, per)
                           for f in range(F)])
    live.sort()
    n_live = len(live)
    t = R.Table(D, R.ADAM, spec.lr, init_seed=spec.init_seed, initial_capacity=64_000_000)
    b_ins = R.Batch()
    for c0 in range(0, n_live, 1_500_000):
        t.insert(b_ins, torch.from_numpy(live[c0:c0 + 1_500_000]).to(DEV))
    t.status_sync()
    assert t.size()[0] == n_live  # rows 0 .. n_live-1 in ascending key order

    # one step of the workload at full size
    bt = W.make_batch(w, 0)
    N = len(bt.values)
    ops = [O.FeatureOp(flags=f.flags, tag=f.tag, tag_shift=f.tag_shift) for f in w.features]
    okeys = O.feature_hash(ops, bt.values, bt.feat_offsets)
    keys = R.feature_hash([R.Feature(flags=f.flags, tag=f.tag, tag_shift=f.tag_shift)
                           for f in w.features],
                          torch.from_numpy(bt.values).to(DEV), bt.feat_offsets.tolist())
    assert np.array_equal(keys.cpu().numpy(), okeys)
    bo_dev = torch.from_numpy(bt.bag_offsets).to(DEV)
    pooled = torch.empty((B, F, D), dtype=torch.float32, device=DEV)
    b = R.Batch()
    t.lookup_pooled(b, keys, bo_dev, F, B, R.SUM, pooled)
    uq, inv, rows, n_new = b.get_unique(N)
    torch.cuda.synchronize()

    # integers, at full size: ascending unique keys, inverse, row assignment
    assert bool((uq[1:] > uq[:-1]).all())
    assert torch.equal(uq[inv.long()], keys)
    live_dev = torch.from_numpy(live).to(DEV)
    at = torch.searchsorted(live_dev, uq)
    found = (at < n_live) & (live_dev[at.clamp(max=n_live - 1)] == uq)
    assert torch.equal(rows[found], at[found])  # pre-inserted keys keep their rows
    assert n_new == int((~found).sum())
    assert torch.equal(rows[~found], n_live + torch.arange(n_new, device=DEV))  # ascending key order
    assert t.size()[0] == n_live + n_new

    # pooled sums of sampled bags against the oracle on those bags alone
    # (every row is still at its initial value)
    bags = rng.choice(F * B, size=300, replace=False)
    lo, hi = bt.bag_offsets[bags], bt.bag_offsets[bags + 1]
    mkeys = np.concatenate([okeys[a:c] for a, c in zip(lo, hi)])
    mbo = np.concatenate([[0], np.cumsum(hi - lo)]).astype(np.int64)
    ot = O.Table(D, O.ADAM, spec.lr, init_seed=spec.init_seed)
    ref = ot.lookup(mkeys, mbo, 1, len(bags), O.SUM).pooled[:, 0, :]
    pc = pooled.cpu().numpy()
    got = np.stack([pc[j % B, j // B] for j in bags])
    close(got, ref, "pooled, sampled bags")

    # one Adam step: updated rows of sampled keys against the oracle fed the
    # key's gradient summed in float64 over all its occurrences
    gp = W.make_grad((B, F, D), 4242)
    t.backward_update(b, torch.from_numpy(gp).to(DEV))
    t.status_sync()
    U = len(uq)
    pick = np.unique(np.concatenate([rng.choice(U, size=48, replace=False),
                                     np.argsort(-torch.bincount(inv.long()).cpu().numpy())[:8]]))
    skeys = uq[torch.from_numpy(pick).to(DEV)]
    cur = torch.empty((len(pick), D), dtype=torch.float32, device=DEV)
    b3 = R.Batch()
    sbo = torch.arange(len(pick) + 1, dtype=torch.int64, device=DEV)
    t.lookup_pooled(b3, skeys, sbo, 1, len(pick), R.SUM, None, cur)
    cur = cur.cpu().numpy()
    for n, u in enumerate(pick):
        occ = torch.nonzero(inv == int(u)).flatten().cpu().numpy()
        bag = np.searchsorted(bt.bag_offsets, occ, side="right") - 1
        g = gp[bag % B, bag // B].astype(np.float64).sum(axis=0).astype(np.float32)
        o1 = O.Table(D, O.ADAM, spec.lr, init_seed=spec.init_seed)
        o1.lookup(np.array([int(skeys[n])], np.int64), np.array([0, 1], np.int64), 1, 1, O.SUM)
        o1.backward_update(g.reshape(1, 1, D))
        _, emb, _ = o1.export()
        close(cur[n], emb[0], f"updated row of unique key {int(u)} ({len(occ)} occurrences)")
    for x in (b3, b, b_ins):
        x.close()
    t.close()
