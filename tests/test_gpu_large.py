"""GPU parity at sizes past the sample-sort dedup (radix-sort path) and at the
full large-table workload.

- A 2.5M-occurrence batch (above the 1.6M sample-sort limit) runs through the
  LSD radix dedup and is compared with the oracle element by element.
- A 1.8M-occurrence batch of 300,000 bags at D = 64 (pooled gradients of
  77 MB, more than the row update keeps in L2) takes the row update that
  gathers the keys seen 2 to 16 times ahead of its walk, with pooled
  gradients only and with pooled and unpooled ones; compared element by
  element over two Adam steps with signed gradients.
- The large-table workload at full size (50M pre-inserted keys, 65536 x 100
  bags of geometric length, 32.8M occurrences, two steps) is too large for the
  oracle, so integers are checked by properties that hold at any size (unique
  keys strictly ascending, keys == uniq[inv], every unique key has an
  occurrence, U equals the number of distinct keys, pre-inserted keys keep
  their rows, new keys take the next rows in ascending key order) and floating
  point on sampled bags and keys, each recomputed by the oracle from the
  pages' definitions: the pooled sums of sampled bags, and emb, Adam m and
  Adam v of sampled keys after two steps with signed gradients, the oracle fed
  each key's gradient summed over all its occurrences in float64 (m after the
  first step is (1 - beta1) g, so the gradient's magnitude is pinned, not only
  its sign).
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


@pytest.mark.parametrize("unpooled", [False, True], ids=["pooled", "pooled+unpooled"])
def test_gather_ahead_parity(R, unpooled):
    rng = np.random.default_rng(37)
    B, D = 300_000, 64
    lengths = rng.integers(1, 12, size=B).astype(np.int64)  # ~1.8M occurrences
    bo = np.zeros(B + 1, np.int64)
    np.cumsum(lengths, out=bo[1:])
    N = int(bo[-1])
    assert N > 1_600_000 and B * D * 4 > 64 << 20
    # a pool of 1M keys (singletons and keys seen a few times) and 64 hot
    # keys at 3 % of the positions (segments longer than 16)
    keys = rng.integers(0, 1_000_000, size=N).astype(np.int64) * 104729 + 11
    hot = rng.random(N) < 0.03
    keys[hot] = rng.integers(0, 64, size=int(hot.sum())) * 104729 + 11
    spec = W.TableSpec("t", [0], D, "adam", 0.01, "sum", pooled=True, unpooled=unpooled, init_seed=29)
    p = Pair(R, spec)
    k_dev = torch.from_numpy(keys).to(DEV)
    bo_dev = torch.from_numpy(bo).to(DEV)
    for step in range(2):
        pooled = torch.empty((B, 1, D), dtype=torch.float32, device=DEV)
        unp = torch.empty((N, D), dtype=torch.float32, device=DEV) if unpooled else None
        p.gpu.lookup_pooled(p.batch, k_dev, bo_dev, 1, B, R.SUM, pooled, unp)
        r = p.ora.lookup(keys, bo, 1, B, O.SUM, pooled=True, unpooled=unpooled)
        uq, inv, rows, n_new = p.batch.get_unique(N)
        assert np.array_equal(uq.cpu().numpy(), r.uniq)
        assert np.array_equal(inv.cpu().numpy(), r.inv)
        assert np.array_equal(rows.cpu().numpy(), r.rows)
        assert n_new == r.n_new
        cnt = np.bincount(r.inv, minlength=len(r.uniq))
        assert ((cnt >= 2) & (cnt <= 16)).sum() > 100_000 and (cnt > 16).sum() == 64
        close(pooled.cpu().numpy(), r.pooled, f"pooled step {step}")
        if unpooled:
            close(unp.cpu().numpy(), r.unpooled, f"unpooled step {step}")
        gp = W.make_grad((B, 1, D), 90 + step, signed=True)
        gu = W.make_grad((N, D), 95 + step, signed=True) if unpooled else None
        p.gpu.backward_update(p.batch, torch.from_numpy(gp).to(DEV),
                              None if gu is None else torch.from_numpy(gu).to(DEV))
        p.ora.backward_update(gp, gu)
        p.gpu.status_sync()
        compare_tables(p, f"step {step}")
    p.close()


def _host_grad(inv_dev, u, bag_offsets, gp, B):
    """fp32 gradient of unique index u: its occurrences' pooled-gradient rows
    summed in float64, rounded once (the oracle's definition of g(u))."""
    occ = torch.nonzero(inv_dev == int(u)).flatten().cpu().numpy()
    bag = np.searchsorted(bag_offsets, occ, side="right") - 1
    return gp[bag % B, bag // B].astype(np.float64).sum(axis=0).astype(np.float32), len(occ)


def _check_dedup(R, t, b, keys, N, live_dev, live_before, n_before):
    """Integer checks of one full-size lookup that hold at any size."""
    uq, inv, rows, n_new = b.get_unique(N)
    torch.cuda.synchronize()
    U = uq.numel()
    assert bool((uq[1:] > uq[:-1]).all())                       # strictly ascending
    assert torch.equal(uq[inv.long()], keys)                     # keys == uniq[inv]
    cnt = torch.bincount(inv.long(), minlength=U)
    assert cnt.numel() == U and int((cnt == 0).sum()) == 0       # every unique key occurs
    assert U == int(torch.unique(keys).numel())                  # U = distinct keys
    n_live = live_dev.numel()
    at = torch.searchsorted(live_dev, uq)
    found = (at < n_live) & (live_dev[at.clamp(max=n_live - 1)] == uq)
    assert torch.equal(rows[found], at[found])                   # pre-inserted keys keep their rows
    # keys already added by an earlier step keep their rows too; the rest are new
    old = rows[~found] < n_before
    assert int((rows[~found][old] >= live_before).sum()) == int(old.sum())
    assert n_new == int((~found).sum()) - int(old.sum())
    fresh_rows = rows[~found][~old]
    assert torch.equal(fresh_rows, n_before + torch.arange(n_new, device=DEV))  # ascending key order
    assert t.size()[0] == n_before + n_new
    return uq, inv, rows, n_new, cnt


def test_large_workload_full_size_sampled(R):
    """Two steps of the large-table workload at full size with signed
    gradients: integers by properties, pooled rows of sampled bags, and the
    emb, Adam m and Adam v of sampled keys after both steps against the oracle
    fed each key's gradient summed in float64 over all its occurrences."""
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
    live_dev = torch.from_numpy(live).to(DEV)

    ops = [O.FeatureOp(flags=f.flags, tag=f.tag, tag_shift=f.tag_shift) for f in w.features]
    rfeats = [R.Feature(flags=f.flags, tag=f.tag, tag_shift=f.tag_shift) for f in w.features]
    b = R.Batch()
    pooled = torch.empty((B, F, D), dtype=torch.float32, device=DEV)
    steps = []
    n_before = n_live
    for step in range(2):
        bt = W.make_batch(w, step)
        N = len(bt.values)
        okeys = O.feature_hash(ops, bt.values, bt.feat_offsets)
        keys = R.feature_hash(rfeats, torch.from_numpy(bt.values).to(DEV), bt.feat_offsets.tolist())
        assert np.array_equal(keys.cpu().numpy(), okeys)
        bo_dev = torch.from_numpy(bt.bag_offsets).to(DEV)
        t.lookup_pooled(b, keys, bo_dev, F, B, R.SUM, pooled)
        uq, inv, rows, n_new, cnt = _check_dedup(R, t, b, keys, N, live_dev, n_live, n_before)
        assert n_new > 0.04 * N  # the workload's 5% fresh IDs are new rows
        if step == 0:
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
        gp = W.make_grad((B, F, D), 4242 + step, signed=True)
        t.backward_update(b, torch.from_numpy(gp).to(DEV))
        t.status_sync()
        steps.append((bt, uq, inv, rows, cnt, gp))
        n_before += n_new

    # sampled keys: random and hottest keys of step 0, fresh keys of step 0,
    # random keys of step 1 (some present in both steps)
    uq0, inv0, rows0, cnt0 = steps[0][1], steps[0][2], steps[0][3], steps[0][4]
    uq1, inv1, rows1, cnt1 = steps[1][1], steps[1][2], steps[1][3], steps[1][4]
    U0, U1 = uq0.numel(), uq1.numel()
    fresh0 = torch.nonzero(rows0 >= n_live).flatten().cpu().numpy()
    pick0 = np.unique(np.concatenate([rng.choice(U0, 40, replace=False),
                                      torch.argsort(cnt0, descending=True)[:8].cpu().numpy(),
                                      rng.choice(fresh0, 8, replace=False)]))
    skeys = set(uq0[torch.from_numpy(pick0).to(DEV)].cpu().tolist())
    skeys |= set(uq1[torch.from_numpy(rng.choice(U1, 24, replace=False)).to(DEV)].cpu().tolist())
    skeys = np.array(sorted(skeys), np.int64)
    # each sampled key's gradient per step (zero when absent), its row, and
    # the oracle table stepped the same way (a dummy key keeps its Adam step
    # counter in line with the GPU table's when no sampled key is present)
    ot = O.Table(D, O.ADAM, spec.lr, init_seed=spec.init_seed)
    dummy = np.int64(-7)
    row_of = {}
    for s_i, (bt, uq, inv, rows, cnt, gp) in enumerate(steps):
        uqh = uq.cpu().numpy()
        pos = np.searchsorted(uqh, skeys)
        present = (pos < len(uqh)) & (uqh[np.minimum(pos, len(uqh) - 1)] == skeys)
        ks, gs = [dummy], [np.zeros(D, np.float32)]
        for k, pz, pr in zip(skeys, pos, present):
            if not pr:
                continue
            g, nocc = _host_grad(inv, pz, bt.bag_offsets, gp, B)
            assert nocc == int(cnt[pz])
            ks.append(k)
            gs.append(g)
            row_of[int(k)] = int(rows[pz])
        order = np.argsort(np.array(ks))
        kk = np.array(ks, np.int64)[order]
        gg = np.stack(gs)[order]
        ot.lookup(kk, np.arange(len(kk) + 1, dtype=np.int64), 1, len(kk), O.SUM)
        ot.backward_update(gg.reshape(len(kk), 1, D))
    rsel = torch.tensor([row_of[int(k)] for k in skeys], dtype=torch.int64, device=DEV)
    gk, ge, gs_ = t.read_rows(rsel)
    assert np.array_equal(gk.cpu().numpy(), skeys)
    okeys_, oemb, ostate = ot.export()  # rows in insertion order
    where = {int(k): i for i, k in enumerate(okeys_)}
    idx = np.array([where[int(k)] for k in skeys])
    close(ge.cpu().numpy(), oemb[idx], "emb of sampled keys after two Adam steps")
    close(gs_.cpu().numpy()[:, :D], ostate[idx][:, :D], "Adam m of sampled keys")
    close(gs_.cpu().numpy()[:, D:], ostate[idx][:, D:], "Adam v of sampled keys")
    assert t.size()[1] == 2
    for x in (b, b_ins):
        x.close()
    t.close()
