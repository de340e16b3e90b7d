"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Integers (keys, unique list, inverse index, row offsets, row order) must be
bit-exact; fp32 outputs (pooled, unpooled, updated rows and optimiser state)
must satisfy |gpu - ref| <= 1e-6 + 1e-5 |ref| elementwise.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity_util import RTOL, ATOL, Pair, close, compare_tables, run_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    import recommender_sparse_embedding_b200 as R
    from recommender_sparse_embedding_b200 import build
    build.build()
    assert torch.cuda.is_available()
    R.load()
    return R


DEV = "cuda"


# ---------------------------------------------------------------- feature transform
def test_feature_hash_all_op_kinds(R):
    rng = np.random.default_rng(5)
    F = 300  # more features than one launch takes
    lens = rng.integers(0, 200, size=F)
    lens[7] = 0
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N = int(offs[-1])
    vals = rng.integers(-(2**62), 2**62, size=N, dtype=np.int64)
    vals[::13] = rng.integers(-50, 50, size=len(vals[::13]))
    bnd = np.unique(rng.integers(-40, 40, size=11)).astype(np.int64)
    bnd_dev = torch.from_numpy(bnd).to(DEV)
    rf, of = [], []
    for f in range(F):
        k = f % 6
        if k == 0:
            spec = dict(flags=W.BUCKETIZE | W.TAG, tag=f, tag_shift=40)
        elif k == 1:
            spec = dict(flags=W.HASH | W.MOD | W.TAG, hash_seed=77 * f, mod=1 << 40, tag=f, tag_shift=40)
        elif k == 2:
            spec = dict(flags=W.HASH | W.MOD, hash_seed=f, mod=10_000_019)
        elif k == 3:
            spec = dict(flags=W.HASH, hash_seed=2**63 + f)
        elif k == 4:
            spec = dict(flags=W.MOD | W.TAG, mod=999_983, tag=f, tag_shift=30)
        else:
            spec = dict(flags=0)
        b = spec["flags"] & W.BUCKETIZE
        rf.append(R.Feature(boundaries=bnd_dev if b else None, **spec))
        of.append(O.FeatureOp(boundaries=bnd.tolist() if b else [], **spec))
    got = R.feature_hash(rf, torch.from_numpy(vals).to(DEV), offs.tolist()).cpu().numpy()
    R.feature_status_sync()
    ref = O.feature_hash(of, vals, offs)
    assert np.array_equal(got, ref)


def test_feature_bucketize_float_values(R):
    # float64 features (values as bit patterns in the int64 array) beside
    # int64 ones in one launch: random doubles with many equal to a
    # boundary, infinities, signed zeros, NaNs and denormals
    rng = np.random.default_rng(9)
    F = 140  # more features than one launch takes
    lens = rng.integers(0, 300, size=F)
    lens[3] = 0
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    N = int(offs[-1])
    fb = np.unique(np.round(rng.normal(size=40), 2))
    fb[0] = -np.inf  # a boundary every value but NaN passes
    x = np.round(rng.normal(scale=1.5, size=N), 2)
    x[::7] = rng.choice(fb[1:], size=len(x[::7]))
    special = np.array([np.inf, -np.inf, 0.0, -0.0, np.nan, -np.nan, 5e-324, -5e-324, 1e308, -1e308])
    x[::11] = rng.choice(special, size=len(x[::11]))
    ib = np.unique(rng.integers(-40, 40, size=9)).astype(np.int64)
    vals = x.view(np.int64).copy()
    rf, of = [], []
    for f in range(F):
        if f % 3 == 2:  # an int64 bucketize feature: its own values
            lo, hi = offs[f], offs[f + 1]
            vals[lo:hi] = rng.integers(-50, 50, size=hi - lo)
            spec = dict(flags=W.BUCKETIZE | W.TAG, tag=f, tag_shift=48)
            rf.append(R.Feature(boundaries=torch.from_numpy(ib).to(DEV), **spec))
            of.append(O.FeatureOp(boundaries=ib.tolist(), **spec))
        else:
            spec = dict(flags=W.BUCKETIZE | W.FLOAT | (W.TAG if f % 3 else 0), tag=f, tag_shift=48)
            rf.append(R.Feature(boundaries=torch.from_numpy(fb).to(DEV), **spec))
            of.append(O.FeatureOp(boundaries=fb.tolist(), **spec))
    got = R.feature_hash(rf, torch.from_numpy(vals).to(DEV), offs.tolist()).cpu().numpy()
    R.feature_status_sync()
    ref = O.feature_hash(of, vals, offs)
    assert np.array_equal(got, ref)


def test_feature_hash_tag_overflow_is_reported(R):
    vals = torch.tensor([1, 2, 300, 4], dtype=torch.int64, device=DEV)
    R.feature_hash([R.Feature(flags=R.TAG, tag=1, tag_shift=8)], vals, [0, 4])
    with pytest.raises(R.RecisError) as e:
        R.feature_status_sync()
    assert e.value.code == 1
    R.feature_status_sync()  # cleared


# ---------------------------------------------------------------- workloads
@pytest.mark.parametrize("name,B,steps", [
    ("tiny", 256, 3),
    ("criteo26", 512, 3),
    ("seq8", 96, 2),
    ("longseq", 6, 2),
    ("large", 48, 2),
])
def test_workload_parity_scaled(R, name, B, steps):
    run_workload(R, W.WORKLOADS[name].scaled(B), steps=steps)


@pytest.mark.parametrize("name,steps", [("criteo26", 2), ("longseq", 2), ("seq8", 1)])
def test_workload_parity_full_size(R, name, steps):
    run_workload(R, W.WORKLOADS[name], steps=steps)


def test_signed_gradients_and_growth(R):
    # tiny initial capacity and blocks: the IDMap rehashes and blocks are
    # mapped while the run goes on; signed gradients exercise cancellation
    run_workload(R, W.WORKLOADS["criteo26"].scaled(256), steps=3, initial_capacity=16,
                 block_rows=64, grad_signed=True)


@pytest.mark.parametrize("D,opt,comb", [(4, "adam", "sum"), (8, "adagrad", "mean"),
                                        (12, "adam", "mean"), (48, "adagrad", "sum"),
                                        (96, "adam", "sum"), (256, "adagrad", "mean"),
                                        (1024, "adam", "sum")])
def test_dims_optimisers_combiners(R, D, opt, comb):
    w = W.WORKLOADS["tiny"].scaled(64)
    t = w.tables[0]
    w.tables = [W.TableSpec("t", t.features, D, opt, 0.05, comb, pooled=True, unpooled=True,
                            init_seed=99)]
    run_workload(R, w, steps=2)


# ---------------------------------------------------------------- edge cases
def _single(R, keys, lengths, D=16, opt="adagrad", comb="sum", F=1, steps=2, unpooled=False,
            grad_signed=False, init_acc=0.0):
    """Run explicit keys / bag lengths (F features x B bags) on both sides."""
    keys = np.asarray(keys, np.int64)
    lengths = np.asarray(lengths, np.int64)
    B = len(lengths) // F
    bo = np.zeros(len(lengths) + 1, np.int64)
    np.cumsum(lengths, out=bo[1:])
    assert bo[-1] == len(keys)
    spec = W.TableSpec("t", list(range(F)), D, opt, 0.05, comb, pooled=True, unpooled=unpooled,
                       init_seed=5)
    p = Pair(R, spec, init_acc=init_acc)
    k_dev = torch.from_numpy(keys).to(DEV)
    bo_dev = torch.from_numpy(bo).to(DEV)
    N = len(keys)
    for step in range(steps):
        pooled = torch.empty((B, F, D), dtype=torch.float32, device=DEV)
        unp = torch.empty((N, D), dtype=torch.float32, device=DEV) if unpooled else None
        p.gpu.lookup_pooled(p.batch, k_dev, bo_dev, F, B, p.combiner_r, pooled, unp)
        r = p.ora.lookup(keys, bo, F, B, p.combiner_o, unpooled=unpooled)
        uq, inv, rows, n_new = p.batch.get_unique(N)
        assert np.array_equal(uq.cpu().numpy(), r.uniq)
        assert np.array_equal(inv.cpu().numpy(), r.inv)
        assert np.array_equal(rows.cpu().numpy(), r.rows)
        assert n_new == r.n_new
        close(pooled.cpu().numpy(), r.pooled, "pooled")
        if unpooled:
            close(unp.cpu().numpy(), r.unpooled, "unpooled")
        gp = W.make_grad((B, F, D), 50 + step, signed=grad_signed)
        gu = W.make_grad((N, D), 60 + step, signed=grad_signed) if unpooled else None
        p.gpu.backward_update(p.batch, torch.from_numpy(gp).to(DEV),
                              None if gu is None else torch.from_numpy(gu).to(DEV))
        p.ora.backward_update(gp, gu)
        p.gpu.status_sync()
        compare_tables(p, f"step {step}")
    p.close()


def test_adagrad_initial_accumulator(R):
    # new rows' Adagrad state starts at the table's initial accumulator
    rng = np.random.default_rng(8)
    lengths = rng.integers(0, 5, size=600)
    keys = rng.integers(0, 2000, size=int(lengths.sum()))
    _single(R, keys, lengths, D=24, opt="adagrad", comb="mean", F=3, init_acc=0.25)


def test_empty_batch(R):
    _single(R, [], [0] * 10, opt="adam")


def test_empty_bags_mean(R):
    rng = np.random.default_rng(3)
    lengths = rng.integers(0, 4, size=400)
    lengths[:5] = 0
    lengths[-5:] = 0
    keys = rng.integers(0, 300, size=int(lengths.sum()))
    _single(R, keys, lengths, comb="mean", F=4)


@pytest.mark.parametrize("comb", ["sum", "mean"])
def test_one_huge_bag(R, comb):
    rng = np.random.default_rng(4)
    keys = rng.integers(0, 5000, size=60_000)
    _single(R, keys, [60_000], D=16, comb=comb, unpooled=True)


@pytest.mark.parametrize("D,comb", [(4, "sum"), (64, "mean"), (200, "sum"), (1024, "mean")])
def test_one_hot_stretches_among_multi_hot(R, D, comb):
    # runs of one-occurrence bags (gathered directly) cut by empty and
    # multi-occurrence bags (the segmented walk), with the unpooled output
    rng = np.random.default_rng(21 + D)
    F, B = 3, 3000
    lengths = np.ones(F * B, np.int64)
    for s in rng.choice(F * B, size=60, replace=False):
        lengths[s] = rng.choice([0, 2, 3])
    keys = rng.integers(0, 4000, size=int(lengths.sum()))
    _single(R, keys, lengths, D=D, comb=comb, F=F, unpooled=True, opt="adam")


def test_all_occurrences_one_key(R):
    # one unique key: the sort has no active pass and one segment spans every chunk
    _single(R, np.full(70_000, 123456789), np.ones(70_000, np.int64), D=32, opt="adam")


def test_adversarial_key_order_oversized_bucket(R):
    # the first call's splitters come from keys at fixed positions; put
    # spread-out keys there and crowd every other key between the two
    # smallest, so one bucket holds almost the whole batch and is sorted and
    # streamed from global memory
    N = 24_000
    rng = np.random.default_rng(12)
    keys = 1 + rng.permutation(1_000_000)[: N].astype(np.int64)
    for ns in (2048, 4096, 8192):
        sampled = (np.arange(ns, dtype=np.int64) * N) // ns
        keys[sampled] = np.arange(ns, dtype=np.int64) * 1_000_000_000
    _single(R, keys, np.ones(N, np.int64), D=8, steps=2)


@pytest.mark.parametrize("B", [12_602, 12_603, 15_000])
def test_batch_sizes_around_the_one_warp_local_sort(R, B):
    # 26 x B keys: 327,652 and 327,678 (one warp per bucket, 2047
    # splitters) and 390,000 (one CTA per bucket, 1023 splitters)
    run_workload(R, W.WORKLOADS["criteo26"].scaled(B), steps=2)


def test_splitter_reuse_across_batch_sizes(R):
    # one batch object, calls of 200K, 390K, 200K and 100K keys: quantiles of
    # 2047 splitters serve a 1023-splitter call (every second one); a call
    # that needs more splitters than the last call left draws a sample
    rng = np.random.default_rng(14)
    D = 8
    spec = W.TableSpec("t", [0], D, "adagrad", 0.05, "sum", pooled=True, init_seed=6)
    p = Pair(R, spec)
    for step, N in enumerate((200_000, 390_000, 200_000, 100_000)):
        keys = np.minimum(rng.zipf(1.1, size=N), 10**9).astype(np.int64) * 7_919 + rng.integers(0, 3, size=N)
        bo = np.arange(N + 1, dtype=np.int64)
        pooled = torch.empty((N, 1, D), dtype=torch.float32, device=DEV)
        p.gpu.lookup_pooled(p.batch, torch.from_numpy(keys).to(DEV), torch.from_numpy(bo).to(DEV),
                            1, N, R.SUM, pooled)
        r = p.ora.lookup(keys, bo, 1, N, O.SUM)
        uq, inv, rows, n_new = p.batch.get_unique(N)
        assert np.array_equal(uq.cpu().numpy(), r.uniq)
        assert np.array_equal(inv.cpu().numpy(), r.inv)
        assert np.array_equal(rows.cpu().numpy(), r.rows)
        assert n_new == r.n_new
        close(pooled.cpu().numpy(), r.pooled, f"pooled call {step}")
        gp = W.make_grad((N, 1, D), 80 + step)
        p.gpu.backward_update(p.batch, torch.from_numpy(gp).to(DEV))
        p.ora.backward_update(gp)
        p.gpu.status_sync()
        compare_tables(p, f"call {step}")
    p.close()


def test_hot_key_among_others(R):
    # one key holds 40% of the batch: its equality bucket is streamed
    N = 30_000
    rng = np.random.default_rng(13)
    keys = rng.integers(0, 1 << 40, size=N)
    keys[rng.random(N) < 0.4] = 77
    _single(R, keys, np.ones(N, np.int64), D=16, opt="adam", grad_signed=True)


@pytest.mark.parametrize("D,opt,comb,unpooled", [(4, "adagrad", "sum", False), (8, "adam", "mean", True),
                                                  (64, "adam", "sum", False), (256, "adam", "sum", True),
                                                  (1024, "adagrad", "mean", False)])
def test_long_segments_over_many_spans(R, D, opt, comb, unpooled):
    # over 524K occurrences: the long-segment reduction walks spans of more
    # than one 16-position chunk; keys of 20K occurrences span hundreds of
    # spans (combined by a whole CTA), keys of 300 or 40 a few (one lane
    # group), the rest are short; multi-hot bags, signed gradients
    rng = np.random.default_rng(21)
    keys = np.concatenate([np.repeat(np.arange(24, dtype=np.int64) * 1_000_003 + 11, 20_000),
                           np.repeat(np.arange(100, dtype=np.int64) * 7_919 + 3, 300),
                           np.repeat(np.arange(1000, dtype=np.int64) * 104_729 + 5, 40),
                           rng.integers(1 << 20, 1 << 44, size=100_000 if D <= 256 else 20_000)])
    keys = keys[rng.permutation(len(keys))]
    lengths = rng.integers(1, 9, size=len(keys))
    ends = np.cumsum(lengths)
    last = int(np.searchsorted(ends, len(keys)))
    lengths = lengths[: last + 1]
    lengths[-1] -= ends[last] - len(keys)
    assert lengths.min() > 0 and lengths.sum() == len(keys)
    _single(R, keys, lengths, D=D, opt=opt, comb=comb, unpooled=unpooled, grad_signed=True)


@pytest.mark.parametrize("N", [50_000, 1_700_000])
def test_new_rows_bit_exact(R, N):
    # fresh rows (seeded hash of the key; optimiser state initial) equal the
    # oracle's bit for bit, on the sample-sort path and on the radix path
    rng = np.random.default_rng(N)
    keys = rng.integers(-(1 << 62), 1 << 62, size=N)
    keys[keys == -1] = 7
    spec = W.TableSpec("t", [0], 8, "adagrad", 0.05, "sum", pooled=True, init_seed=17)
    p = Pair(R, spec, init_acc=0.125)
    bo = np.array([0, N], np.int64)
    pooled = torch.empty((1, 1, 8), dtype=torch.float32, device=DEV)
    p.gpu.lookup_pooled(p.batch, torch.from_numpy(keys).to(DEV), torch.from_numpy(bo).to(DEV), 1, 1,
                        p.combiner_r, pooled)
    p.ora.lookup(keys, bo, 1, 1, p.combiner_o)
    p.gpu.status_sync()
    gk, ge, gs, _ = p.gpu.export()
    ok, oe, os_ = p.ora.export()
    assert np.array_equal(gk, ok)
    assert np.array_equal(ge, oe)
    assert np.array_equal(gs, os_)
    p.close()


def test_gradients_in_pinned_host_memory(R):
    # gradients the GPU reads from pinned host memory (not device memory):
    # the backward gathers them with cp.async instead of the bulk-copy engine
    rng = np.random.default_rng(31)
    N, B, D = 40_000, 5_000, 32
    keys = np.concatenate([np.full(3_000, 42, np.int64), rng.integers(0, 1 << 40, size=N - 3_000)])
    keys = keys[rng.permutation(N)]
    bo = np.linspace(0, N, B + 1).astype(np.int64)
    spec = W.TableSpec("t", [0], D, "adam", 0.05, "mean", pooled=True, unpooled=True, init_seed=8)
    p = Pair(R, spec)
    k_dev, bo_dev = torch.from_numpy(keys).to(DEV), torch.from_numpy(bo).to(DEV)
    for step in range(2):
        pooled = torch.empty((B, 1, D), dtype=torch.float32, device=DEV)
        unp = torch.empty((N, D), dtype=torch.float32, device=DEV)
        p.gpu.lookup_pooled(p.batch, k_dev, bo_dev, 1, B, p.combiner_r, pooled, unp)
        p.ora.lookup(keys, bo, 1, B, p.combiner_o, unpooled=True)
        gp = W.make_grad((B, 1, D), 70 + step, signed=True)
        gu = W.make_grad((N, D), 80 + step, signed=True)
        gp_h = torch.from_numpy(gp).pin_memory()
        gu_h = torch.from_numpy(gu).pin_memory()
        # the binding takes CUDA tensors only; the C ABI takes any address the GPU can read
        assert R.load().recis_backward_update(p.gpu.handle, p.batch.handle, gp_h.data_ptr(), gu_h.data_ptr(),
                                              None) == R.OK
        torch.cuda.synchronize()
        p.ora.backward_update(gp, gu)
        p.gpu.status_sync()
        compare_tables(p, f"step {step}")
    p.close()


@pytest.mark.parametrize("comb", ["sum", "mean"])
def test_bag_lengths_around_the_pool_chunk(R, comb):
    # about 330K occurrences of D = 64: pool chunks of 32 positions; bags of
    # 1 to 100 occurrences, many one shorter or longer than half a chunk, a
    # chunk or two, so bags cross chunk ends whole (up to half a chunk long)
    # or are cut into pieces
    rng = np.random.default_rng(41)
    lengths = rng.choice([1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 100], size=9_000)
    N = int(lengths.sum())
    assert 227_500 <= N < 454_000  # chunks of 32 positions for this N and D
    keys = np.minimum(rng.zipf(1.2, size=N), 1 << 40).astype(np.int64) * 7_919
    _single(R, keys, lengths, D=64, opt="adam", comb=comb, unpooled=True, grad_signed=True)


def test_all_new_then_all_old(R):
    keys = np.arange(50_000, dtype=np.int64) * 1_000_003
    _single(R, keys[::-1].copy(), np.ones(50_000, np.int64), D=8, steps=3)


def test_negative_and_extreme_keys(R):
    keys = np.array([-(2**63), 2**63 - 1, -2, 0, 5, -(2**63), 7, 2**62], np.int64)
    _single(R, keys, [3, 0, 5], D=8)


def test_determinism(R):
    w = W.WORKLOADS["seq8"].scaled(64)
    outs = []
    for _ in range(2):
        pairs = run_workload(R, w, steps=2, return_pairs=True, check_unique=False)
        outs.append([p.gpu.export() for p in pairs])
        for p in pairs:
            p.close()
    for a, b in zip(outs[0], outs[1]):
        for x, y in zip(a[:3], b[:3]):
            assert np.array_equal(x, y)


def test_reserved_key_reported_and_table_stays_usable(R):
    t = R.Table(8, R.ADAGRAD, 0.1)
    b = R.Batch()
    keys = torch.tensor([3, -1, 4], dtype=torch.int64, device=DEV)
    bo = torch.tensor([0, 3], dtype=torch.int64, device=DEV)
    out = torch.empty((1, 1, 8), dtype=torch.float32, device=DEV)
    t.lookup_pooled(b, keys, bo, 1, 1, R.SUM, out)
    with pytest.raises(R.RecisError) as e:
        t.status_sync()
    assert e.value.code == 4
    keys2 = torch.tensor([3, 4], dtype=torch.int64, device=DEV)
    bo2 = torch.tensor([0, 2], dtype=torch.int64, device=DEV)
    t.lookup_pooled(b, keys2, bo2, 1, 1, R.SUM, out)
    t.status_sync()
    t.close()
    b.close()


def test_bad_arguments_rejected_on_host(R):
    t = R.Table(8, R.ADAGRAD, 0.1)
    b = R.Batch()
    keys = torch.tensor([3, 4], dtype=torch.int64, device=DEV)
    bo = torch.tensor([0, 2], dtype=torch.int64, device=DEV)
    with pytest.raises(R.RecisError):
        t.lookup_pooled(b, keys, bo, 1, 1, R.SUM, None, None)  # no output
    with pytest.raises(R.RecisError):
        t.backward_update(R.Batch())  # batch without lookup
    with pytest.raises(R.RecisError):
        R.Table(6, R.ADAGRAD, 0.1)  # dim not a multiple of 4
    t.close()
    b.close()


def test_export_import_round_trip(R):
    w = W.WORKLOADS["criteo26"].scaled(128)
    pairs = run_workload(R, w, steps=2, return_pairs=True)
    p = pairs[0]
    keys, emb, st, step = p.gpu.export()
    t2 = R.Table(p.spec.dim, R.ADAM, p.spec.lr, init_seed=p.spec.init_seed)
    t2.import_rows(keys, emb, st, step)
    k2, e2, s2, step2 = t2.export()
    assert np.array_equal(k2, keys) and np.array_equal(e2, emb) and np.array_equal(s2, st)
    assert step2 == step
    # one more step on both tables gives the same rows
    bt = W.make_batch(w, 7)
    dev = torch.device(DEV)
    kk = R.feature_hash([R.Feature(flags=f.flags, hash_seed=f.hash_seed, mod=f.mod, tag=f.tag,
                                   tag_shift=f.tag_shift) for f in w.features],
                        torch.from_numpy(bt.values).to(dev), bt.feat_offsets.tolist())
    bo = torch.from_numpy(bt.bag_offsets).to(dev)
    g = torch.from_numpy(W.make_grad((w.B, w.F, 64), 9)).to(dev)
    b2 = R.Batch()
    for t, bb in ((p.gpu, p.batch), (t2, b2)):
        out = torch.empty((w.B, w.F, 64), dtype=torch.float32, device=dev)
        t.lookup_pooled(bb, kk, bo, w.F, w.B, R.SUM, out)
        t.backward_update(bb, g)
    a, c = p.gpu.export(), t2.export()
    for x, y in zip(a[:3], c[:3]):
        assert np.array_equal(x, y)
    t2.close()
    b2.close()
    p.close()


def test_insert_returns_rows_of_every_key(R):
    t = R.Table(16, R.ADAM, 0.01)
    b = R.Batch()
    rng = np.random.default_rng(8)
    keys = rng.integers(0, 20_000, size=30_000)
    kd = torch.from_numpy(keys).to(DEV)
    rows = torch.empty_like(kd)
    t.insert(b, kd, rows)
    uq = np.unique(keys)
    r = rows.cpu().numpy()
    assert np.array_equal(r, np.searchsorted(uq, keys))  # new rows in ascending key order
    k, _, _, _ = t.export()
    assert np.array_equal(k, uq)
    t.close()
    b.close()
