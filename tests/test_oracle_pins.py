"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks one part of the oracle against a published value, a closed
form, an invariant, or a library routine that computes the same thing
(numpy.unique, numpy.searchsorted, torch.nn.functional.embedding_bag and its
autograd, torch.optim.Adagrad / Adam / SparseAdam in float64).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
M64 = 2**64 - 1


def _read_golden(name):
    seed = gamma = None
    vals = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("seed"):
                seed = int(line.split()[1], 0)
            elif line.startswith("gamma"):
                gamma = int(line.split()[1], 0)
            else:
                vals.append(int(line))
    return seed, gamma, vals


# ---------------------------------------------------------------- hash / mod / tag
def test_hash_matches_published_splitmix64_vector():
    seed, gamma, vals = _read_golden("splitmix64_seed1234567.txt")
    for k, v in enumerate(vals, start=1):
        assert O.hash64((seed + k * gamma) & M64) == v


def test_hash_is_bijective_on_a_million_inputs():
    rng = np.random.default_rng(1)
    x = np.unique(rng.integers(-(2**63), 2**63 - 1, size=1_000_000, dtype=np.int64))
    ops = [O.FeatureOp(flags=O.HASH, hash_seed=0)]
    k = O.feature_hash(ops, x, np.array([0, len(x)]))
    assert len(np.unique(k)) == len(x)


def test_hash_seed_mod_and_negative_ids():
    x = np.array([0, 1, -5, 2**62 + 3, -(2**63), 123456789], np.int64)
    seed = 0xDEADBEEF12345
    mod = 10_000_019
    ops = [O.FeatureOp(flags=O.HASH | O.MOD, hash_seed=seed, mod=mod)]
    k = O.feature_hash(ops, x, np.array([0, len(x)]))
    for xi, ki in zip(x.tolist(), k.tolist()):
        # negative IDs are reinterpreted as uint64; remainder is unsigned
        assert ki == O.hash64((xi & M64) ^ seed) % mod
    # mod 2^40 is the low-40-bit mask (closed form)
    ops = [O.FeatureOp(flags=O.HASH | O.MOD, hash_seed=seed, mod=1 << 40)]
    k40 = O.feature_hash(ops, x, np.array([0, len(x)]))
    full = O.feature_hash([O.FeatureOp(flags=O.HASH, hash_seed=seed)], x, np.array([0, len(x)]))
    assert np.array_equal(k40, full & ((1 << 40) - 1))


def test_tag_layout_and_overflow():
    x = np.arange(0, 1000, dtype=np.int64) * 977
    offs = np.array([0, 500, 1000])
    ops = [O.FeatureOp(flags=O.TAG, tag=3, tag_shift=48), O.FeatureOp(flags=O.TAG, tag=77, tag_shift=48)]
    k = O.feature_hash(ops, x, offs)
    assert np.all(k[:500] >> 48 == 3) and np.all(k[500:] >> 48 == 77)
    assert np.array_equal(k & ((1 << 48) - 1), x)
    with pytest.raises(O.OracleError) as e:
        O.feature_hash([O.FeatureOp(flags=O.TAG, tag=1, tag_shift=8)], np.array([256]), np.array([0, 1]))
    assert e.value.code == O.INVALID_ARG
    with pytest.raises(O.OracleError):  # tag too wide for the bits above the shift
        O.feature_hash([O.FeatureOp(flags=O.TAG, tag=1 << 15, tag_shift=48)], np.array([1]), np.array([0, 1]))


def test_bucketize_is_numpy_searchsorted_right():
    rng = np.random.default_rng(2)
    b = np.unique(rng.integers(-1000, 1000, size=37))
    x = rng.integers(-1200, 1200, size=5000)
    x[:len(b)] = b  # values equal to boundaries
    ops = [O.FeatureOp(flags=O.BUCKETIZE | O.TAG, tag=5, tag_shift=40, boundaries=b.tolist())]
    k = O.feature_hash(ops, x, np.array([0, len(x)]))
    assert np.array_equal(k & ((1 << 40) - 1), np.searchsorted(b, x, side="right"))
    assert np.all(k >> 40 == 5)
    with pytest.raises(O.OracleError):
        O.feature_hash([O.FeatureOp(flags=O.BUCKETIZE | O.HASH)], x, np.array([0, len(x)]))


def test_float_bucketize_hand_worked_values():
    # boundaries -1.5, 0, 2.25, 1e300: the count of boundaries <= x, compared
    # as doubles (-0.0 equals 0.0; a NaN is above no boundary)
    b = [-1.5, 0.0, 2.25, 1e300]
    xs = np.array([-np.inf, -1.5, -1.4999, -0.0, 0.0, 5e-324, 2.25, 3.0, 1e300, np.inf, np.nan,
                   -np.nan], dtype=np.float64)
    want = [0, 1, 1, 2, 2, 2, 3, 3, 4, 4, 0, 0]
    ops = [O.FeatureOp(flags=O.BUCKETIZE | O.FLOAT | O.TAG, tag=3, tag_shift=48, boundaries=b)]
    k = O.feature_hash(ops, xs.view(np.int64), np.array([0, len(xs)]))
    assert (k & ((1 << 48) - 1)).tolist() == want
    assert np.all(k >> 48 == 3)
    # FLOAT without BUCKETIZE is not an op
    with pytest.raises(O.OracleError):
        O.feature_hash([O.FeatureOp(flags=O.FLOAT)], xs.view(np.int64), np.array([0, len(xs)]))


def test_float_bucketize_is_numpy_searchsorted_right():
    rng = np.random.default_rng(5)
    b = np.unique(np.round(rng.normal(size=63), 2))
    x = np.round(rng.normal(scale=1.5, size=6000), 2)  # many values equal to boundaries
    x[:len(b)] = b
    ops = [O.FeatureOp(flags=O.BUCKETIZE | O.FLOAT, boundaries=b.tolist()),
           O.FeatureOp(flags=O.BUCKETIZE, boundaries=[-3, 0, 7])]
    ints = np.arange(-5, 10, dtype=np.int64)
    vals = np.concatenate([x.view(np.int64), ints])
    k = O.feature_hash(ops, vals, np.array([0, len(x), len(vals)]))
    assert np.array_equal(k[:len(x)], np.searchsorted(b, x, side="right"))
    assert np.array_equal(k[len(x):], np.searchsorted(np.array([-3, 0, 7]), ints, side="right"))


# ---------------------------------------------------------------- dedup / IDMap
def _tiny_batch(seed=0, B=64):
    w = W.WORKLOADS["tiny"].scaled(B)
    b = W.make_batch(w, 0, seed=seed)
    keys = O.feature_hash([O.FeatureOp(flags=O.TAG, tag=f, tag_shift=48) for f in range(w.F)],
                          b.values, b.feat_offsets)
    return w, b, keys


def test_dedup_is_numpy_unique_and_rows_are_a_bijection():
    w, b, keys = _tiny_batch()
    t = O.Table(16, O.ADAGRAD, 0.01, init_seed=3)
    r = t.lookup(keys, b.bag_offsets, w.F, w.B)
    u, inv = np.unique(keys, return_inverse=True)
    assert np.array_equal(r.uniq, u) and np.array_equal(r.inv, inv)
    assert np.array_equal(r.uniq[r.inv], keys)
    assert r.n_new == len(u) and t.size == len(u)
    # first batch: new rows are consecutive in ascending key order
    assert np.array_equal(r.rows, np.arange(len(u)))
    # second batch: old keys keep rows, new keys get the next rows in key order
    _, b2, keys2 = _tiny_batch(seed=9)
    r2 = t.lookup(keys2, b2.bag_offsets, w.F, w.B)
    old = dict(zip(r.uniq.tolist(), r.rows.tolist()))
    new_keys = [k for k in r2.uniq.tolist() if k not in old]
    for k, row in zip(r2.uniq.tolist(), r2.rows.tolist()):
        if k in old:
            assert row == old[k]
    new_rows = [row for k, row in zip(r2.uniq.tolist(), r2.rows.tolist()) if k not in old]
    assert new_rows == list(range(len(u), len(u) + len(new_keys)))
    assert r2.n_new == len(new_keys)
    ek, _, _ = t.export()
    assert len(set(ek.tolist())) == t.size  # one row per key
    for k, row in zip(r2.uniq.tolist(), r2.rows.tolist()):
        assert ek[row] == k


def test_reserved_key_and_bad_offsets_are_rejected():
    t = O.Table(4, O.ADAGRAD, 0.1)
    with pytest.raises(O.OracleError) as e:
        t.lookup(np.array([1, -1, 2]), np.array([0, 3]), 1, 1)
    assert e.value.code == O.RESERVED_KEY
    with pytest.raises(O.OracleError):
        t.lookup(np.array([1, 2]), np.array([0, 3]), 1, 1)
    assert t.size == 0


def test_empty_batch():
    t = O.Table(8, O.ADAM, 0.1)
    r = t.lookup(np.zeros(0, np.int64), np.zeros(4, np.int64), 1, 3)
    assert r.pooled.shape == (3, 1, 8) and np.all(r.pooled == 0) and len(r.uniq) == 0
    t.backward_update(np.ones((3, 1, 8), np.float32))
    assert t.step == 1 and t.size == 0


# ---------------------------------------------------------------- initialiser
def test_init_range_granularity_and_independence():
    D = 32
    t = O.Table(D, O.ADAM, 0.1, init_seed=77)
    keys = np.arange(4000, dtype=np.int64) * 7919 + 13
    t.lookup(keys, np.array([0, len(keys)]), 1, 1)
    k, emb, st = t.export()
    s = np.float32(1.0 / math.sqrt(D))
    assert np.all(emb >= -s) and np.all(emb < s)
    # emb is the one fp32 rounding of (q * 2^-24 - 1/2) * 2s for an integer
    # q in [0, 2^24): recover q and rebuild the value
    u = emb.astype(np.float64) / (2.0 * float(s)) + 0.5
    q = np.round(u * 2**24)
    assert np.all(q >= 0) and np.all(q < 2**24)
    assert np.array_equal(((q / 2**24 - 0.5) * (2.0 * float(s))).astype(np.float32), emb)
    assert abs(emb.mean()) < 3e-3
    assert abs(emb.var() - float(s) ** 2 / 3) < 0.02 * float(s) ** 2
    # columns and keys differ (no dropped index)
    assert len(np.unique(emb[0])) == D and len(np.unique(emb[:, 0])) > 3990
    assert np.all(st == 0)
    # the row depends on (key, seed) only, not on insertion order
    t2 = O.Table(D, O.ADAM, 0.1, init_seed=77)
    t2.lookup(keys[::-1].copy(), np.array([0, len(keys)]), 1, 1)
    k2, e2, _ = t2.export()
    m2 = dict(zip(k2.tolist(), range(len(k2))))
    assert np.array_equal(e2[[m2[x] for x in k.tolist()]], emb)
    t3 = O.Table(D, O.ADAM, 0.1, init_seed=78)
    t3.lookup(keys, np.array([0, len(keys)]), 1, 1)
    assert not np.array_equal(t3.export()[1], emb)
    t4 = O.Table(D, O.ADAGRAD, 0.1, adagrad_init_acc=0.25)
    t4.lookup(keys[:5], np.array([0, 5]), 1, 1)
    assert np.all(t4.export()[2] == np.float32(0.25))


def test_init_row_rebuilt_from_the_hash():
    # a fresh row rebuilt value by value from the pinned hash: seed mixed into
    # the key, one hash per column, the top 24 bits as a uniform on [0, 1)
    D, seed = 8, 0x1234_5678_9ABC_DEF0
    t = O.Table(D, O.ADAM, 0.1, init_seed=seed)
    keys = np.array([0, 1, -2, 123456789, -(1 << 62), (1 << 62) + 5], np.int64)  # -1 is reserved
    t.lookup(keys, np.array([0, len(keys)]), 1, 1)
    k, emb, _ = t.export()
    two_s = 2.0 * float(np.float32(1.0 / math.sqrt(D)))
    for key, row in zip(k.tolist(), emb):
        base = O.hash64((key & M64) ^ seed)
        want = [np.float32(((O.hash64((base + j) & M64) >> 40) / 2.0**24 - 0.5) * two_s) for j in range(D)]
        assert np.array_equal(row, np.array(want, np.float32))


# ---------------------------------------------------------------- pooling / grad
def _dense(t):
    k, emb, st = t.export()
    return torch.from_numpy(emb.astype(np.float64))


@pytest.mark.parametrize("combiner", [O.SUM, O.MEAN])
def test_pooling_is_embedding_bag(combiner):
    w = W.WORKLOADS["tiny"].scaled(96)
    b = W.make_batch(w, 0)
    # include empty bags
    lengths = b.lengths.copy()
    lengths[::7] = 0
    bo = np.zeros(len(lengths) + 1, np.int64)
    np.cumsum(lengths, out=bo[1:])
    keys = (np.arange(bo[-1]) * 31 % 500).astype(np.int64)
    t = O.Table(16, O.ADAGRAD, 0.01, init_seed=5)
    r = t.lookup(keys, bo, w.F, w.B, combiner=combiner, unpooled=True)
    Wt = _dense(t)
    idx = torch.from_numpy(r.rows[r.inv].astype(np.int64))
    mode = "sum" if combiner == O.SUM else "mean"
    ref = torch.nn.functional.embedding_bag(idx, Wt, torch.from_numpy(bo[:-1]), mode=mode)
    ref = ref.reshape(w.F, w.B, 16).transpose(0, 1).numpy().astype(np.float32)
    assert np.array_equal(r.pooled, ref)  # double sum, one rounding: identical
    assert np.array_equal(r.unpooled, Wt.numpy().astype(np.float32)[r.rows[r.inv]])


@pytest.mark.parametrize("combiner", [O.SUM, O.MEAN])
def test_gradient_is_autograd_of_embedding_bag(combiner):
    w = W.WORKLOADS["tiny"].scaled(80)
    b = W.make_batch(w, 1)
    keys = (b.values % 300).astype(np.int64)
    t = O.Table(16, O.ADAGRAD, 0.01, init_seed=5)
    r = t.lookup(keys, b.bag_offsets, w.F, w.B, combiner=combiner, unpooled=True)
    gp = W.make_grad((w.B, w.F, 16), 3, signed=True)
    gu = W.make_grad((len(keys), 16), 4, signed=True)
    Wt = _dense(t).clone().requires_grad_(True)
    idx = torch.from_numpy(r.rows[r.inv].astype(np.int64))
    mode = "sum" if combiner == O.SUM else "mean"
    out = torch.nn.functional.embedding_bag(idx, Wt, torch.from_numpy(b.bag_offsets[:-1]), mode=mode)
    out = out.reshape(w.F, w.B, 16).transpose(0, 1)
    un = torch.nn.functional.embedding(idx, Wt)
    loss = (out * torch.from_numpy(gp).double()).sum() + (un * torch.from_numpy(gu).double()).sum()
    loss.backward()
    g = t.backward_update(gp, gu, return_grad=True, n_unique=len(r.uniq))
    np.testing.assert_allclose(g, Wt.grad.numpy()[r.rows], rtol=1e-12, atol=1e-12)


def test_gradient_counts_each_occurrence_once():
    keys = np.array([5, 9, 5, 5, 2, 9, 5, 11], np.int64)
    bo = np.array([0, 1, 3, 6, 8])  # 4 bags, F=1
    t = O.Table(4, O.ADAGRAD, 0.1)
    r = t.lookup(keys, bo, 1, 4)
    g = t.backward_update(np.ones((4, 1, 4), np.float32), return_grad=True, n_unique=len(r.uniq))
    counts = np.array([np.sum(keys == k) for k in r.uniq], np.float64)
    assert np.array_equal(g, np.repeat(counts[:, None], 4, axis=1))


# ---------------------------------------------------------------- optimisers
def _one_row_table(opt, lr, w0, **kw):
    t = O.Table(len(w0), opt, lr, **kw)
    t.import_rows(np.array([7]), np.array([w0], np.float32))
    return t


def test_adagrad_constant_gradient_closed_form():
    # acc_k = k g^2, so step k moves lr * sign(g) / sqrt(k)
    w0 = np.array([1.0, -2.0, 0.5, 0.0])
    g = np.array([0.5, -1.0, 2.0, 0.0], np.float32)
    t = _one_row_table(O.ADAGRAD, 0.1, w0)
    for k in range(1, 6):
        t.lookup(np.array([7]), np.array([0, 1]), 1, 1)
        t.backward_update(g.reshape(1, 1, 4))
        expect = w0 - 0.1 * np.sign(g) * sum(1 / math.sqrt(i) for i in range(1, k + 1))
        _, emb, st = t.export()
        np.testing.assert_allclose(emb[0], expect, rtol=2e-7, atol=1e-7)
        np.testing.assert_allclose(st[0], k * g.astype(np.float64) ** 2, rtol=1e-7)


def test_adam_constant_gradient_closed_form():
    # with a constant gradient the bias-corrected moments are g and g^2, so
    # every step moves lr * sign(g) (eps is negligible here)
    w0 = np.array([1.0, -2.0, 0.5, 0.0])
    g = np.array([0.5, -1.0, 2.0, 0.0], np.float32)
    t = _one_row_table(O.ADAM, 0.1, w0)
    for k in range(1, 6):
        t.lookup(np.array([7]), np.array([0, 1]), 1, 1)
        t.backward_update(g.reshape(1, 1, 4))
        _, emb, st = t.export()
        np.testing.assert_allclose(emb[0], w0 - 0.1 * k * np.sign(g), rtol=1e-6, atol=2e-7)
        np.testing.assert_allclose(st[0, :4], (1 - 0.9**k) * g, rtol=1e-6)
        np.testing.assert_allclose(st[0, 4:], (1 - 0.999**k) * g.astype(np.float64) ** 2, rtol=1e-6)
    assert t.step == 5


def _run_vs_torch(opt, steps=3, all_touched=True, eps=None, init_acc=0.0):
    D, F, B = 8, 2, 24
    rng = np.random.default_rng(11)
    keys0 = np.unique(rng.integers(0, 1000, size=60))
    t = O.Table(D, opt, 0.05, eps=eps, init_seed=2, adagrad_init_acc=init_acc)
    t.lookup(keys0, np.array([0, len(keys0)]), 1, 1)  # insert all keys, no update
    _, emb, st = t.export()
    Wt = torch.nn.Parameter(torch.from_numpy(emb.astype(np.float64)))
    if opt == O.ADAGRAD:
        topt = torch.optim.Adagrad([Wt], lr=0.05, eps=1e-10 if eps is None else eps,
                                   initial_accumulator_value=init_acc)
    elif all_touched:
        topt = torch.optim.Adam([Wt], lr=0.05, betas=(0.9, 0.999), eps=1e-8 if eps is None else eps)
    else:
        topt = torch.optim.SparseAdam([Wt], lr=0.05, betas=(0.9, 0.999), eps=eps)
    for s in range(steps):
        lengths = rng.integers(1, 6, size=F * B)
        bo = np.zeros(F * B + 1, np.int64)
        np.cumsum(lengths, out=bo[1:])
        n = int(bo[-1])
        if all_touched:
            sel = np.concatenate([np.arange(len(keys0)), rng.integers(0, len(keys0), size=n - len(keys0))])
            rng.shuffle(sel)
        else:
            sel = rng.integers(0, len(keys0) // 2 + 5 * s, size=n)
        keys = keys0[sel]
        r = t.lookup(keys, bo, F, B)
        gp = W.make_grad((B, F, D), 100 + s, signed=True)
        t.backward_update(gp)
        idx = torch.from_numpy(r.rows[r.inv].astype(np.int64))
        out = torch.nn.functional.embedding_bag(idx, Wt, torch.from_numpy(bo[:-1]), mode="sum",
                                                sparse=not all_touched)
        loss = (out.reshape(F, B, D).transpose(0, 1) * torch.from_numpy(gp).double()).sum()
        topt.zero_grad()
        loss.backward()
        topt.step()
    _, emb, st = t.export()
    np.testing.assert_allclose(emb, Wt.detach().numpy(), rtol=1e-5, atol=1e-6)
    return t, topt, Wt, st


def test_adagrad_matches_torch_adagrad():
    t, topt, Wt, st = _run_vs_torch(O.ADAGRAD)
    np.testing.assert_allclose(st, topt.state[Wt]["sum"].numpy(), rtol=1e-5, atol=1e-6)


def test_adagrad_initial_accumulator_matches_torch_adagrad():
    # a table's Adagrad accumulator starts at adagrad_init_acc, like
    # torch.optim.Adagrad's initial_accumulator_value
    t, topt, Wt, st = _run_vs_torch(O.ADAGRAD, init_acc=0.25)
    np.testing.assert_allclose(st, topt.state[Wt]["sum"].numpy(), rtol=1e-5, atol=1e-6)


def test_adam_matches_torch_adam_when_all_rows_touched():
    t, topt, Wt, st = _run_vs_torch(O.ADAM)
    D = Wt.shape[1]
    np.testing.assert_allclose(st[:, :D], topt.state[Wt]["exp_avg"].numpy(), rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(st[:, D:], topt.state[Wt]["exp_avg_sq"].numpy(), rtol=1e-5, atol=1e-9)


def test_lazy_adam_matches_sparse_adam_with_vanishing_eps():
    # SparseAdam adds eps before bias correction, torch.optim.Adam after it;
    # with eps -> 0 the two forms coincide and SparseAdam pins the lazy,
    # touched-rows-only update with one step counter per table.
    t, topt, Wt, st = _run_vs_torch(O.ADAM, steps=4, all_touched=False, eps=1e-30)
    assert t.step == 4
