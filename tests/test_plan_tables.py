"""Table merging (the A0 step: same-attribute tables merged into one logical
table at model-creation time, each feature tagged).  CPU only.

The oracle's plan is pinned against the groupings the workloads were written
with by hand from their configurations (criteo26: one table of 26 features
above 40-bit values; seq8: one table per dimension) and against brute-force
invariants on random feature sets; the library's recis_plan_tables, host code
that needs no GPU, must then give the same plan as the oracle.
"""
import itertools

import numpy as np
import pytest

import oracle as O
import workloads as W


def _attrs(t: W.TableSpec, bits: int, cap: int = 0):
    adam = t.optimizer == "adam"
    return dict(dim=t.dim, optimizer=O.ADAM if adam else O.ADAGRAD, lr=t.lr, beta1=0.9,
                beta2=0.999, eps=1e-8 if adam else 1e-10, adagrad_init_acc=0.0,
                init_scale=1.0 / np.sqrt(t.dim), init_seed=t.init_seed, capacity=cap,
                value_bits=bits)


def _workload_features(w: W.Workload):
    """Per feature (in order): the attributes of the table the workload puts it
    in, and its value width (40 bits after mod 2^40, else 48)."""
    owner = {f: t for t in w.tables for f in t.features}
    return [_attrs(owner[f], 40 if w.features[f].flags & W.MOD else 48, 1000)
            for f in range(w.F)]


@pytest.mark.parametrize("name", sorted(W.WORKLOADS))
def test_oracle_plan_matches_the_workloads_tables(name):
    w = W.WORKLOADS[name]
    table_of, tag_of, shift_of, caps = O.plan_tables(_workload_features(w))
    assert len(caps) == len(w.tables)
    for ti, t in enumerate(w.tables):
        members = [f for f in range(w.F) if table_of[f] == ti]
        assert members == list(t.features)                    # the hand-written grouping
        assert [int(tag_of[f]) for f in members] == list(range(len(members)))
        assert all(int(shift_of[f]) == w.features[f].tag_shift for f in members)
        assert caps[ti] == 1000 * len(members)


def _random_features(rng, F):
    dims = [8, 16, 64]
    feats = []
    for _ in range(F):
        d = int(rng.choice(dims))
        opt = int(rng.integers(0, 2))
        feats.append(dict(dim=d, optimizer=opt, lr=float(rng.choice([0.01, 0.001])), beta1=0.9,
                          beta2=0.999, eps=1e-8 if opt else 1e-10, adagrad_init_acc=0.0,
                          init_scale=float(rng.choice([0.1, 0.2])), init_seed=int(rng.integers(0, 2)),
                          capacity=int(rng.integers(0, 100)), value_bits=int(rng.integers(1, 50))))
    return feats


def _attr_key(a):
    return tuple(a[k] for k in ("dim", "optimizer", "lr", "beta1", "beta2", "eps",
                                "adagrad_init_acc", "init_scale", "init_seed"))


@pytest.mark.parametrize("seed", range(6))
def test_oracle_plan_brute_force_invariants(seed):
    rng = np.random.default_rng(seed)
    feats = _random_features(rng, 40)
    table_of, tag_of, shift_of, caps = O.plan_tables(feats)
    # same table iff same attributes
    for a, b in itertools.combinations(range(len(feats)), 2):
        assert (table_of[a] == table_of[b]) == (_attr_key(feats[a]) == _attr_key(feats[b]))
    # tables numbered by first appearance
    firsts = [int(np.nonzero(table_of == t)[0][0]) for t in range(len(caps))]
    assert firsts == sorted(firsts)
    for t in range(len(caps)):
        m = np.nonzero(table_of == t)[0]
        assert [int(tag_of[f]) for f in m] == list(range(len(m)))   # rank in the table
        assert all(shift_of[f] == max(feats[g]["value_bits"] for g in m) for f in m)
        assert caps[t] == sum(feats[f]["capacity"] for f in m)
        # tagged keys of different features never collide
        keys = {(int(tag_of[f]) << int(shift_of[f])) | v for f in m
                for v in (0, (1 << feats[f]["value_bits"]) - 1)}
        assert len(keys) == 2 * len(m) - sum(1 for f in m if feats[f]["value_bits"] == 0)


def test_oracle_plan_rejects_tags_that_do_not_fit():
    a = _attrs(W.WORKLOADS["tiny"].tables[0], 62)
    O.plan_tables([dict(a), dict(a)])            # 2 tags: 1 bit above 62 bits
    with pytest.raises(O.OracleError):
        O.plan_tables([dict(a), dict(a), dict(a)])  # 3 tags need 2 bits
    with pytest.raises(O.OracleError):
        O.plan_tables([dict(a, value_bits=63)])


def _lib_plan(R, feats):
    specs = []
    for a in feats:
        cfg = R.recis.table_config(a["dim"], a["optimizer"], a["lr"], beta1=a["beta1"],
                                   beta2=a["beta2"], eps=a["eps"],
                                   adagrad_init_acc=a["adagrad_init_acc"],
                                   init_scale=a["init_scale"], init_seed=a["init_seed"],
                                   initial_capacity=a["capacity"])
        specs.append((cfg, a["value_bits"]))
    return R.recis.plan_tables(specs)


@pytest.mark.parametrize("seed", range(6))
def test_library_plan_equals_oracle_plan(seed):
    import recommender_sparse_embedding_b200 as R
    from recommender_sparse_embedding_b200 import build
    build.build()
    R.load()
    rng = np.random.default_rng(100 + seed)
    feats = _random_features(rng, 60)
    table_of, tag_of, shift_of, caps = O.plan_tables(feats)
    plan = _lib_plan(R, feats)
    assert plan.table_of == [int(x) for x in table_of]
    assert plan.tag_of == [int(x) for x in tag_of]
    assert plan.tag_shift_of == [int(x) for x in shift_of]
    assert [c.initial_capacity for c in plan.tables] == [int(c) for c in caps]
    for t, c in enumerate(plan.tables):
        f = int(np.nonzero(table_of == t)[0][0])
        assert (c.dim, c.optimizer, c.lr, c.init_seed) == (feats[f]["dim"], feats[f]["optimizer"],
                                                           feats[f]["lr"], feats[f]["init_seed"])


def test_library_plan_of_the_workloads_and_errors():
    import recommender_sparse_embedding_b200 as R
    R.load()
    for w in W.WORKLOADS.values():
        feats = _workload_features(w)
        table_of, tag_of, shift_of, _ = O.plan_tables(feats)
        plan = _lib_plan(R, feats)
        assert plan.table_of == [int(x) for x in table_of]
        assert plan.tag_shift_of == [int(x) for x in shift_of]
    a = _attrs(W.WORKLOADS["tiny"].tables[0], 62)
    _lib_plan(R, [a, a])
    with pytest.raises(R.RecisError):
        _lib_plan(R, [a, a, a])
