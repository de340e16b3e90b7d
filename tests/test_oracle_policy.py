"""Pins of the oracle's admission and eviction (RecIS README, Core architecture
> Embedding Engine: the table supports feature eviction and admission
policies).  Readings (the README names the policies only): a key not in the
table is a candidate whose count rises by one per lookup it appears in, and it
gets a row on the lookup where the count reaches the threshold; every lookup
advances the table's clock; eviction removes rows and candidates last touched
before a given clock; freed rows are reused by later new keys, oldest first,
in ascending row order.  Each case below is worked by hand.
"""
import numpy as np

import oracle as O

D = 4


def _look(t, keys, bags=None, comb=O.SUM):
    keys = np.asarray(keys, np.int64)
    bo = np.array(bags if bags is not None else [0, len(keys)], np.int64)
    return t.lookup(keys, bo, 1, len(bo) - 1, comb)


def _init_rows(keys):
    """The initial rows of keys, from a plain table that admits at once."""
    ref = O.Table(D, O.ADAGRAD, 0.1)
    r = _look(ref, sorted(keys), list(range(len(keys) + 1)))
    k, e, _ = ref.export()
    return {int(a): e[i] for i, a in enumerate(k)}


def test_admission_counts_lookups_not_occurrences():
    t = O.Table(D, O.ADAGRAD, 0.1, admit_threshold=3)
    A, B = 10, 20
    r = _look(t, [A, A, B])                       # lookup 1: A x2, B x1 -> counts 1, 1
    assert list(r.rows) == [-1, -1] and r.n_new == 0 and t.size == 0
    assert not r.pooled.any()                     # candidates pool as zeros
    t.backward_update(np.ones((1, 1, D), np.float32))
    assert t.size == 0                            # their gradient is dropped
    r = _look(t, [A])                             # lookup 2: A -> 2
    assert list(r.rows) == [-1] and t.size == 0
    r = _look(t, [A, B])                          # lookup 3: A -> 3 admitted, B -> 2
    assert list(r.rows) == [0, -1] and r.n_new == 1 and t.size == 1
    init = _init_rows([A, B])
    np.testing.assert_array_equal(r.pooled[0, 0], init[A])   # B adds zeros
    r = _look(t, [A, B], comb=O.MEAN)             # lookup 4: B -> 3 admitted (row 1)
    assert list(r.rows) == [0, 1] and r.n_new == 1
    k, e, _ = t.export()
    assert list(k) == [A, B]


def test_candidate_mean_divides_by_the_whole_bag():
    t = O.Table(D, O.ADAGRAD, 0.1, admit_threshold=2)
    A, B = 3, 4
    _look(t, [A])                                  # A -> 1
    r = _look(t, [A, B], comb=O.MEAN)              # A admitted, B candidate
    init = _init_rows([A])
    np.testing.assert_allclose(r.pooled[0, 0], (init[A].astype(np.float64) / 2).astype(np.float32))


def test_gradient_reaches_only_admitted_rows():
    g = np.full((1, 1, D), 0.5, np.float32)
    t = O.Table(D, O.ADAGRAD, 0.1, admit_threshold=2)
    _look(t, [7])
    _look(t, [7, 8])                               # 7 admitted, 8 candidate
    t.backward_update(g)
    ref = O.Table(D, O.ADAGRAD, 0.1)               # the same step on key 7 alone
    _look(ref, [7])
    ref.backward_update(g)
    k, e, s = t.export()
    rk, re, rs = ref.export()
    assert list(k) == [7]
    np.testing.assert_array_equal(e, re)
    np.testing.assert_array_equal(s, rs)


def test_eviction_frees_rows_in_row_order_and_new_keys_reuse_them():
    t = O.Table(D, O.ADAGRAD, 0.1)
    r = _look(t, [5, 1, 3])                        # clock 1: rows 1->0, 3->1, 5->2
    assert list(r.rows) == [0, 1, 2]
    t.backward_update(np.ones((1, 1, D), np.float32))
    _look(t, [3, 7])                               # clock 2: 3 touched, 7 -> row 3
    _look(t, [1])                                  # clock 3: 1 touched
    assert t.clock == 3
    assert t.evict(3) == 3                         # rows of 3 (clock 2), 5 (1), 7 (2)
    k, _, _ = t.export()
    assert list(k) == [1] and t.size == 1
    r = _look(t, [9, 2, 5])                        # new keys 2, 5, 9 take rows 1, 2, 3
    assert list(r.uniq) == [2, 5, 9] and list(r.rows) == [1, 2, 3] and r.n_new == 3
    k, e, s = t.export()
    assert list(k) == [1, 2, 5, 9]
    init = _init_rows([5])
    np.testing.assert_array_equal(e[2], init[5])   # 5 starts over from its initial row
    assert not s[2].any()                          # and its optimiser state


def test_eviction_removes_candidates_too():
    t = O.Table(D, O.ADAGRAD, 0.1, admit_threshold=2)
    _look(t, [11])                                 # clock 1: 11 -> count 1
    _look(t, [12])                                 # clock 2
    t.evict(2)                                     # 11 last seen at clock 1: dropped
    r = _look(t, [11])                             # count starts over: 1
    assert list(r.rows) == [-1]
    r = _look(t, [11])                             # 2: admitted
    assert list(r.rows) == [0]


def test_random_policy_invariants():
    rng = np.random.default_rng(3)
    t = O.Table(D, O.ADAM, 0.01, admit_threshold=2)
    seen = {}        # key -> clock of its last lookup (tracked here, by hand)
    counts = {}      # candidate key -> lookups seen in
    live = set()
    for step in range(40):
        keys = rng.integers(0, 60, size=rng.integers(1, 30))
        r = _look(t, keys)
        clock = t.clock
        for k in np.unique(keys):
            k = int(k)
            seen[k] = clock
            if k not in live:
                counts[k] = counts.get(k, 0) + 1
                if counts[k] >= 2:
                    live.add(k)
                    del counts[k]
        assert set(int(k) for k, rw in zip(r.uniq, r.rows) if rw >= 0) == live & set(int(k) for k in keys)
        t.backward_update(rng.random((1, 1, D)).astype(np.float32))
        if step % 7 == 6:
            cut = clock - 3
            gone = {k for k in live if seen[k] < cut}
            assert t.evict(cut) == len(gone)
            live -= gone
            counts = {k: c for k, c in counts.items() if seen[k] >= cut}
        k, _, _ = t.export()
        assert set(int(x) for x in k) == live and len(k) == len(set(k)) == t.size
