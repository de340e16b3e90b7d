"""Error paths of the library, reached without faulting the GPU.

- A lookup holding the reserved key -1 is rejected as a whole (no key
  inserted, no row created) on both dedup paths; the table then equals the
  oracle's, which never saw that batch, and stays usable.
- A lookup whose new keys would pass max_rows is rejected as a whole with
  RECIS_ERR_TABLE_FULL and the table stays usable.
- A growth of the EmbeddingBlocks that cannot be mapped (a test cap on the
  mapped bytes stands in for a failed allocation) returns RECIS_ERR_OOM at
  once; the same lookup succeeds once the cap is lifted.
- A bounded device-side wait that gives up (the test lowers the bound to one
  poll) is reported, here through the allocation-free dedup (U = -1, every
  access in bounds), and the next call with the default bound is correct.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity_util import Pair, compare_tables

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


def _step(R, p, keys_np, B, gseed, expect_ok=True):
    """One lookup + backward of keys_np as B bags of near-equal length on
    both sides (the oracle only when the GPU call is expected to succeed)."""
    N = len(keys_np)
    bo = np.linspace(0, N, B + 1).astype(np.int64)
    D = p.spec.dim
    pooled = torch.empty((B, 1, D), dtype=torch.float32, device=DEV)
    p.gpu.lookup_pooled(p.batch, torch.from_numpy(keys_np).to(DEV), torch.from_numpy(bo).to(DEV),
                        1, B, p.combiner_r, pooled)
    gp = W.make_grad((B, 1, D), gseed, signed=True)
    if expect_ok:
        p.gpu.backward_update(p.batch, torch.from_numpy(gp).to(DEV))
        p.gpu.status_sync()
        r = p.ora.lookup(keys_np, bo, 1, B, p.combiner_o)
        p.ora.backward_update(gp)
        np.testing.assert_allclose(pooled.cpu().numpy(), r.pooled, rtol=1e-5, atol=1e-6)
        return None
    with pytest.raises(R.RecisError) as e:
        p.gpu.status_sync()
    return e.value.code


@pytest.mark.parametrize("N", [5000, 1_700_000])
def test_reserved_key_rejects_the_batch_whole(R, N):
    # N = 5000: sample-sort dedup; N = 1.7M: radix-sort dedup
    rng = np.random.default_rng(5)
    spec = W.TableSpec("t", [0], 16, "adam", 0.01, "sum", init_seed=3)
    p = Pair(R, spec)
    first = rng.integers(0, 1 << 40, size=3000).astype(np.int64)
    _step(R, p, first, 100, 1)
    bad = np.concatenate([first, rng.integers(1 << 41, 1 << 42, size=N - len(first) - 1),
                          [-1]]).astype(np.int64)
    assert len(bad) == N
    rng.shuffle(bad)
    n0 = p.gpu.size()[0]
    assert _step(R, p, bad, 200, 2, expect_ok=False) == R.recis.ERR_RESERVED_KEY
    assert p.gpu.size()[0] == n0  # nothing inserted
    compare_tables(p, "after the rejected batch")
    # keys of the rejected batch are new to both sides afterwards
    good = bad[bad != -1][:4000]
    _step(R, p, good, 150, 3)
    compare_tables(p, "after the batch that follows")
    p.close()


def test_table_full_rejects_the_batch_whole(R):
    rng = np.random.default_rng(6)
    spec = W.TableSpec("t", [0], 8, "adagrad", 0.1, "sum", init_seed=4)
    p = Pair(R, spec)
    p.gpu.close()
    p.gpu = R.Table(8, R.ADAGRAD, 0.1, init_seed=4, max_rows=1000)
    a = rng.choice(1 << 40, size=600, replace=False).astype(np.int64)
    _step(R, p, np.concatenate([a, a[:100]]), 50, 1)
    more = np.concatenate([a[:200], rng.integers(1 << 41, 1 << 42, size=500)]).astype(np.int64)
    assert _step(R, p, more, 50, 2, expect_ok=False) == R.recis.ERR_TABLE_FULL
    assert p.gpu.size()[0] == 600
    compare_tables(p, "after the rejected batch")
    fits = np.concatenate([a[:50], more[200:500]]).astype(np.int64)  # 300 new: 900 rows
    _step(R, p, fits, 40, 3)
    assert p.gpu.size()[0] == 900
    compare_tables(p, "after the batch that fits")
    p.close()


def test_growth_allocation_failure_reported(R):
    rng = np.random.default_rng(7)
    spec = W.TableSpec("t", [0], 64, "adam", 0.01, "sum", init_seed=5)
    p = Pair(R, spec)
    p.gpu.close()
    p.gpu = R.Table(64, R.ADAM, 0.01, init_seed=5, initial_capacity=1000, block_rows=1024)
    a = rng.integers(0, 1 << 40, size=1500).astype(np.int64)
    _step(R, p, a, 30, 1)
    big = rng.integers(1 << 41, 1 << 42, size=20000).astype(np.int64)
    R.recis.debug_set(R.recis.DEBUG_MAP_LIMIT, 2 << 20)  # the blocks mapped so far
    try:
        with pytest.raises(R.RecisError) as e:
            p.gpu.lookup_pooled(p.batch, torch.from_numpy(big).to(DEV),
                                torch.tensor([0, len(big)], dtype=torch.int64, device=DEV), 1, 1,
                                R.SUM, torch.empty((1, 1, 64), dtype=torch.float32, device=DEV))
        assert e.value.code == R.recis.ERR_OOM
    finally:
        R.recis.debug_set(R.recis.DEBUG_MAP_LIMIT, 0)
    compare_tables(p, "after the refused growth")
    _step(R, p, big, 200, 2)
    compare_tables(p, "after the growth")
    p.close()


def test_bounded_wait_gives_up_and_is_reported(R):
    rng = np.random.default_rng(8)
    keys_np = rng.integers(0, 50_000, size=262_144).astype(np.int64)
    keys = torch.from_numpy(keys_np).to(DEV)
    R.recis.debug_set(R.recis.DEBUG_SPIN_LIMIT, 1)
    gave_up = 0
    try:
        for _ in range(5):
            uniq, inv, U = R.recis.unique_static(keys)
            torch.cuda.synchronize()
            u = int(U.item())
            if u == -1:
                gave_up += 1
            else:  # the waits happened to find every predecessor done
                assert np.array_equal(uniq[:u].cpu().numpy(), np.unique(keys_np))
    finally:
        R.recis.debug_set(R.recis.DEBUG_SPIN_LIMIT, 0)
    assert gave_up > 0
    uniq, inv, U = R.recis.unique_static(keys)
    ref, ref_inv = np.unique(keys_np, return_inverse=True)
    u = int(U.item())
    assert u == len(ref)
    assert np.array_equal(uniq[:u].cpu().numpy(), ref)
    assert np.array_equal(inv.cpu().numpy(), ref_inv)


def test_misaligned_pointers_rejected_on_the_host(R):
    # vector loads and row copies need aligned arrays: the entry points
    # refuse a misaligned pointer before any work is queued, and the table
    # then works as before
    L = R.load()
    spec = W.TableSpec("t", [0], 16, "adagrad", 0.05, "sum", pooled=True, init_seed=3)
    p = Pair(R, spec)
    N, B, D = 64, 8, 16
    keys = torch.arange(1, N + 2, dtype=torch.int64, device=DEV)  # one spare element to shift into
    bo = torch.linspace(0, N, B + 1, device=DEV).to(torch.int64)
    pooled = torch.empty((B * D + 4,), dtype=torch.float32, device=DEV)
    s = None  # the legacy default stream
    bad_keys = keys.data_ptr() + 4
    assert L.recis_lookup_pooled(p.gpu.handle, p.batch.handle, bad_keys, N, bo.data_ptr(), 1, B, R.SUM,
                                 pooled.data_ptr(), None, s) == R.ERR_INVALID_ARG
    assert L.recis_lookup_pooled(p.gpu.handle, p.batch.handle, keys.data_ptr(), N, bo.data_ptr(), 1, B, R.SUM,
                                 pooled.data_ptr() + 4, None, s) == R.ERR_INVALID_ARG
    assert L.recis_lookup_pooled(p.gpu.handle, p.batch.handle, keys.data_ptr(), N, bo.data_ptr(), 1, B, R.SUM,
                                 pooled.data_ptr(), None, s) == R.OK
    grad = torch.ones((B * D + 4,), dtype=torch.float32, device=DEV)
    assert L.recis_backward_update(p.gpu.handle, p.batch.handle, grad.data_ptr() + 8, None, s) == R.ERR_INVALID_ARG
    assert L.recis_backward_update(p.gpu.handle, p.batch.handle, grad.data_ptr(), None, s) == R.OK
    p.gpu.status_sync()
    kh = keys[:N].cpu().numpy()
    p.ora.lookup(kh, bo.cpu().numpy(), 1, B, p.combiner_o)
    p.ora.backward_update(np.ones((B, 1, D), np.float32))
    compare_tables(p, "after the refused calls")
    p.close()
