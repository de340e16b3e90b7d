"""Admission and eviction on the GPU against the oracle (the Embedding
Engine's feature admission and eviction policies of the RecIS README).

Every step compares the dedup (rows are -1 for keys that are still
candidates), the pooled rows and the whole exported table, with eviction on
both sides at the same clocks, through both dedup paths (sample sort for
batches up to 1.6M keys, radix sort above).
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity_util import Pair, close, compare_tables, run_workload

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


@pytest.mark.parametrize("name,B,T", [("tiny", 256, 2), ("criteo26", 1024, 3), ("seq8", 64, 2),
                                       ("longseq", 8, 2)])
def test_admission_parity(R, name, B, T):
    run_workload(R, W.WORKLOADS[name].scaled(B), steps=4, admit_threshold=T, grad_signed=True)


@pytest.mark.parametrize("name,B,T,every,age", [("tiny", 256, 1, 2, 2), ("criteo26", 1024, 2, 2, 1),
                                                 ("seq8", 64, 1, 3, 2)])
def test_eviction_parity(R, name, B, T, every, age):
    run_workload(R, W.WORKLOADS[name].scaled(B), steps=6, admit_threshold=T, evict_every=every,
                 evict_age=age)


def test_admission_and_eviction_on_the_radix_path(R):
    # batches above the sample-sort limit: the radix dedup and its unique pass
    rng = np.random.default_rng(41)
    spec = W.TableSpec("t", [0], 8, "adam", 0.01, "sum", init_seed=29)
    p = Pair(R, spec, admit_threshold=2, evictable=True)
    B = 700_000
    for step in range(3):
        lengths = rng.integers(1, 5, size=B).astype(np.int64)
        bo = np.zeros(B + 1, np.int64)
        np.cumsum(lengths, out=bo[1:])
        N = int(bo[-1])
        assert N > 1_600_000
        keys = rng.integers(0, 900_000, size=N).astype(np.int64) * 7919 - 3_000_000_000
        pooled = torch.empty((B, 1, 8), dtype=torch.float32, device=DEV)
        p.gpu.lookup_pooled(p.batch, torch.from_numpy(keys).to(DEV), torch.from_numpy(bo).to(DEV),
                            1, B, R.SUM, pooled)
        r = p.ora.lookup(keys, bo, 1, B, O.SUM)
        uq, inv, rows, n_new = p.batch.get_unique(N)
        assert np.array_equal(uq.cpu().numpy(), r.uniq)
        assert np.array_equal(rows.cpu().numpy(), r.rows)
        assert n_new == r.n_new
        close(pooled.cpu().numpy(), r.pooled, f"pooled step {step}")
        gp = W.make_grad((B, 1, 8), 90 + step, signed=True)
        p.gpu.backward_update(p.batch, torch.from_numpy(gp).to(DEV))
        p.ora.backward_update(gp)
        p.gpu.status_sync()
        compare_tables(p, f"step {step}")
        if step == 1:
            cut = p.ora.clock
            assert p.gpu.evict(cut) == p.ora.evict(cut)
            compare_tables(p, "after eviction")
    p.close()


def test_evicted_rows_are_reused_in_row_order_and_save_skips_them(R, tmp_path):
    spec = W.TableSpec("t", [0], 16, "adagrad", 0.1, "sum", init_seed=31)
    p = Pair(R, spec, evictable=True)
    for keys in ([5, 1, 3], [3, 7], [1]):
        k = np.array(keys, np.int64)
        bo = np.array([0, len(k)], np.int64)
        out = torch.empty((1, 1, 16), dtype=torch.float32, device=DEV)
        p.gpu.lookup_pooled(p.batch, torch.from_numpy(k).to(DEV), torch.from_numpy(bo).to(DEV), 1, 1,
                            R.SUM, out)
        p.ora.lookup(k, bo, 1, 1)
    assert p.gpu.evict(3) == p.ora.evict(3) == 3
    compare_tables(p, "after eviction")
    path = str(tmp_path / "t.safetensors")
    p.gpu.save(path)
    from safetensors.numpy import load_file
    assert list(load_file(path)["keys"]) == [1]
    k = np.array([9, 2, 5], np.int64)
    p.gpu.lookup_pooled(p.batch, torch.from_numpy(k).to(DEV), torch.tensor([0, 3], device=DEV), 1, 1,
                        R.SUM, torch.empty((1, 1, 16), dtype=torch.float32, device=DEV))
    r = p.ora.lookup(k, np.array([0, 3], np.int64), 1, 1)
    uq, inv, rows, n_new = p.batch.get_unique(3)
    assert list(rows.cpu().numpy()) == list(r.rows) == [1, 2, 3]
    compare_tables(p, "after reuse")
    p.close()
