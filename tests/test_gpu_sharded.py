"""Sharded tables on the GPU (the README's distributed optimisation: keys split
over nodes, requests deduplicated, rows fetched by All-to-All): the CUDA
engine's dedup, owner partition, pooling from received rows, per-key gradient
reduction and the owners' lookups and updates, against one unsharded oracle
table fed every rank's bags as one batch.

- Four ranks emulated as threads of one process on one GPU, exchanging
  through shared memory of the process (the machines of this build offer one
  GPU per run, so real multi-GPU all-to-alls cannot be run here).
- One real rank in an NCCL process group: the same step through
  torch.distributed's all-to-all.
"""
import os
import socket
import threading

import numpy as np
import pytest
import torch

import oracle as O
import shard_util as S

pytestmark = pytest.mark.gpu
STEPS = 3


@pytest.fixture(scope="module")
def R():
    import recommender_sparse_embedding_b200 as R
    from recommender_sparse_embedding_b200 import build
    build.build()
    assert torch.cuda.is_available()
    R.load()
    return R


def _check(R, world, results, combiner):
    ref, ref_pooled = S.reference(world, STEPS, combiner=combiner)
    rk, re, rs = ref.export()
    where = {int(k): i for i, k in enumerate(rk)}
    seen = 0
    for r in range(world):
        pooled, keys, emb, state, step = results[r]
        for i in range(STEPS):
            np.testing.assert_allclose(pooled[i], ref_pooled[i][r], rtol=1e-5, atol=1e-6)
        assert all(S.owner([k], world)[0] == r for k in keys)
        idx = np.array([where[int(k)] for k in keys], np.int64)
        np.testing.assert_allclose(emb, re[idx], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(state, rs[idx], rtol=1e-5, atol=1e-6)
        assert step == ref.step
        seen += len(keys)
    assert seen == len(rk)


def _run_rank(R, st, rank, combiner, dev):
    pooled = []
    for step in range(STEPS):
        k, bo, g = S.batch(rank, step)
        out = st.lookup_pooled(torch.from_numpy(k).to(dev), torch.from_numpy(bo).to(dev), 1, len(bo) - 1,
                               combiner)
        pooled.append(out.cpu().numpy())
        st.backward_update(torch.from_numpy(g).to(dev))
    keys, emb, state, step = st.engine.table.export()
    return pooled, keys, emb, state, step


@pytest.mark.parametrize("combiner", [0, 1])
def test_four_emulated_ranks_match_the_unsharded_table(R, combiner):
    from recommender_sparse_embedding_b200.sharded import CudaEngine, ShardedTable
    world = 4
    dev = torch.device("cuda", 0)
    shared = S.shared_state(world)
    tables = [ShardedTable(S.D, R.ADAM, 0.01, engine=CudaEngine(S.D, R.ADAM, 0.01, init_seed=5),
                           exchange=S.ThreadExchange(shared, r, world), salt=S.SALT) for r in range(world)]
    results, errors = [None] * world, []

    def body(r):
        try:
            torch.cuda.set_device(0)
            results[r] = _run_rank(R, tables[r], r, combiner, dev)
        except BaseException as e:  # noqa: BLE001 -- reported below
            errors.append(e)
            shared["bar"].abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    for t in tables:
        t.close()
    assert not errors, errors
    _check(R, world, results, combiner)


def test_one_nccl_rank(R):
    import torch.distributed as dist
    from datetime import timedelta

    from recommender_sparse_embedding_b200.sharded import ShardedTable
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=timedelta(seconds=120))
    try:
        st = ShardedTable(S.D, R.ADAM, 0.01, init_seed=5, salt=S.SALT)
        res = _run_rank(R, st, 0, 0, torch.device("cuda", 0))
        st.close()
    finally:
        dist.destroy_process_group()
    _check(R, 1, [res], 0)
