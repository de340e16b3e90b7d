"""The sharded-table protocol (dedup, partition by owner, all-to-all of keys,
rows and gradients) on gloo ranks on CPU (two ranks; three with one rank
that has no bags but still owns a shard and serves the others), each rank's
arithmetic done by the numpy/oracle engine, against one unsharded oracle
table fed all ranks' bags as one batch: pooled rows every step and the final
state of every key (the union of the shards) within the usual tolerance."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STEPS = 3


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, out_dir, combiner, empty_rank):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import shard_util as S
    from recommender_sparse_embedding_b200.sharded import ShardedTable

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        st = ShardedTable(S.D, 1, 0.01, engine=S.OracleEngine(), salt=S.SALT)
        pooled = []
        for step in range(STEPS):
            k, bo, g = S.batch(rank, step, B=S.bags_of(rank, empty_rank))
            out = st.lookup_pooled(torch.from_numpy(k), torch.from_numpy(bo), 1, len(bo) - 1, combiner)
            pooled.append(out.numpy())
            st.backward_update(torch.from_numpy(g))
        keys, emb, state = st.engine.table.export()
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), keys=keys, emb=emb, state=state,
                 step=st.engine.table.step, **{f"p{i}": p for i, p in enumerate(pooled)})
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,combiner,empty_rank", [(2, 0, -1), (2, 1, -1), (3, 0, 1)],
                         ids=["2 ranks sum", "2 ranks mean", "3 ranks, rank 1 without bags"])
def test_gloo_ranks_match_the_unsharded_table(tmp_path, world, combiner, empty_rank):
    import shard_util as S
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path), combiner, empty_rank),
                       nprocs=world, start_method="spawn")
    ref, ref_pooled = S.reference(world, STEPS, combiner=combiner, empty_rank=empty_rank)
    rk, re, rs = ref.export()
    where = {int(k): i for i, k in enumerate(rk)}
    seen = 0
    for r in range(world):
        d = np.load(tmp_path / f"r{r}.npz")
        for i in range(STEPS):
            np.testing.assert_allclose(d[f"p{i}"], ref_pooled[i][r], rtol=1e-5, atol=1e-6)
        assert all(S.owner([k], world)[0] == r for k in d["keys"])  # each key on its owner
        idx = np.array([where[int(k)] for k in d["keys"]])
        np.testing.assert_allclose(d["emb"], re[idx], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(d["state"], rs[idx], rtol=1e-5, atol=1e-6)
        assert int(d["step"]) == ref.step
        seen += len(d["keys"])
    assert seen == len(rk)  # the shards hold every key exactly once
