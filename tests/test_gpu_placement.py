"""Placement of a table's memory (RecIS README, Efficient dynamic embedding:
the IDMap and the EmbeddingBlocks can live in GPU or in CPU memory): the same
workloads at parity with the oracle with the EmbeddingBlocks in host memory,
the IDMap in host memory, or both.  A placement the system cannot provide is
refused at create with RECIS_ERR_INVALID_ARG and a reason; the test then
checks that refusal and skips the parity part.
"""
import pytest
import torch

import workloads as W
from parity_util import Pair, run_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    import recommender_sparse_embedding_b200 as R
    from recommender_sparse_embedding_b200 import build
    build.build()
    assert torch.cuda.is_available()
    R.load()
    return R


@pytest.mark.parametrize("placement", [1, 2, 3])
@pytest.mark.parametrize("name,B", [("tiny", 256), ("criteo26", 512), ("seq8", 48)])
def test_placement_parity(R, placement, name, B):
    w = W.WORKLOADS[name].scaled(B)
    try:
        pairs = [Pair(R, t, placement=placement, block_rows=1024) for t in w.tables]
    except R.RecisError as e:
        assert e.code == R.recis.ERR_INVALID_ARG and "host" in str(e)
        pytest.skip(f"placement {placement} not provided here: {e}")
    # growth of host-placed blocks and of a host IDMap happens on the way
    run_workload(R, w, steps=3, pairs=pairs, grad_signed=True)
