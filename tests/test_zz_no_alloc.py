"""The allocation-free dedup entry point (recis_unique_static).

It serves callers that cannot allocate device memory (a framework memory pool
that forbids foreign cudaMalloc calls, graph recording with allocation
disabled, fixed device-memory budgets).  Its output must equal
numpy.unique(return_inverse=True) of the keys and the dedup of the regular
path (recis_lookup_pooled + recis_batch_get_unique) on the same keys, bit for
bit, on consecutive calls that share its static scratch.  This file
sorts last so that a run stopping at the first failure has run every other
test first.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _regular_dedup(R, keys):
    t = R.Table(4, R.ADAGRAD, 0.1)
    b = R.Batch()
    n = keys.numel()
    bo = torch.tensor([0, n], dtype=torch.int64, device=keys.device)
    out = torch.empty((1, 1, 4), dtype=torch.float32, device=keys.device)
    t.lookup_pooled(b, keys, bo, 1, 1, R.SUM, out)
    uq, inv, _, _ = b.get_unique(n)
    res = uq.cpu().numpy(), inv.cpu().numpy()
    t.close()
    b.close()
    return res


def test_unique_static_matches_regular_dedup_on_two_calls():
    import recommender_sparse_embedding_b200 as R
    from recommender_sparse_embedding_b200 import build
    build.build()
    L = R.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    rng = np.random.default_rng(31)
    cases = [
        rng.integers(-(2**62), 2**62, size=200_000, dtype=np.int64) % 150_000,  # heavy repeats
        (rng.integers(0, 2**40, size=262_144, dtype=np.int64) | (7 << 40)),      # the maximum N
    ]
    free_after_first = None
    for call, keys_np in enumerate(cases):
        keys = torch.from_numpy(keys_np).to(dev)
        n = keys.numel()
        uniq = torch.empty(n, dtype=torch.int64, device=dev)
        inv = torch.empty(n, dtype=torch.int32, device=dev)
        U = torch.empty(1, dtype=torch.int64, device=dev)
        torch.cuda.synchronize()
        if call == 1:
            free_after_first = torch.cuda.mem_get_info()[0]
        rc = L.recis_unique_static(keys.data_ptr(), n, uniq.data_ptr(), inv.data_ptr(),
                                   U.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert rc == 0, L.recis_last_error_string()
        torch.cuda.synchronize()
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free_after_first  # nothing allocated
        u = int(U.item())
        ref_uniq, ref_inv = _regular_dedup(R, keys)
        assert u == len(ref_uniq)
        assert np.array_equal(uniq[:u].cpu().numpy(), ref_uniq)
        assert np.array_equal(inv.cpu().numpy(), ref_inv)
        # and directly against the definition (numpy's unique with inverse)
        np_uniq, np_inv = np.unique(keys_np, return_inverse=True)
        assert np.array_equal(uniq[:u].cpu().numpy(), np_uniq)
        assert np.array_equal(inv.cpu().numpy(), np_inv.reshape(-1))


def test_unique_static_rejects_oversized_input():
    import recommender_sparse_embedding_b200 as R
    L = R.load()
    rc = L.recis_unique_static(None, 262_145, None, None, None, None)
    assert rc == R.recis.ERR_INVALID_ARG
    assert b"262144" in L.recis_last_error_string()
