"""SafeTensors saver and loader of a table (the Saver of the RecIS README:
sparse parameters stored and delivered in the SafeTensors standard format).

The file the library writes is read back by the safetensors package (the
format's reference implementation) and compared with the table's export;
a saved table loads into a fresh one unchanged; a file the safetensors package
writes from the oracle's table loads into the library, and one more training
step on both sides keeps them at parity.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity_util import Pair, compare_tables, run_workload

safetensors_numpy = pytest.importorskip("safetensors.numpy")
from safetensors import safe_open  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    import recommender_sparse_embedding_b200 as R
    from recommender_sparse_embedding_b200 import build
    build.build()
    assert torch.cuda.is_available()
    R.load()
    return R


def _state_names(spec):
    return ["accum"] if spec.optimizer == "adagrad" else ["adam_m", "adam_v"]


@pytest.mark.parametrize("name,B", [("tiny", 256), ("criteo26", 512), ("seq8", 64)])
def test_save_reads_back_and_loads(R, tmp_path, name, B):
    w = W.WORKLOADS[name].scaled(B)
    pairs = run_workload(R, w, steps=2, return_pairs=True)
    for p in pairs:
        spec = p.spec
        path = str(tmp_path / f"{spec.name}.safetensors")
        p.gpu.save(path)
        keys, emb, state, step = p.gpu.export()
        D = spec.dim
        got = safetensors_numpy.load_file(path)
        assert np.array_equal(got["keys"], keys)
        assert np.array_equal(got["emb"], emb)
        for k, nm in enumerate(_state_names(spec)):
            assert np.array_equal(got[nm], state[:, k * D:(k + 1) * D])
        with safe_open(path, framework="numpy") as f:
            md = f.metadata()
        assert md["format"] == "recis-embedding-table"
        assert int(md["dim"]) == D and int(md["step"]) == step and int(md["rows"]) == len(keys)
        assert md["optimizer"] == spec.optimizer
        # a fresh table of the same attributes gets the same rows and step
        t2 = R.Table(D, R.ADAM if spec.optimizer == "adam" else R.ADAGRAD, spec.lr,
                     init_seed=spec.init_seed)
        t2.load_file(path)
        k2, e2, s2, st2 = t2.export()
        assert np.array_equal(k2, keys) and np.array_equal(e2, emb) and np.array_equal(s2, state)
        assert st2 == step
        t2.close()
        p.close()


def test_file_from_the_reference_writer_loads_and_trains_on(R, tmp_path):
    w = W.WORKLOADS["criteo26"].scaled(256)
    spec = w.tables[0]
    D = spec.dim
    # an oracle table after two steps, written by the safetensors package
    ora = O.Table(D, O.ADAM, spec.lr, init_seed=spec.init_seed)
    ops = [O.FeatureOp(flags=f.flags, hash_seed=f.hash_seed, mod=f.mod, tag=f.tag,
                       tag_shift=f.tag_shift) for f in w.features]
    for step in range(2):
        bt = W.make_batch(w, step)
        keys = O.feature_hash(ops, bt.values, bt.feat_offsets)
        ora.lookup(keys, bt.bag_offsets, w.F, w.B)
        ora.backward_update(W.make_grad((w.B, w.F, D), 50 + step))
    k, e, s = ora.export()
    path = str(tmp_path / "oracle.safetensors")
    safetensors_numpy.save_file({"keys": k, "emb": e, "adam_m": np.ascontiguousarray(s[:, :D]),
                                 "adam_v": np.ascontiguousarray(s[:, D:])}, path,
                                metadata={"step": str(ora.step)})
    p = Pair(R, spec)
    p.gpu.load_file(path)
    p.ora = ora
    compare_tables(p, "after loading the oracle's file")
    # one more step on both sides
    run_workload(R, w, steps=1, batch_seed=99, pairs=[p])


def test_load_rejects_a_file_of_another_dim(R, tmp_path):
    path = str(tmp_path / "d8.safetensors")
    safetensors_numpy.save_file({"keys": np.arange(3, dtype=np.int64),
                                 "emb": np.zeros((3, 8), np.float32),
                                 "accum": np.zeros((3, 8), np.float32)}, path)
    t = R.Table(16, R.ADAGRAD, 0.1)
    with pytest.raises(R.RecisError) as e:
        t.load_file(path)
    assert e.value.code == R.recis.ERR_INVALID_ARG
    assert t.size()[0] == 0
    t8 = R.Table(8, R.ADAGRAD, 0.1)
    t8.load_file(path)
    assert t8.size()[0] == 3
    t.close()
    t8.close()
