"""CPU checks of the boundary: the library builds, loads and exports every entry
point that include/recis.h declares (no compute call needs a GPU here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "recis.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(recis_[a-z_]+)\s*\(", src)))


def test_header_declares_the_five_core_calls():
    d = _declared()
    for name in ("recis_table_create", "recis_feature_hash", "recis_lookup_pooled",
                 "recis_backward_update", "recis_table_export"):
        assert name in d


def test_library_loads_and_exports_every_declared_symbol():
    from recommender_sparse_embedding_b200 import build
    path = build.build()
    lib = ctypes.CDLL(path)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_the_header():
    import recommender_sparse_embedding_b200.recis as R
    assert sorted(R.EXPORTS) == _declared()
    R.load()


def test_binding_fails_loudly_without_library(tmp_path):
    import recommender_sparse_embedding_b200.recis as R
    with pytest.raises(RuntimeError):
        _load_fresh(R, str(tmp_path / "nope.so"))


def _load_fresh(R, path):
    saved = R._lib
    R._lib = None
    try:
        return R.load(path)
    finally:
        R._lib = saved


def test_oracle_and_library_share_no_code():
    # the oracle is test infrastructure: nothing under the package mentions it
    pkg = os.path.join(ROOT, "recommender_sparse_embedding_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "oracle.h" not in txt, f
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".cpp", ".h", ".py")):
            txt = open(os.path.join(ROOT, "oracle", f)).read()
            assert "recommender_sparse_embedding_b200" not in txt and "recis.h" not in txt, f
