"""B200 (sm_100a) dynamic-hash sparse embedding engine.

The hot path (feature hash/mod/bucketize/tag, dedup, IDMap find-or-insert,
gather + bag pooling, per-unique gradient reduction fused with the Adagrad or
Adam row update) runs in librecis.so, built from csrc/ by build.build().  This
package is its thin ctypes binding (recis.py); PyTorch provides device memory
and streams only.
"""
from .recis import (ADAGRAD, ADAM, BUCKETIZE, ERR_INVALID_ARG, FLOAT, HASH, MEAN, MOD, OK, SUM, TAG,  # noqa: F401
                    Batch, Feature, RecisError, Table, feature_hash, feature_status_sync, launch_count,
                    load, profile_collect, profile_enable)
