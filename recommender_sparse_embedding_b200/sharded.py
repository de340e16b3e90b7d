"""Tables sharded over the ranks of a process group (RecIS README, Key
optimisations > Distributed optimisation: the parameters are split evenly over
the compute nodes; every node merges and deduplicates its requests, sends them
to the nodes that own the IDs and fetches the embeddings back with an
All-to-All collective).

Key k lives on rank owner(k) = H(k ^ salt) mod world (H: the SplitMix64
finaliser).  A step on every rank:

  forward   dedup the batch (unique keys + inverse); group the unique keys by
            owner; all-to-all of the per-owner counts, then of the keys; every
            owner looks its received keys up in its shard (find-or-insert, one
            bag per key); all-to-all of the rows back; pool them into the
            rank's bags.
  backward  the gradient of every unique key summed over the rank's
            occurrences, in the order the keys were sent; all-to-all to the
            owners; every owner applies them with its optimiser as the
            unpooled gradients of its lookup (a key sent by several ranks is
            summed there).

Every rank calls every collective in the same order.  The exchange uses
torch.distributed (NCCL for CUDA tensors, gloo for CPU ones); the arithmetic
runs in an engine: CudaEngine calls the CUDA library on device tensors.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch
import torch.distributed as dist

from . import recis as _r

DEFAULT_SALT = 0x9E3779B97F4A7C15


class Exchange:
    """all-to-all over a torch.distributed process group."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def counts(self, send_counts: Sequence[int], device) -> List[int]:
        """Every rank learns how many items each other rank sends it."""
        s = torch.tensor(list(send_counts), dtype=torch.int64, device=device)
        r = torch.empty_like(s)
        dist.all_to_all_single(r, s, group=self.group)
        return [int(x) for x in r.tolist()]

    def tensors(self, send: torch.Tensor, send_counts: Sequence[int], recv_counts: Sequence[int]) -> torch.Tensor:
        """Rows send[sum(send_counts[:o]) : ...] go to rank o; the result holds
        the rows every rank sent here, rank 0's first."""
        out = torch.empty((sum(recv_counts),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
        dist.all_to_all_single(out, send.contiguous(), output_split_sizes=list(recv_counts),
                               input_split_sizes=list(send_counts), group=self.group)
        return out


class CudaEngine:
    """The steps of the sharded lookup on this rank's GPU (librecis)."""

    def __init__(self, dim: int, optimizer: int, lr: float, **table_kwargs):
        self.dim = dim
        self.table = _r.Table(dim, optimizer, lr, **table_kwargs)  # this rank's shard
        self.req = _r.Batch()  # scratch of the requesting side
        self.own = _r.Batch()  # scratch of the owning side

    def close(self):
        self.table.close()
        self.req.close()
        self.own.close()

    def dedup(self, keys: torch.Tensor):
        n = keys.numel()
        uniq = torch.empty(max(n, 1), dtype=torch.int64, device=keys.device)
        inv = torch.empty(max(n, 1), dtype=torch.int32, device=keys.device)
        U = torch.empty(1, dtype=torch.int64, device=keys.device)
        _r._check(_r.load().recis_batch_dedup(self.req.handle, _r._dev(keys, torch.int64), n, uniq.data_ptr(),
                                              inv.data_ptr(), U.data_ptr(), _r._stream(None)), "recis_batch_dedup")
        u = int(U.item())
        if u < 0:
            raise _r.RecisError(_r.ERR_TIMEOUT, "recis_batch_dedup", "a bounded device-side wait gave up")
        return uniq[:u], inv[:n]

    def partition(self, uniq: torch.Tensor, world: int, salt: int):
        n = uniq.numel()
        out = torch.empty(max(n, 1), dtype=torch.int64, device=uniq.device)
        pos = torch.empty(max(n, 1), dtype=torch.int32, device=uniq.device)
        counts = torch.empty(world, dtype=torch.int64, device=uniq.device)
        _r._check(_r.load().recis_partition_keys(self.req.handle, uniq.data_ptr() if n else None, n, world,
                                                 salt & (2**64 - 1), out.data_ptr(), pos.data_ptr(),
                                                 counts.data_ptr(), _r._stream(None)), "recis_partition_keys")
        return out[:n], pos[:n], [int(x) for x in counts.tolist()]

    def serve_lookup(self, keys: torch.Tensor) -> torch.Tensor:
        n = keys.numel()
        rows = torch.empty((max(n, 1), self.dim), dtype=torch.float32, device=keys.device)
        bo = torch.arange(n + 1, dtype=torch.int64, device=keys.device)
        _r._check(_r.load().recis_lookup_pooled(self.table.handle, self.own.handle,
                                                keys.data_ptr() if n else None, n, bo.data_ptr(), 1 if n else 0,
                                                n, _r.SUM, None, rows.data_ptr(), _r._stream(None)),
                  "recis_lookup_pooled")
        return rows[:n]

    def pool(self, rows, pos, inv, bag_offsets, F, B, combiner):
        out = torch.empty((B, F, self.dim), dtype=torch.float32, device=rows.device)
        _r._check(_r.load().recis_pool_rows(rows.data_ptr(), pos.data_ptr(), inv.data_ptr(),
                                            _r._dev(bag_offsets, torch.int64), F, B, self.dim, combiner,
                                            out.data_ptr(), _r._stream(None)), "recis_pool_rows")
        return out

    def reduce(self, n_unique, pos, bag_offsets, F, B, combiner, grad_pooled, grad_unpooled):
        dev = pos.device
        g = torch.empty((max(n_unique, 1), self.dim), dtype=torch.float32, device=dev)
        _r._check(_r.load().recis_reduce_grad(self.req.handle, _r._dev(bag_offsets, torch.int64), F, B,
                                              self.dim, combiner, _r._dev(grad_pooled, torch.float32),
                                              _r._dev(grad_unpooled, torch.float32), pos.data_ptr(),
                                              g.data_ptr(), _r._stream(None)), "recis_reduce_grad")
        return g[:n_unique]

    def serve_backward(self, grads: torch.Tensor):
        _r._check(_r.load().recis_backward_update(self.table.handle, self.own.handle, None,
                                                  grads.data_ptr() if grads.numel() else None,
                                                  _r._stream(None)), "recis_backward_update")


class ShardedTable:
    """One logical table whose keys are spread over the ranks of `group`.
    `engine` does this rank's arithmetic (a CudaEngine by default) and
    `exchange` its all-to-alls (an Exchange over `group` by default); every
    rank must call lookup_pooled and backward_update the same number of
    times."""

    def __init__(self, dim: int, optimizer: int, lr: float, group=None, salt: int = DEFAULT_SALT,
                 engine=None, exchange=None, **table_kwargs):
        self.x = exchange if exchange is not None else Exchange(group)
        self.salt = salt
        self.dim = dim
        self.engine = engine if engine is not None else CudaEngine(dim, optimizer, lr, **table_kwargs)
        self._ctx = None

    def close(self):
        if hasattr(self.engine, "close"):
            self.engine.close()

    def lookup_pooled(self, keys: torch.Tensor, bag_offsets: torch.Tensor, F: int, B: int,
                      combiner: int = _r.SUM) -> torch.Tensor:
        e, x = self.engine, self.x
        uniq, inv = e.dedup(keys)
        send_keys, pos, send_counts = e.partition(uniq, x.world, self.salt)
        recv_counts = x.counts(send_counts, keys.device)
        recv_keys = x.tensors(send_keys, send_counts, recv_counts)
        rows = e.serve_lookup(recv_keys)
        back = x.tensors(rows, recv_counts, send_counts)  # this rank's unique keys' rows, in send order
        self._ctx = (uniq.numel(), pos, bag_offsets, F, B, combiner, send_counts, recv_counts)
        return e.pool(back, pos, inv, bag_offsets, F, B, combiner)

    def backward_update(self, grad_pooled: Optional[torch.Tensor] = None,
                        grad_unpooled: Optional[torch.Tensor] = None):
        if self._ctx is None:
            raise RuntimeError("backward_update before lookup_pooled")
        U, pos, bag_offsets, F, B, combiner, send_counts, recv_counts = self._ctx
        g = self.engine.reduce(U, pos, bag_offsets, F, B, combiner, grad_pooled, grad_unpooled)
        self.engine.serve_backward(self.x.tensors(g, send_counts, recv_counts))
        self._ctx = None
