"""Helpers of the sharded-table tests: a CPU engine built from numpy and the
oracle (so gloo ranks can run the sharded protocol without a GPU), an
in-process exchange for virtual ranks on one GPU, the workload of a step, and
the unsharded reference (one oracle table fed every rank's batch as one)."""
import threading

import numpy as np
import torch

import oracle as O
import workloads as W

D = 16
SALT = 0x9E3779B97F4A7C15


def owner(keys, world, salt=SALT):
    """H(key ^ salt) mod world, with the oracle's hash."""
    return np.array([O.hash64((int(k) ^ salt) & (2**64 - 1)) % world for k in keys], np.int64)


class OracleEngine:
    """The engine steps on CPU tensors: numpy for the requester, an oracle
    table for this rank's shard."""

    def __init__(self, optimizer=O.ADAM, lr=0.01, init_seed=5):
        self.table = O.Table(D, optimizer, lr, init_seed=init_seed)
        self.dim = D

    def dedup(self, keys):
        u, inv = np.unique(keys.numpy(), return_inverse=True)
        self._inv = inv
        return torch.from_numpy(u), torch.from_numpy(inv.astype(np.int32))

    def partition(self, uniq, world, salt):
        u = uniq.numpy()
        o = owner(u, world, salt) if len(u) else np.zeros(0, np.int64)
        order = np.argsort(o, kind="stable")
        pos = np.empty(len(u), np.int32)
        pos[order] = np.arange(len(u), dtype=np.int32)
        counts = [int((o == r).sum()) for r in range(world)]
        return torch.from_numpy(u[order].copy()), torch.from_numpy(pos), counts

    def serve_lookup(self, keys):
        k = keys.numpy()
        r = self.table.lookup(k, np.arange(len(k) + 1, dtype=np.int64), 1, len(k), pooled=False,
                              unpooled=True)
        return torch.from_numpy(r.unpooled)

    def pool(self, rows, pos, inv, bag_offsets, F, B, combiner):
        rows, pos, inv, bo = rows.numpy(), pos.numpy(), inv.numpy(), bag_offsets.numpy()
        out = np.zeros((B, F, D), np.float32)
        for j in range(F * B):
            lo, hi = bo[j], bo[j + 1]
            acc = rows[pos[inv[lo:hi]]].astype(np.float64).sum(axis=0) if hi > lo else np.zeros(D)
            if combiner == O.MEAN and hi > lo:
                acc = acc / (hi - lo)
            out[j % B, j // B] = acc.astype(np.float32)
        return torch.from_numpy(out)

    def reduce(self, n_unique, pos, bag_offsets, F, B, combiner, grad_pooled, grad_unpooled):
        bo = bag_offsets.numpy()
        g = np.zeros((n_unique, D), np.float64)
        for j in range(F * B):
            lo, hi = bo[j], bo[j + 1]
            for i in range(lo, hi):
                t = grad_pooled.numpy()[j % B, j // B].astype(np.float64)
                if combiner == O.MEAN:
                    t = t / (hi - lo)
                g[self._inv[i]] += t
        out = np.zeros((n_unique, D), np.float32)
        out[pos.numpy()] = g.astype(np.float32)
        return torch.from_numpy(out)

    def serve_backward(self, grads):
        self.table.backward_update(None, grads.numpy())


class ThreadExchange:
    """All-to-all between virtual ranks that are threads of one process."""

    def __init__(self, shared, rank, world):
        self.s, self.rank, self.world = shared, rank, world

    def counts(self, send_counts, device):
        self.s["c"][self.rank] = list(send_counts)
        self.s["bar"].wait()
        r = [self.s["c"][o][self.rank] for o in range(self.world)]
        self.s["bar"].wait()
        return r

    def tensors(self, send, send_counts, recv_counts):
        offs = np.concatenate([[0], np.cumsum(send_counts)])
        self.s["t"][self.rank] = (send, offs)
        self.s["bar"].wait()
        parts = [self.s["t"][o][0][self.s["t"][o][1][self.rank]:self.s["t"][o][1][self.rank + 1]]
                 for o in range(self.world)]
        out = torch.cat(parts) if parts else send[:0]
        self.s["bar"].wait()
        return out


def shared_state(world):
    # a timeout turns a rank that failed into an error in the others, not a hang
    return {"c": [None] * world, "t": [None] * world, "bar": threading.Barrier(world, timeout=300)}


def batch(rank, step, B=48, n_ids=300):
    """One rank's batch of a step: B bags of length 1..6, Zipf keys (shared
    hot keys across ranks), and its pooled gradient."""
    rng = np.random.default_rng([rank, step, 11])
    lengths = rng.integers(1, 7, size=B)
    bo = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    keys = (W.Zipf(n_ids, 1.1).sample(rng, int(bo[-1])) * 7919 - 50_000).astype(np.int64)
    g = W.make_grad((B, 1, D), 1000 * step + rank, signed=True)
    return keys, bo, g


def bags_of(rank, empty_rank=-1):
    """Bags of a rank's batch: none for the rank that sends nothing."""
    return 0 if rank == empty_rank else 48


def reference(world, steps, combiner=O.SUM, optimizer=O.ADAM, empty_rank=-1):
    """The unsharded table: every step, all ranks' bags as one batch."""
    t = O.Table(D, optimizer, 0.01, init_seed=5)
    pooled = []
    for step in range(steps):
        ks, bos, gs = [], [np.zeros(1, np.int64)], []
        for r in range(world):
            k, bo, g = batch(r, step, B=bags_of(r, empty_rank))
            bos.append(bo[1:] + sum(len(x) for x in ks))
            ks.append(k)
            gs.append(g)
        keys, bo, g = np.concatenate(ks), np.concatenate(bos), np.concatenate(gs)
        res = t.lookup(keys, bo, 1, len(bo) - 1, combiner)
        splits = np.cumsum([0] + [len(x) for x in gs])
        pooled.append([res.pooled[splits[r]:splits[r + 1]] for r in range(world)])
        t.backward_update(g)
    return t, pooled
