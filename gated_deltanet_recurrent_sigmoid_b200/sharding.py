"""Split a decode batch across data-parallel ranks (one process per GPU).

Every (sequence, value head) unit of the fused update is independent, so a
batch shards by sequence with no exchange: each rank owns a contiguous range
of sequences, their activation rows, and the state slots they name (its own
pool).  The pages' deployment shards value heads across TP ranks instead,
again with no communication inside this op.  This module is host-side
bookkeeping only; it holds none of the update's arithmetic.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .workloads import Workload


def shard_range(N: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of the sequences rank `rank` of `world` owns: contiguous,
    sizes differ by at most one, the first N % world ranks take the extra one."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world / rank")
    base, extra = divmod(N, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


@dataclasses.dataclass
class Shard:
    workload: Workload          # the rank's own problem (local pool, local slot ids)
    seqs: np.ndarray            # global sequence ids, in order
    token_rows: np.ndarray      # global token rows of those sequences, in order
    global_slots: np.ndarray    # global slot id of each local pool slot


def shard_workload(w: Workload, world: int, rank: int) -> Shard:
    """The sub-problem of one rank: its sequences, their tokens, and a local
    pool holding exactly the slots they name (padded sequences keep -1)."""
    start, stop = shard_range(w.spec.N, world, rank)
    seqs = np.arange(start, stop)
    lens = w.seq_lens
    starts = np.concatenate([[0], np.cumsum(lens)])
    rows = (np.concatenate([np.arange(starts[i], starts[i] + lens[i]) for i in seqs]).astype(np.int64)
            if len(seqs) else np.zeros(0, np.int64))
    flat = lambda x, tail: np.ascontiguousarray(x.reshape((-1,) + x.shape[-tail:])[rows])
    idx = w.state_indices[seqs]
    live = idx >= 0
    global_slots = idx[live].astype(np.int64)
    local_idx = np.full(len(seqs), -1, dtype=np.int32)
    local_idx[live] = np.arange(live.sum(), dtype=np.int32)
    cu = np.zeros(len(seqs) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens[seqs])
    spec = dataclasses.replace(w.spec, name=f"{w.spec.name}_r{rank}of{world}", N=len(seqs),
                               num_slots=int(live.sum()), T=None, varlen=True)
    sub = Workload(spec, flat(w.q, 2), flat(w.k, 2), flat(w.v, 2), flat(w.a, 1), flat(w.b, 1),
                   w.A_log, w.dt_bias, np.ascontiguousarray(w.state_pool[global_slots]), local_idx, cu)
    return Shard(sub, seqs, rows, global_slots)
