"""Data-parallel sharding of a decode batch, checked with world_size-2 gloo
ranks on the CPU: each rank runs the oracle on its shard; the gathered
results equal the single-process result bit for bit (units are independent)."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_deltanet_recurrent_sigmoid_b200 import sharding, workloads as wl


@pytest.mark.parametrize("N,world", [(10, 3), (3, 4), (512, 2), (0, 2)])
def test_shard_range_partitions(N, world):
    ranges = [sharding.shard_range(N, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == N
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SPEC = wl.shrink(wl.sweep_spec(64), 9, name="shard_case")


def _rank_main(rank, world, port, result_dir):
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.generate(SPEC)
        sh = sharding.shard_workload(w, world, rank)
        sw = sh.workload
        status, out, state, _ = oracle.update(sw.q, sw.k, sw.v, sw.a, sw.b, sw.A_log, sw.dt_bias, sw.state_pool,
                                              sw.state_indices, sw.cu_seqlens)
        assert status == 0
        gathered = [None] * world
        dist.all_gather_object(gathered, (sh.token_rows, out, sh.global_slots, state))
        if rank == 0:
            np.save(os.path.join(result_dir, "gathered.npy"), np.array(gathered, dtype=object), allow_pickle=True)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_shards_reassemble_the_full_result(tmp_path, oracle_lib):
    import oracle
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    gathered = np.load(os.path.join(tmp_path, "gathered.npy"), allow_pickle=True)
    w = wl.generate(SPEC)
    _, out_ref, state_ref, _ = oracle.update(w.q, w.k, w.v, w.a, w.b, w.A_log, w.dt_bias, w.state_pool,
                                             w.state_indices, w.cu_seqlens)
    out = np.full_like(out_ref, np.nan)
    state = w.state_pool.astype(np.float64)
    for rows, o, slots, st in gathered:
        out[rows] = o
        state[slots] = st
    assert np.array_equal(out, out_ref, equal_nan=True)
    assert np.array_equal(state, state_ref)
