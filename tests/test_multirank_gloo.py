"""Multi-rank host logic on CPU with the gloo backend (world size 2): the data-parallel
sharding, the max-over-ranks timing used by bench.py, and the property that makes the
path shard with no collective -- per-rank runs over disjoint sequences reproduce the
single-process result exactly (checked with the oracle, which runs on the CPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_160_b200.sharding import pack, shard_sequences


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, lengths, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from gated_delta_rule_160_b200 import workloads as W
        # max over ranks, as bench.py reports time
        assert bench.max_over_ranks(float(rank + 1), world) == float(world)
        bench.barrier(world)
        # each rank runs the oracle on its shard of a packed batch
        T = int(sum(lengths))
        d = W.token_inputs(T, 2, 2, 16, 8, torch.float32, "cpu", seed=31)
        mine = shard_sequences(lengths, world, rank)
        ranges, cu = pack(lengths, mine)
        idx = np.concatenate([np.arange(a, z) for a, z in ranges]) if ranges else np.zeros(0, np.int64)
        sub = {k: d[k][idx].contiguous() for k in d}
        if mine:
            o, st = oracle.fwd_ref(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["b"], sub["w"],
                                   cu_seqlens=np.asarray(cu, np.int32))
        else:
            o, st = np.zeros((0, 2, 8)), np.zeros((0, 2, 16, 8))
        gathered = [None] * world
        dist.all_gather_object(gathered, (mine, idx.tolist(), o, st))
        if rank == 0:
            np.save(os.path.join(result_dir, "gathered.npy"), np.array(gathered, dtype=object), allow_pickle=True)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_shard_sequences_partition_and_balance():
    rng = np.random.default_rng(4)
    lengths = rng.integers(128, 8193, size=64).tolist()
    for world in (1, 2, 3, 8):
        shards = [shard_sequences(lengths, world, r) for r in range(world)]
        allidx = sorted(i for s in shards for i in s)
        assert allidx == list(range(64))
        loads = [sum(lengths[i] for i in s) for s in shards]
        assert max(loads) - min(loads) <= max(lengths)
    with pytest.raises(ValueError):
        shard_sequences(lengths, 2, 2)


def test_two_gloo_ranks_reproduce_single_process(tmp_path, oracle_mod):
    lengths = [5, 0, 17, 1, 9, 12, 3]
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), lengths, str(tmp_path)), nprocs=world, join=True)
    gathered = np.load(tmp_path / "gathered.npy", allow_pickle=True)
    from gated_delta_rule_160_b200 import workloads as W
    T = int(sum(lengths))
    d = W.token_inputs(T, 2, 2, 16, 8, torch.float32, "cpu", seed=31)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    o_full, st_full = oracle_mod.fwd_ref(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], cu_seqlens=cu)
    seen = []
    for mine, idx, o, st in gathered:
        seen += list(mine)
        if mine:
            np.testing.assert_array_equal(o, o_full[np.asarray(idx)])
            np.testing.assert_array_equal(st, st_full[np.asarray(mine)])
    assert sorted(seen) == list(range(len(lengths)))
