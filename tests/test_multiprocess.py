"""The multi-GPU path on CPU: world-size-2 `gloo` process groups.

bench.py runs one process per GPU. With --scaling strong each rank takes a whole number of
GQA groups (its KV heads and their query heads) and computes its slice of the output with
no data exchange; the timing is the maximum over ranks. Here two CPU ranks each compute
their head shard with the float64 oracle, gather the slices and compare the assembled
output with the oracle on the whole problem; the max-over-ranks reduction is checked too.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads
from oracle import diffattn_f64 as ora


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_file):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = workloads.PrefillCase(B=2, S=37, Hq=16, Hkv=4, D=16, dtype="f32", seed=3)
        full = workloads.make_prefill(case)
        shard = bench.shard_prefill_inputs(full, case.Hq, case.Hkv, world, rank)
        part = torch.from_numpy(ora.prefill(shard["q"], shard["k"], shard["v"], shard["lam"]))
        parts = [torch.zeros_like(part) for _ in range(world)]
        dist.all_gather(parts, part)
        # decode step, same sharding of a cache
        dcase = workloads.DecodeCase(B=3, Smax=29, Hq=16, Hkv=4, D=16, len_lo=1, len_hi=29, dtype="f32", seed=4)
        dfull = workloads.make_decode(dcase)
        kv0, kv1, q0, q1 = bench.head_shard(dcase.Hq, dcase.Hkv, world, rank)
        dpart = torch.from_numpy(ora.decode(dfull["q"][:, q0:q1], dfull["kcache"][:, :, kv0:kv1],
                                             dfull["vcache"][:, :, kv0:kv1], dfull["seqlens"],
                                             dfull["lam"][:, q0 // 2:q1 // 2]))
        dparts = [torch.zeros_like(dpart) for _ in range(world)]
        dist.all_gather(dparts, dpart)
        tmax = bench._max_over_ranks(float(rank + 1) * 1.5, dist)
        if rank == 0:
            out = torch.cat(parts, dim=2).numpy()
            ref = ora.prefill(full["q"], full["k"], full["v"], full["lam"])
            dout = torch.cat(dparts, dim=1).numpy()
            dref = ora.decode(dfull["q"], dfull["kcache"], dfull["vcache"], dfull["seqlens"], dfull["lam"])
            np.savez(result_file, err=np.abs(out - ref).max(), derr=np.abs(dout - dref).max(), tmax=tmax)
    finally:
        dist.destroy_process_group()


def test_head_sharded_ranks_assemble_the_full_output(tmp_path):
    world = 2
    result = str(tmp_path / "res.npz")
    mp.spawn(_worker, args=(world, _free_port(), result), nprocs=world, join=True)
    r = np.load(result)
    assert r["err"] < 1e-12 and r["derr"] < 1e-12
    assert r["tmax"] == 3.0


@pytest.mark.parametrize("Hq,Hkv,world", [(64, 8, 2), (64, 8, 4), (64, 8, 8), (16, 2, 2), (32, 4, 4)])
def test_head_shard_partitions_groups(Hq, Hkv, world):
    kv_seen, q_seen = [], []
    for rank in range(world):
        kv0, kv1, q0, q1 = bench.head_shard(Hq, Hkv, world, rank)
        kv_seen += list(range(kv0, kv1))
        q_seen += list(range(q0, q1))
        G = Hq // Hkv
        for h in range(q0, q1):  # every query head's KV head is local to the rank
            assert kv0 <= h // G < kv1
        assert (q1 - q0) % 2 == 0  # whole pairs
    assert kv_seen == list(range(Hkv)) and q_seen == list(range(Hq))


def test_head_shard_rejects_uneven_split():
    with pytest.raises(ValueError):
        bench.head_shard(64, 8, 3, 0)
