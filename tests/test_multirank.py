"""The bench's multi-rank plumbing on CPU: two gloo ranks (replicas, weak scaling)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from dit_attention_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        # each rank's own step time; everyone must report the slowest
        mx = bench.max_over_ranks(10.0 + 5.0 * r, w, "cpu")
        tiny = synth.Workload("t", B=1, H=1, D=16, Sq=8, Skv=8, seed=3)
        q, _, _ = bench.replica_inputs(tiny, r)
        gathered = [torch.zeros(8 * 16, dtype=torch.int32) for _ in range(w)]
        dist.all_gather(gathered, torch.from_numpy(q.reshape(-1).astype(np.int32)))
        ref_line = bench.run_reference(type("A", (), {"warmup": 0, "steps": 0, "cpu_seconds": 0.1})(), r, w) \
            if r != 0 else "rank0"
        out[r] = (r, w, lr, mx, [g.numpy().tolist() for g in gathered], ref_line)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in (0, 1):
        rank, w, lr, mx, gathered, ref_line = res[r]
        assert (rank, w, lr) == (r, 2, r)
        assert mx == 15.0                                  # max over ranks
        assert gathered[0] != gathered[1]                  # each replica has its own inputs
    assert res[1][5] is None                               # the reference arm runs on rank 0 only
    assert bench.aggregate_tflops(1e12, 2, 1000.0) == pytest.approx(2.0)
