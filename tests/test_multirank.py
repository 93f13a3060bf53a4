"""The N > 1 path on CPU with gloo, world size 2: each rank derives its own
seeded batch (weak scaling, no exchange on the data path) and the step time
is the max over ranks.  The sharded results gathered from both ranks equal
what one process computes for the same per-rank workloads."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs, rank_workload
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    w = rank_workload(WORKLOADS["tiny"].with_(seqlen=24), rank)
    out = oracle.oracle_fwd(**make_inputs(w), nthreads=1)
    y = torch.from_numpy(out["Y"])
    gathered = [torch.empty_like(y) for _ in range(WORLD)]
    dist.all_gather(gathered, y)
    t = torch.tensor([1.0 + rank])  # a stand-in for each rank's measured step time
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    if rank == 0:
        np.save(os.path.join(out_dir, "gathered.npy"), torch.stack(gathered).numpy())
        np.save(os.path.join(out_dir, "tmax.npy"), t.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_weak_scaling_shards(tmp_path):
    import oracle
    from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs, rank_workload
    mp.start_processes(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD,
                       start_method="spawn", join=True)
    gathered = np.load(tmp_path / "gathered.npy")
    for r in range(WORLD):
        w = rank_workload(WORKLOADS["tiny"].with_(seqlen=24), r)
        np.testing.assert_array_equal(gathered[r], oracle.oracle_fwd(**make_inputs(w), nthreads=1)["Y"])
    assert not np.array_equal(gathered[0], gathered[1])  # ranks really hold different batches
    assert float(np.load(tmp_path / "tmax.npy")[0]) == 2.0
