"""The N > 1 benchmark path on CPU: two gloo ranks, each encoding its own
block (no data exchange), timing reduced with max over ranks, whole-job rate
= every rank's bytes over the slowest rank's time."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import huffman_decode_02_b200 as df11
        import oracle
        import workloads
        w = workloads.normal_matrix(96, 80, 0.02, seed=bench.rank_seed(rank))
        t = df11.encode(w)
        # each rank's stream decodes back to its own weights (oracle, host)
        back = oracle.decode(t.host_array("enc"), t.total_bits, t.host_array("sm"), t.n_elems, t.code_len)
        assert np.array_equal(back, w.reshape(-1))
        fake_ms = 10.0 + 5.0 * rank
        slowest = bench.max_over_ranks(fake_ms, dist, torch.device("cpu"))
        rate = bench.aggregate_rate(2.0 * t.n_elems, world, slowest * 1e-3)
        digest = torch.tensor([float(w.astype(np.int64).sum())])
        gathered = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(gathered, digest)
        out[rank] = (slowest, rate, [float(g.item()) for g in gathered], t.n_elems)
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_host_logic():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0  # max over ranks
    n = res[0][3]
    assert res[0][1] == pytest.approx(2.0 * n * world / 15e-3 / 1e9)
    sums = res[0][2]
    assert sums[0] != sums[1]  # each rank decodes its own block
