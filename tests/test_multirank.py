"""The N > 1 bench path on CPU: two gloo ranks, each with its own batch of the workload
(independent problems, no data-path collective), the step time reduced by max over ranks,
and whole-job throughput = every rank's counted FLOPs / the slowest rank's time."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, N, H, d, G = 1, 64, 4, 8, 16
        q, k, v, _ = synth.s2attn_inputs(bench.rank_seed(5, rank), B, N, H, H, d, 0.5, "f32",
                                         with_dout=False)
        o, _ = oracle.fwd(q, k, v, G, 2.0)
        fake_ms = 10.0 * (rank + 1)
        ms = bench.max_over_ranks(fake_ms)
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, torch.tensor([float(np.abs(o).sum())], dtype=torch.float64))
        np.save(os.path.join(out_dir, "rank%d.npy" % rank),
                np.array([ms] + [float(x.item()) for x in sums]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_independent_batches_and_max_time(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r0 = np.load(tmp_path / "rank0.npy")
    r1 = np.load(tmp_path / "rank1.npy")
    assert r0[0] == r1[0] == 20.0           # max over ranks, seen by both
    assert np.array_equal(r0[1:], r1[1:])   # both ranks gathered the same per-rank sums
    assert r0[1] != r0[2]                   # the ranks worked on different batches
    assert bench.aggregate_tflops(1e12, world, 20.0) == 2 * 1e12 / 0.02 / 1e12


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_seed(7, 0) == 7 and bench.rank_seed(7, 3) == 3007
