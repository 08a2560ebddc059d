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


def _run_bench(args, env_extra=None):
    import json
    import subprocess
    import sys
    env = dict(os.environ)
    env.update(env_extra or {})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py")] + args, cwd=root,
                         env=env, capture_output=True, text=True, timeout=600)
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    return out.returncode, [json.loads(l) for l in lines]


def test_reference_arm_prints_one_line_on_rank_0_only():
    """The reference arm (the oracle on the host cores) prints the bench contract's line on
    rank 0 and nothing on the other ranks."""
    args = ["--impl", "reference", "--workload", "tiny_fp32", "--steps", "1", "--warmup", "3"]
    rc, lines = _run_bench(args)
    assert rc == 0 and len(lines) == 1
    line = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"] == "tiny_fp32"
    rc, lines = _run_bench(args, {"RANK": "1", "WORLD_SIZE": "2"})
    assert rc == 0 and lines == []
