"""The multi-rank host logic of bench.py on CPU: world_size 2 over gloo.

Under weak scaling each rank runs its own independent batch, there is no
collective on the data path, and the reported time is the slowest rank's.  These
tests check that logic without a GPU: the max-over-ranks reduction, the
whole-job aggregate, that ranks draw different batches of the same shape, and
that the reference arm under torchrun prints one line from rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port):
    sys.path.insert(0, ROOT)
    import bench
    from nvfp4_block_scaled_17_b200 import workloads as W
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # the slowest rank's time wins on every rank
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, True)
        assert ms == 10.0 + 5.0 * (world - 1)
        # weak scaling: world x per-rank work in the slowest rank's time
        assert bench.aggregate_tflops(1e12, ms, world) == pytest.approx(world * 1e12 / (ms * 1e-3) / 1e12)
        # independent batches of one shape per rank
        lins = W.vit_block("cpu", seed=bench.rank_seed(rank), tokens=8)
        head = lins[0].x[:2, :8].float().flatten().tolist()
        shapes = [tuple(l.x.shape) for l in lins]
        got = [None] * world
        dist.all_gather_object(got, (head, shapes))
        assert all(g[1] == shapes for g in got)
        assert len({tuple(g[0]) for g in got}) == world
        # the reference arm runs on rank 0 only
        if rank != 0:
            assert bench.run_reference(None, rank, world) is None
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    mp.start_processes(_rank_main, args=(2, free_port()), nprocs=2, join=True,
                       start_method="spawn")


def test_reference_arm_under_torchrun_prints_once():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 2
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "vit_decoder_block_8tiles"
