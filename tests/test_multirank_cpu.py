"""The multi-rank host logic of the benchmark, on CPU with gloo (world size 2).

The layer does not shard across GPUs (independent replicas, no data-path
collective): every rank runs its own batch, and the timing is the maximum over
ranks.  These tests run that logic with two gloo ranks on the host."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    from expert_warp_top_b200 import inputs
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = inputs.CONFIGS["tiny"]
        # each rank times its own steps; the job time is the slowest rank's
        my_ms = 10.0 + 5.0 * rank
        m = bench.max_over_ranks(my_ms, "cpu")
        # independent batches: different seeds give different logits
        lg = inputs.make_logits(cfg, seed=bench.rank_seed(cfg, rank))
        gathered = [torch.empty_like(lg) for _ in range(world)]
        dist.all_gather(gathered, lg)
        out[rank] = (m, bench.whole_job_tokens_per_s(cfg.T, 4, world, m),
                     not torch.equal(gathered[0], gathered[1]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_time_and_batches():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as mgr:  # no fork of this threaded process
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        m, thr, distinct = res[rank]
        assert m == 15.0                      # max over ranks
        assert thr == pytest.approx(2 * 256 * 4 / 15e-3)  # whole-job tokens / slowest rank
        assert distinct                       # each rank has its own batch


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "1", "--warmup", "3", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_max_over_ranks_without_a_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
