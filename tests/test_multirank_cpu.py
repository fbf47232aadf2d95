"""The multi-rank benchmark path on CPU: two gloo ranks (no GPU).

Each rank runs an independent sequence (its own seed); the only collective is
the max-over-ranks reduction of the step time, and the job rate divides the
units every rank processed by that slowest time.  A rank other than 0 of the
reference arm exits at once without output.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from mamba_ssd_scan_mixer_b200 import workloads as W
        elapsed = 10.0 + 5.0 * rank            # rank 1 is the slow one
        m = bench.max_over_ranks(elapsed, world, torch.device("cpu"))
        cfg = W.CONFIGS["zamba2_2p7b_prefill"].with_(seqlen=8, nheads=2)
        first = W.make_prefill_inputs(cfg, bench.rank_seed(rank))["zxbcdt"][0, 0, :4]
        firsts = [torch.zeros(4, dtype=first.dtype) for _ in range(world)]
        dist.all_gather(firsts, first)
        out[rank] = (m, bench.job_rate(4096, 10, m, world),
                     bool(torch.equal(firsts[0], firsts[1])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_distinct_sequences():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    for r in range(world):
        m, rate, same = res[r]
        assert m == 15.0
        assert rate == pytest.approx(2 * 4096 * 10 / 0.015)
        assert not same  # each rank ran its own sequence


def test_reference_arm_on_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "1"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
