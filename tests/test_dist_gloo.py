"""Multi-rank host logic of the benchmark, on CPU with the gloo backend.

The path shards by replication (every rank runs its own batch, no data-path
collective); ranks meet only to take the max of their device times.  Two
gloo ranks check that reduction and the whole-job throughput formula, and
that the reference arm prints on rank 0 only.
"""

import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ms = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu")
    results[rank] = ms
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        assert dict(results) == {0: 15.0, 1: 15.0}


def test_whole_job_throughput_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tflops(1e12, 10, 1, 10.0)
    two = bench.whole_job_tflops(1e12, 10, 2, 10.0)
    assert one == pytest.approx(1000.0) and two == pytest.approx(2000.0)
    assert bench.max_over_ranks(3.5, "cpu") == 3.5     # no process group: identity


def test_reference_arm_is_silent_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         env=env, cwd=ROOT, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_peak_rule_and_stage_statistics():
    """The roofline denominator: the burst cuBLAS figure for a timed region under
    two seconds, the sustained one for longer regions; stage statistics."""
    sys.path.insert(0, ROOT)
    import bench
    peaks = dict(hbm=6000.0, bf16=1600.0, bf16_sust=1400.0, sust_mhz=1350.0, src="test")
    assert bench.bf16_peak(peaks, 0.27)[0] == 1600.0
    assert "burst" in bench.bf16_peak(peaks, 0.27)[1]
    assert bench.bf16_peak(peaks, 2.0)[0] == 1400.0
    assert "sustained" in bench.bf16_peak(peaks, 5.0)[1]
    st = bench.stats([3.0, 1.0, 2.0, 10.0])
    assert st == {"mean": 4.0, "median": 2.5, "min": 1.0, "max": 10.0}
