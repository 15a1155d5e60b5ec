"""Host-side multi-rank logic of bench.py, run as two gloo ranks on the CPU.

bench.py --gpus N runs one rank per GPU; the path has no exchange step (replicas, weak
scaling), so the only cross-rank operations are the barriers around the timed region and
the max over ranks of the device time.  These tests run exactly those helpers with the gloo
backend, plus the reference arm's rule that ranks other than 0 exit without work.
"""

import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup()
    assert (w, r, local) == (world, rank, rank)
    bench.maybe_init_pg(w, "gloo")
    bench.barrier(w)
    # each rank "measured" a different step time; everybody must see the slowest one
    ms = bench.max_over_ranks(w, 10.0 + 5.0 * rank, "cpu")
    bench.barrier(w)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(repr(ms))


def test_max_over_ranks_and_barriers_gloo(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    got = [float(open(tmp_path / f"rank{r}.txt").read()) for r in range(world)]
    assert got == [15.0, 15.0]


def test_whole_job_value_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    b, f = bench.step_units(bench.workload_spec("ffn8b_decode"))
    one = bench.whole_job_value("GB/s", b, f, 1, 2.0)
    assert one == pytest.approx(b / 2e-3 / 1e9)
    # same per-rank step time on 4 ranks: 4x the units in the same time
    assert bench.whole_job_value("GB/s", b, f, 4, 2.0) == pytest.approx(4 * one)
    # the slowest rank sets the time
    assert bench.whole_job_value("GB/s", b, f, 4, 4.0) == pytest.approx(2 * one)
    bp, fp = bench.step_units(bench.workload_spec("ffn8b_prefill"))
    assert bench.whole_job_value("TFLOP/s", bp, fp, 2, 1.0) == pytest.approx(2 * fp / 1e-3 / 1e12)


def test_reference_arm_nonzero_rank_exits_without_work(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    called = []
    monkeypatch.setattr(bench, "host_weights", lambda: called.append(1))
    args = type("A", (), dict(workload="ffn8b_decode", steps=3, warmup=3, gpus=2))()
    assert bench.run_reference(args) == 0
    assert called == [] and capsys.readouterr().out == ""
