"""The multi-GPU bench path on CPU: two ranks over gloo (one process each).

bench.py runs one batch of the workload per GPU with no collective on the
data path; the only cross-rank steps are the barrier and the max over ranks
of the measured time, and rank 0 alone prints. These tests run those steps
with world size 2 on the CPU."""
import datetime
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ms = bench.max_over_ranks(3.0 if rank == 1 else 2.0, torch.device("cpu"))
    value = bench.whole_job_tflops(world, 2e9, ms)
    # each rank draws its own batch (seed = rank): same shapes, other values
    import synth
    q = synth.draw(1, 2, 16, 8, "f32", 1.0, seed=rank)[0]
    out.put((rank, ms, value, q.shape, float(q.sum())))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_report_the_slowest_time_and_all_the_work():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(out.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    (r0, ms0, v0, s0, q0), (r1, ms1, v1, s1, q1) = got
    assert (r0, r1) == (0, 1)
    assert ms0 == ms1 == 3.0                      # the slower rank's time, on both
    assert v0 == v1 == pytest.approx(2 * 2e9 / 3e-3 / 1e12)
    assert s0 == s1 and q0 != q1                  # weak scaling: a batch of its own


def test_single_rank_time_is_its_own():
    import torch
    import bench
    assert bench.max_over_ranks(1.25, torch.device("cpu")) == 1.25
    assert bench.whole_job_tflops(1, 1e12, 1000.0) == pytest.approx(1.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    bench.run_reference(bench.parse())
    assert capsys.readouterr().out == ""
