"""Multi-rank host logic of bench.py on the CPU: two gloo ranks (no GPU).

Each rank decodes its own sequences; the only cross-rank steps are the barrier
and the max over ranks of the step time, and the reference arm runs on rank 0
alone.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    got_ws, got_rank, local = bench.dist_setup(None, backend="gloo")
    step_ms = 1.0 + 0.5 * rank            # the last rank is the slowest
    ms = bench.max_over_ranks(step_ms, got_ws, device="cpu")
    value = bench.whole_job_value(ms, got_ws, 4)
    seed = bench.rank_seed(1000, rank)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got_ws, got_rank, local, ms, value, seed))


def _run_ranks(ws):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    return res


def test_two_ranks_report_the_slowest_step_and_the_whole_job_value():
    res = _run_ranks(2)
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 and r[2] == r[0] and r[3] == r[0] for r in res)
    # every rank sees the slowest rank's step time
    assert [r[4] for r in res] == [1.5, 1.5]
    # 2 ranks x 4 sequences, one token each per 1.5 ms step
    assert res[0][5] == pytest.approx(2 * 4 / 1.5e-3)
    # ranks draw different sequences
    assert res[0][6] != res[1][6]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.whole_job_value(2.0, 1, 4) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(bench.parse(["--impl", "reference", "--steps", "1", "--warmup", "0"]))
    assert capsys.readouterr().out == ""
