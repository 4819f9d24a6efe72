"""Host logic of bench.py's multi-rank path on CPU (gloo, world size 2): the
timing reduction takes the max over ranks, totals add up, and every rank
gets its own replica of the workload."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist = bench.init_dist("gloo")
    try:
        local_ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(local_ms)
        tot = bench.sum_over_ranks(1.0)
        bench.barrier()
        w = bench.rank_workload(W.CAUSAL_GQA, rank)
        q.put((rank, mx, tot, w.seed))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replicas_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]          # max over ranks on every rank
    assert [r[2] for r in res] == [2.0, 2.0]
    assert res[0][3] != res[1][3]                       # distinct replicas


def test_single_process_reductions_are_identity():
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_workload(W.TINY, 0) == W.TINY


def test_reference_arm_line_on_cpu(capsys):
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workload",
                W.TINY.name])
    import json
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TOPS"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"]["workload"] == W.TINY.name


def test_warmup_below_three_is_rejected():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])
