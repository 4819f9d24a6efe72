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


def test_extra_denominators():
    d = bench.extra_denominators(1225.1, 1965.0, nvfp4=False)
    # 2 ops x 8192 MACs x 148 SMs x 1.965 GHz = 4765 TOPS
    assert d["peak_mma_rate"] == pytest.approx(4765.0, abs=1.0)
    assert d["frac_mma_rate"] == pytest.approx(1225.1 / 4765.0, abs=1e-4)
    assert d["peak_datasheet"] == 4500.0 and d["frac_datasheet"] == pytest.approx(0.2722, abs=1e-4)
    nv = bench.extra_denominators(830.0, 1965.0, nvfp4=True)
    assert nv["peak_datasheet"] == 9000.0 and "peak_mma_rate" not in nv
    assert "peak_mma_rate" not in bench.extra_denominators(1000.0, None, nvfp4=False)


def test_both_arms_share_the_config():
    assert bench.workload_config(W.CAUSAL_GQA, 1)["l2"].startswith("inputs larger than L2")
    assert bench.workload_config(W.NVFP4, 2)["parallelism"] == "replicas x2"


def test_oracle_sample_times_the_nvfp4_oracle_for_the_nvfp4_workload(monkeypatch):
    import oracle as O
    seen = []
    real_q, real_a = O.quantize_qkv_nvfp4, O.attention_nvfp4
    monkeypatch.setattr(O, "quantize_qkv_nvfp4", lambda *a, **k: seen.append("q") or real_q(*a, **k))
    monkeypatch.setattr(O, "attention_nvfp4", lambda *a, **k: seen.append("a") or real_a(*a, **k))
    ops, dt = bench.oracle_sample(W.NVFP4, 256)
    assert seen == ["q", "a"] and dt > 0
    assert ops == W.NVFP4.scaled(B=1, Hq=1, Hkv=1, N=256).ops


def test_roofline_peak_is_burst_for_short_timed_regions():
    """roofline.frac divides by the measured bf16 burst rate (x2 INT8/FP8,
    x4 FP4) unless the timed region lasts at least 2 s (then the sustained
    rate, measured over seconds under the power cap)."""
    peaks, _ = bench.load_peaks()
    burst = peaks.get("bf16_tflops", bench.FALLBACK_PEAKS["bf16_tflops"])
    sus = peaks.get("bf16_tflops_sustained", bench.FALLBACK_PEAKS["bf16_tflops_sustained"])
    p, b, s, src = bench.peak_for(W.CAUSAL_GQA, 0.15)
    assert p == b == 2 * burst and s == 2 * sus and "burst" in src
    p, b, s, src = bench.peak_for(W.CAUSAL_GQA, 2.5)
    assert p == 2 * sus and "sustained" in src
    p, _, _, src = bench.peak_for(W.NVFP4, 0.3)
    assert p == 4 * burst and "FP4" in src
    r = bench.roofline_of(W.CAUSAL_GQA, 7.0, 0.15, 1965.0)
    assert r["frac"] == r["frac_burst"] and r["frac_sustained"] > r["frac"]


def test_quantiser_bytes_of_the_workloads():
    # causal GQA: bf16 read + int8/e4m3 written per element, plus scales,
    # means and q.kmean
    assert bench.quantiser_bytes(W.CAUSAL_GQA) == 1216462848
    assert bench.quantiser_bytes(W.NVFP4) > 3 * W.NVFP4.B * W.NVFP4.Hq * W.NVFP4.N * W.NVFP4.D * 2
