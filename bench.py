"""Benchmark of the quantized-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one pass of the whole path over one batch of synthetic input:
the quantisation stage (sage_quantize_qkv: smooth_k, per-block INT8 Q/K,
per-channel FP8 V) followed by the fused INT8-QK / FP8-PV attention
(sage_attn_fwd_quantized), on the causal GQA workload B=4, Hq=32, Hkv=8,
N=16384, d=128 by default.  The metric is attention TOPS,
4*B*Hq*N*N*d / step time (halved for causal).

Timing: W warm-up steps, then K steps bracketed by a barrier and
cuda.synchronize on both sides, CUDA events on the launching stream, max
over ranks.  Inputs (805 MB of bf16 per step) are larger than L2.  SM clocks
and throttle reasons are sampled with nvidia-smi during the timed region.

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica
of the workload (seeded by rank; the path has no exchange step), so the
scaling is weak and the value is the ops of all ranks over the max time.

--impl reference times the CPU oracle (the reference arm) on
rank 0: every step quantises and attends a bounded sample of the workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "attention TOPS at seq 16K hd128 and % of B200 dense INT8/FP8 tensor peak"
UNIT = "TOPS"
# dense INT8/FP8 : BF16 tensor throughput on B200 (4.5 vs 2.25 PFLOP/s nominal)
FP8_PER_BF16 = 2.0
# dense FP4 : BF16 (9 vs 2.25 PFLOP/s nominal)
FP4_PER_BF16 = 4.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Two more denominators reported beside the measured-bf16 one: NVIDIA's dense
# datasheet peaks per B200 (TFLOP/s), and the tcgen05 MMA rate measured on
# this part (a 128x128x32 kind::i8 or kind::f8f6f4 MMA every 64 clocks per
# SM: 8192 MACs per clock per SM) at the SM clock sampled during the run.
DATASHEET_TFLOPS = {"int8/fp8": 4500.0, "fp4": 9000.0}
MMA_MACS_PER_CLK_SM = {"int8/fp8": 8192}
N_SMS = 148


def extra_denominators(achieved, sm_mhz, nvfp4):
    """frac of `achieved` TFLOP/s against the datasheet dense peak and, where
    measured, against the MMA issue rate at the sampled SM clock."""
    kind = "fp4" if nvfp4 else "int8/fp8"
    d = {"peak_datasheet": DATASHEET_TFLOPS[kind],
         "frac_datasheet": round(achieved / DATASHEET_TFLOPS[kind], 4)}
    macs = MMA_MACS_PER_CLK_SM.get(kind)
    if macs and sm_mhz:
        rate = 2.0 * macs * N_SMS * sm_mhz * 1e6 / 1e12
        d.update(peak_mma_rate=round(rate, 1), frac_mma_rate=round(achieved / rate, 4),
                 mma_rate_source=f"measured tcgen05 {kind} MMA rate x {N_SMS} SMs at {sm_mhz:g} MHz")
    return d


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# ------------------------------------------------------------------ ranks
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend):
    import datetime
    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_workload(w: W.Workload, rank: int) -> W.Workload:
    """Replica of the workload for one rank: same shapes, its own seed."""
    return w.scaled(seed=w.seed + 1000 * rank)


# ------------------------------------------------------------------ peaks, clocks
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


CLOCK_FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw",
                "clocks_event_reasons.sw_power_cap", "clocks_event_reasons.hw_slowdown",
                "clocks_event_reasons.hw_thermal_slowdown",
                "clocks_event_reasons.sw_thermal_slowdown",
                "clocks_event_reasons.hw_power_brake_slowdown"]


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons every 200 ms."""

    def __init__(self, gpu_index: int):
        self.proc = None
        self.path = f"/tmp/sage_clocks_{os.getpid()}.csv"
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", "--query-gpu=" + ",".join(CLOCK_FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) == len(CLOCK_FIELDS):
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["sw_power_cap", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "hw_power_brake_slowdown"]
        reasons = sorted({names[i] for r in rows for i in range(5) if r[3 + i] == "Active"})
        sm_sorted = sorted(sm)
        return {"sm_mhz": sm_sorted[len(sm_sorted) // 2] if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle timing
def oracle_sample(w: W.Workload, tokens: int):
    """One bounded sample of workload ``w`` for the CPU oracle: the first
    KV head group (one KV head and its Hq/Hkv Q heads) of batch 0, truncated
    to the first ``tokens`` tokens; quantised and attended in full.
    Returns (ops, seconds)."""
    import oracle as O
    G = w.Hq // w.Hkv
    ukl = w.unpadded_k_len if w.unpadded_k_len and w.unpadded_k_len < tokens else None
    ws = w.scaled(B=1, Hq=G, Hkv=1, N=tokens, unpadded_k_len=ukl)
    q, k, v = W.make_qkv(ws)
    mask = W.make_mask(ws)
    t0 = time.perf_counter()
    if ws.nvfp4:
        oz = O.quantize_qkv_nvfp4(q, k, v, per_block_mean=ws.per_block_mean, unpadded_k_len=ukl)
        O.attention_nvfp4(oz, causal=ws.causal, sm_scale=ws.sm_scale)
    else:
        oz = O.quantize_qkv_i8f8(q, k, v)
        O.attention_i8f8(oz, causal=ws.causal, sm_scale=ws.sm_scale,
                         mask=None if mask is None else mask.numpy())
    dt = time.perf_counter() - t0
    return ws.ops, dt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(w: W.Workload, budget_s=15.0):
    tokens = 2048
    ops, dt = oracle_sample(w, tokens)
    reps = max(1, min(64, int(budget_s / max(dt, 1e-3))))   # ~budget_s of CPU work
    tot_ops, tot_t = 0.0, 0.0
    for _ in range(reps):
        o, t = oracle_sample(w, tokens)
        tot_ops += o
        tot_t += t
    return {"value": tot_ops / tot_t / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "cpu": cpu_model(), "sample": f"{reps} x (first KV-head group of batch 0, {w.Hq // w.Hkv} Q heads, first "
                      f"{tokens} tokens: oracle quantise + attend in full); {tot_t:.1f} s of CPU work"}


def workload_config(w: W.Workload, ranks: int):
    """The `config` object of both arms' JSON lines."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "D": w.D,
            "causal": w.causal, "return_lse": True, "mask": w.mask, "input_dtype": "bf16",
            "nvfp4": w.nvfp4, "unpadded_k_len": w.unpadded_k_len,
            "l2": f"inputs larger than L2 (q/k/v bf16 "
                  f"{(w.B * (w.Hq + 2 * w.Hkv) * w.N * w.D * 2) >> 20} MiB per step, not flushed)",
            "parallelism": f"replicas x{ranks}"}


# ------------------------------------------------------------------ our arm
def quantiser_bytes(w: W.Workload) -> int:
    """The quantiser's algorithmic bytes: bf16 Q/K/V read once, codes,
    scales, means, q.kmean and (NVFP4) qk_correction written once."""
    eq, ekv = w.B * w.Hq * w.N * w.D, w.B * w.Hkv * w.N * w.D
    nqb = (w.N + 127) // 128
    if w.nvfp4:
        return (2 * (eq + 2 * ekv) + (eq + 2 * ekv) // 2 + (eq + 2 * ekv) // 16
                + w.B * w.Hq * nqb * (nqb * 128) * 4 + w.B * w.Hq * nqb * w.D * 4
                + w.B * w.Hkv * w.D * 4 + w.B * w.Hq * w.N * 4)
    return (3 * (eq + 2 * ekv) + (w.B * w.Hq + w.B * w.Hkv) * nqb * 4
            + 2 * w.B * w.Hkv * w.D * 4 + w.B * w.Hq * w.N * 4)


class StepRunner:
    """Device buffers and one step (quantise + attend) of workload ``w``."""

    def __init__(self, S, w: W.Workload, device, rank: int = 0):
        self.S, self.w, self.device = S, w, device
        wr = rank_workload(w, rank)
        self.q, self.k, self.v = W.make_qkv(wr, device=device)
        self.mask = W.make_mask(wr, device=device)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(w.B, w.Hq, w.N, dtype=torch.float32, device=device)
        self.stream = torch.cuda.current_stream(device)
        if w.nvfp4:
            ukl = w.unpadded_k_len or w.N
            self.z = S.QuantizedNvfp4.empty(w.B, w.Hq, w.Hkv, w.N, w.N, w.D, ukl, w.per_block_mean,
                                            device)
            nbytes = S.lib().sage_quantize_nvfp4_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.N, w.D)
            self.launches = 6       # column sums x2, means, codes, correction; attention
        else:
            self.z = S.QuantizedQKV.empty(w.B, w.Hq, w.Hkv, w.N, w.N, w.D, device, with_qdk=True)
            nbytes = S.lib().sage_quantize_workspace_bytes(w.B, w.Hkv, w.N, w.D)
            # K-mean/V-amax partials, their combination, block codes; attention
            # (+ the mask's tile classification)
            self.launches = 4 + (1 if self.mask is not None else 0)
        self.qws = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)

    def step(self, ev_q=None, ev_a=None, ev_b=None):
        S, w, z = self.S, self.w, self.z
        if ev_q is not None:
            ev_q.record(self.stream)
        if w.nvfp4:
            S.sage_quantize_qkv_nvfp4(self.q, self.k, self.v, per_block_mean=w.per_block_mean,
                                      unpadded_k_len=w.unpadded_k_len, out=z, ws=self.qws)
        else:
            S.sage_quantize_qkv(self.q, self.k, self.v, out=z, ws=self.qws)
        if ev_a is not None:
            ev_a.record(self.stream)
        if w.nvfp4:
            S.sage_attn_fwd_nvfp4(z, sm_scale=w.sm_scale, causal=w.causal, return_lse=True,
                                  out=self.out, lse=self.lse)
        else:
            S.sage_attn_fwd_quantized(z, causal=w.causal, sm_scale=w.sm_scale, return_lse=True,
                                      mask=self.mask, out=self.out, lse=self.lse)
        if ev_b is not None:
            ev_b.record(self.stream)

    def timed(self, steps):
        """Run ``steps`` steps with CUDA events on the launching stream:
        (whole-region ms, mean attention ms, mean quantiser ms)."""
        evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(self.device)
        e0.record(self.stream)
        for i in range(steps):
            self.step(*evs[i])
        e1.record(self.stream)
        torch.cuda.synchronize(self.device)
        return (e0.elapsed_time(e1), sum(a.elapsed_time(b) for _, a, b in evs) / steps,
                sum(q.elapsed_time(a) for q, a, _ in evs) / steps)


def peak_for(w: W.Workload, timed_s: float):
    """Denominator of roofline.frac: the measured bf16 GEMM rate times the
    dense INT8/FP8 (x2) or FP4 (x4) ratio; the burst figure for a timed region
    shorter than 2 s, the sustained one (measured over seconds, under the
    power cap) for a longer one."""
    peaks, src = load_peaks()
    ratio = FP4_PER_BF16 if w.nvfp4 else FP8_PER_BF16
    sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]) * ratio
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * ratio
    kind = "FP4" if w.nvfp4 else "INT8/FP8"
    if timed_s >= 2.0:
        return sus, burst, sus, f"{src} bf16 sustained x{ratio:g} (dense {kind}:BF16; timed region {timed_s:.2f} s >= 2 s)"
    return burst, burst, sus, f"{src} bf16 burst x{ratio:g} (dense {kind}:BF16; timed region {timed_s:.2f} s < 2 s)"


def roofline_of(w: W.Workload, attn_ms: float, timed_s: float, sm_mhz):
    """roofline object for the attention kernel of workload ``w``."""
    peak, burst, sus, src = peak_for(w, timed_s)
    achieved = w.visible_ops / (attn_ms * 1e-3) / 1e12
    r = {"bound": "tensor",
         "kernel": "attn_fwd_nvfp4_kernel<128>" if w.nvfp4 else "attn_fwd_i8f8_kernel<128>",
         "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
         "frac": round(achieved / peak, 4), "traffic": None, "peak_source": src,
         "peak_burst": round(burst, 1), "frac_burst": round(achieved / burst, 4),
         "peak_sustained": round(sus, 1), "frac_sustained": round(achieved / sus, 4),
         "attn_ms": round(attn_ms, 4)}
    r.update(extra_denominators(achieved, sm_mhz, w.nvfp4))
    return r


def quantize_of(w: W.Workload, quant_ms: float):
    peaks, src = load_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    qbytes = quantiser_bytes(w)
    gbs = qbytes / (quant_ms * 1e-3) / 1e9
    return {"kernels": "all quantiser kernels of the step", "ms": round(quant_ms, 4),
            "algorithmic_bytes": qbytes, "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(gbs / hbm, 4), "peak_source": f"{src} HBM copy bandwidth"}


EXTRA_WORKLOADS = [W.TINY, W.LLM_MASK, W.VIDEO_DIT, W.NVFP4]


def extra_configs(S, device, main: W.Workload, warmup=3, min_s=0.25):
    """The other workloads' figures, each timed in this run after the main
    timed region: per workload a few warm-up steps, then enough timed steps
    for about ``min_s`` seconds (at least 10), with the SM clock sampled."""
    res = {}
    for w in EXTRA_WORKLOADS:
        if w.name == main.name:
            continue
        r = StepRunner(S, w, device)
        for _ in range(warmup):
            r.step()
        t_ms, _, _ = r.timed(3)
        steps = max(10, int(min_s * 1e3 / max(t_ms / 3, 1e-3)))
        sampler = ClockSampler(device.index or 0)
        time.sleep(0.3)
        ms, attn_ms, quant_ms = r.timed(steps)
        clocks = sampler.stop()
        st, site = S.sage_get_device_status()
        if st != S.SAGE_OK:
            raise RuntimeError(f"device wait timed out at site {site} ({w.name})")
        ms_step = ms / steps
        e = {"config": workload_config(w, 1), "steps": steps, "warmup": warmup,
             "ms_per_step": round(ms_step, 4),
             "value": round(w.ops / (ms_step * 1e-3) / 1e12, 2), "unit": UNIT,
             "roofline": roofline_of(w, attn_ms, ms * 1e-3, (clocks or {}).get("sm_mhz")),
             "quantize": quantize_of(w, quant_ms), "clocks": clocks}
        if w.visible_ops != w.ops:
            e["value_visible_pairs"] = round(w.visible_ops / (ms_step * 1e-3) / 1e12, 2)
        res[w.name] = e
        del r
        torch.cuda.empty_cache()
    return res


def run_ours(args, w):
    import quantized_attention_05_b200 as S
    ws_, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if ws_ > 1:
        init_dist("nccl")
    S.lib()
    runner = StepRunner(S, w, device, rank)
    q, k, v, mask, out, lse = runner.q, runner.k, runner.v, runner.mask, runner.out, runner.lse
    stream = runner.stream
    launches_per_step = runner.launches

    for _ in range(args.warmup):
        runner.step()
    torch.cuda.synchronize(device)
    st, site = S.sage_get_device_status()
    if st != S.SAGE_OK:
        raise RuntimeError(f"device wait timed out at site {site}")

    sampler = ClockSampler(local) if rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    barrier(device)
    ms_local, attn_ms_local, quant_ms_local = runner.timed(args.steps)
    barrier(device)
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(ms_local, device)
    attn_ms = max_over_ranks(attn_ms_local, device)
    quant_ms = max_over_ranks(quant_ms_local, device)
    st, site = S.sage_get_device_status()
    if st != S.SAGE_OK:
        raise RuntimeError(f"device wait timed out at site {site}")

    # ---- end to end through the C ABI with host buffers
    k_e2e = max(1, min(args.steps, 8))
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    outh = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    lseh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    maskh = None if mask is None else mask.cpu().pin_memory()
    md = None if mask is None else torch.empty_like(mask)
    if w.nvfp4:
        ws_host = torch.empty(S.sage_attn_fwd_nvfp4_host_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.N, w.D),
                              dtype=torch.uint8, device=device)
        e2e_api = "sage_attn_fwd_nvfp4_host on pinned host buffers (chunked, copies overlapped)"
    else:
        # the host-resident entry point: chunked, copies overlapped with the kernels
        ws_host = torch.empty(S.sage_attn_fwd_host_workspace_bytes(
            w.B, w.Hq, w.Hkv, w.N, w.N, w.D, None if mask is None else tuple(mask.shape[:2])),
            dtype=torch.uint8, device=device)
        e2e_api = "sage_attn_fwd_host on pinned host buffers (chunked, copies overlapped)"

    def e2e_step():
        if md is not None:
            md.copy_(maskh, non_blocking=True)
        if w.nvfp4:
            S.sage_attn_fwd_nvfp4_host(qh, kh, vh, sm_scale=w.sm_scale, causal=w.causal,
                                       per_block_mean=w.per_block_mean,
                                       unpadded_k_len=w.unpadded_k_len, return_lse=True, out=outh,
                                       lse=lseh, ws=ws_host, device=device)
        else:
            S.sage_attn_fwd_host(qh, kh, vh, causal=w.causal, sm_scale=w.sm_scale, return_lse=True,
                                 mask=md, out=outh, lse=lseh, ws=ws_host, device=device)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(device)
    barrier(device)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(k_e2e):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / k_e2e, device)
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v)) + (0 if mask is None else mask.numel())
    d2h = out.numel() * out.element_size() + lse.numel() * 4

    ranks = ws_
    ms_step = ms / args.steps
    value = ranks * w.ops / (ms_step * 1e-3) / 1e12
    roof = roofline_of(w, attn_ms, ms * 1e-3, (clocks or {}).get("sm_mhz"))
    tr_path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if os.path.exists(tr_path):
        try:
            tr = json.load(open(tr_path))
            if tr.get("workload") == w.name and tr.get("kernel_hash") == kernel_hash():
                roof["traffic"] = tr.get("bytes_per_launch")
        except (OSError, ValueError):
            pass
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": ranks,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("nvfp4 (e2m1 x e2m1, e4m3 block-16 scales) -> f32" if w.nvfp4 else
                  "i8xi8->i32 (QK), e4m3xe4m3->f32 (PV)"), "data": "synthetic",
        "config": workload_config(w, ranks),
        "roofline": roof,
        "e2e": {"value": round(ranks * w.ops / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 3), "api": e2e_api},
        "quantize": quantize_of(w, quant_ms),
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if w.visible_ops != w.ops:      # a mask hides pairs: the step's TOPS over the visible ones too
        line["value_visible_pairs"] = round(ranks * w.visible_ops / (ms_step * 1e-3) / 1e12, 2)
    if ranks == 1 and not args.no_extra:
        del runner, q, k, v, mask, qh, kh, vh, outh, lseh, ws_host
        torch.cuda.empty_cache()
        line["extra"] = {"configs": extra_configs(S, device, w),
                         "note": "the other workloads, each timed in this run after the main timed "
                                 "region (same step, metric and roofline rules)"}
    if rank == 0 and ranks == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


def kernel_hash():
    """Hash of the attention kernel source: a recorded DRAM traffic figure is
    reported only while the kernel it was measured on is unchanged."""
    import hashlib
    h = hashlib.sha256()
    for f in ("attn_fwd_i8f8.cuh", "sage_ptx.cuh"):
        with open(os.path.join(ROOT, "quantized_attention_05_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------ reference arm
def run_reference(args, w):
    ws_, rank, _ = dist_env()
    if rank != 0:
        return
    tokens = 1024
    for _ in range(args.warmup):
        oracle_sample(w, tokens)
    tot_ops, tot_t = 0.0, 0.0
    for _ in range(args.steps):
        o, t = oracle_sample(w, tokens)
        tot_ops += o
        tot_t += t
    value = tot_ops / tot_t / 1e12
    sample = (f"each step: first KV-head group of batch 0 ({w.Hq // w.Hkv} Q heads), first {tokens} "
              f"tokens, oracle quantise + attend in full")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws_, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * tot_t / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64 (oracle)", "data": "synthetic", "impl": "reference",
        "config": workload_config(w, ws_),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "cpu": cpu_model(), "sample": sample + "; rank 0 only, on the host cores"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=W.CAUSAL_GQA.name, choices=sorted(W.BY_NAME))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads' figures (extra.configs)")
    ap.add_argument("--B", type=int, default=None,
                    help="override the batch size (smaller cases for profiling)")
    ap.add_argument("--N", type=int, default=None,
                    help="override the sequence length (smaller cases for profiling; an "
                         "unpadded key length scales with it)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = W.BY_NAME[args.workload]
    if args.B is not None:
        w = w.scaled(B=args.B, name=w.name.replace(f"_b{w.B}_", f"_b{args.B}_"))
    if args.N is not None:
        ukl = None if w.unpadded_k_len is None else w.unpadded_k_len * args.N // w.N
        w = w.scaled(N=args.N, unpadded_k_len=ukl, name=w.name.replace(f"_n{w.N}_", f"_n{args.N}_"))
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
