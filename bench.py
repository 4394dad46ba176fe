#!/usr/bin/env python
"""Benchmark of the batch-invariant hot path on B200.

One *step* is one pass of every kernel of the path over a batch of M token rows
(default 1024) shaped like a Qwen3-8B layer plus its LM head:

    h1   = bi_rmsnorm(x, g_attn)                      [M, 4096]    bf16
    qkv  = bi_addmm(b_qkv, h1, [W_q; W_k; W_v])       [M, 6144]    bias N(0, 0.01) on q, 0 on k, v
    o    = bi_addmm(x, q, W_o)                        [M, 4096]    residual add (q = qkv[:, :4096])
    h2   = bi_rmsnorm(o, g_mlp)
    a    = bi_matmul_silu_mul(h2, [W_g; W_u])         [M, 12288]   SiLU(gate) * up in the epilogue
                                                                   (--mlp unfused: bi_matmul, then bi_silu_mul)
    y    = bi_addmm(o, a, W_down)                     [M, 4096]    residual add
    hf   = bi_rmsnorm(y, g_final)
    lg   = bi_matmul(hf, W_lm)                        [M, 151936]  bf16 logits
    lp   = bi_log_softmax(lg)                         [M, 151936]  fp32, one block per row
    ce   = bi_mean(lp)                                [M]          mean log-prob (= -H(uniform, p))

(attention itself is not one of the batch-invariant reduction kernels; q stands
in for its output).  Weights are nn.Linear-style [N, K] bf16 N(0, 0.02), RMSNorm
gains 1 + N(0, 0.1), activations N(0, 1), all seeded.  The working set (~3 GB)
is far larger than the 126 MB L2, so no flush is needed between steps.

Printed: ONE JSON line on rank 0.  `value` = GEMM FLOPs of all ranks' steps /
max-over-ranks device time (TFLOP/s).  `--impl reference` times the fp64 CPU
oracle on a bounded sample of the same step instead (rank 0 only).
`--sweep` prints per-kernel M sweeps (not part of the JSON contract).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "bi_matmul TFLOP/s & row-op GB/s vs M (bitwise batch-invariant), % roofline"
WORKLOAD = "qwen3_8b_layer_plus_lm_head_logprobs"
HIDDEN, KV, FFN, VOCAB = 4096, 1024, 12288, 151936
EPS = 1e-6
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# (name, K, N) of the GEMMs of one step (FLOP accounting; q, k and v run as one launch).
GEMMS = [("q", HIDDEN, HIDDEN), ("k", HIDDEN, KV), ("v", HIDDEN, KV), ("o", HIDDEN, HIDDEN),
         ("gate_up", HIDDEN, 2 * FFN), ("down", FFN, HIDDEN), ("lm_head", HIDDEN, VOCAB)]
QKV = HIDDEN + 2 * KV
OPS_UNFUSED = ["rms1", "qkv", "o", "rms2", "gate_up", "silu_mul", "down", "rms3", "lm_head",
               "log_softmax", "mean"]
OPS_FUSED = ["rms1", "qkv", "o", "rms2", "gate_up_silu", "down", "rms3", "lm_head", "log_softmax", "mean"]


def gemm_flops_per_row() -> int:
    return sum(2 * K * N for _, K, N in GEMMS)


def row_op_bytes_per_row() -> dict:
    """Algorithmic HBM bytes per row of each row op (read inputs once, write outputs once)."""
    return {
        "rms1": 2 * HIDDEN + 2 * HIDDEN, "rms2": 2 * HIDDEN + 2 * HIDDEN, "rms3": 2 * HIDDEN + 2 * HIDDEN,
        "silu_mul": 2 * (2 * FFN) + 2 * FFN,
        "log_softmax": 2 * VOCAB + 4 * VOCAB,
        "mean": 4 * VOCAB + 4,
    }


def gemm_bytes(M: int, K: int, N: int, extra_in: int = 0) -> int:
    return 2 * (M * K + K * N + M * N) + extra_in


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_gemm_lm_head.json")
GEMM_SOURCES = [os.path.join(ROOT, "invariant_bi_matmul_02_b200", "csrc", n)
                for n in ("gemm.cuh", "gemm_pair.cuh", "maxsum.cuh", "ptx.cuh")]


def gemm_source_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for p in GEMM_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(rows: int, case: str):
    """DRAM bytes per LM-head launch from the committed ncu summary, or None when the
    capture is missing, was taken on another case or row count, or predates the GEMM source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    if (d.get("gemm_source_sha") != gemm_source_sha() or int(d.get("rows", -1)) != rows
            or d.get("kernel_case") != case):
        return None
    return int(d["dram_bytes_per_launch"])


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- workload

def make_weights() -> dict:
    """The step's weights on the host (bf16), drawn from fixed seeds; identical on every rank."""
    from invariant_bi_matmul_02_b200 import inputs
    return {
        "W_q": inputs.weight_normal(11, (HIDDEN, HIDDEN)),
        "W_k": inputs.weight_normal(12, (KV, HIDDEN)),
        "W_v": inputs.weight_normal(13, (KV, HIDDEN)),
        "W_o": inputs.weight_normal(14, (HIDDEN, HIDDEN)),
        "W_gu": inputs.weight_normal(15, (2 * FFN, HIDDEN)),
        "W_down": inputs.weight_normal(16, (HIDDEN, FFN)),
        "W_lm": inputs.weight_normal(17, (VOCAB, HIDDEN)),
        "g_attn": inputs.gain(18, HIDDEN),
        "g_mlp": inputs.gain(19, HIDDEN),
        "g_final": inputs.gain(20, HIDDEN),
        "b_q": inputs.bias(21, HIDDEN),
    }


class Workload:
    """Weights (shared by all ranks) and this rank's rows, resident on the device."""

    def __init__(self, rows: int, row0: int, device, fused_mlp: bool = True):
        import torch
        from invariant_bi_matmul_02_b200 import inputs
        self.M = rows
        self.fused = fused_mlp
        self.ops = OPS_FUSED if fused_mlp else OPS_UNFUSED
        self.host = make_weights()
        self.x_host = inputs.rows_normal(10, row0, rows, HIDDEN)
        self.dev = {k: v.to(device) for k, v in self.host.items()}
        # q, k and v as one projection: W_qkv = [W_q; W_k; W_v], bias zero on the k, v columns
        self.dev["W_qkv"] = torch.cat([self.dev["W_q"], self.dev["W_k"], self.dev["W_v"]]).contiguous()
        self.dev["b_qkv"] = torch.cat([self.dev["b_q"], torch.zeros(2 * KV, dtype=torch.bfloat16,
                                                                     device=device)]).contiguous()
        self.x = self.x_host.to(device)
        e = lambda *s, dt=torch.bfloat16: torch.empty(*s, dtype=dt, device=device)
        M = rows
        self.buf = {
            "h1": e(M, HIDDEN), "qkv": e(M, QKV), "o": e(M, HIDDEN),
            "h2": e(M, HIDDEN), "gu": e(M, 2 * FFN), "a": e(M, FFN), "y": e(M, HIDDEN),
            "hf": e(M, HIDDEN), "lg": e(M, VOCAB), "lp": e(M, VOCAB, dt=torch.float32),
            "ce": e(M, dt=torch.float32),
        }


def run_step(wl: Workload, x, marks=None, only=None, ce=None):
    """One pass of the hot path.  `marks` (CUDA events) brackets each op (len(OPS) + 1 events),
    or, with `only` naming an op, that op alone (2 events).  `ce`: where the per-row result goes
    (the workload's own buffer by default)."""
    from invariant_bi_matmul_02_b200 import binding as bi
    W, B = wl.dev, wl.buf
    if ce is None:
        ce = B["ce"]

    def mark(k):
        if marks is not None:
            marks[k].record()

    i = 0

    def begin(name):
        if only is not None and name == only:
            mark(0)

    def end(name):
        nonlocal i
        i += 1
        if only is None:
            mark(i)
        elif name == only:
            mark(1)

    if only is None:
        mark(0)
    begin("rms1"); bi.bi_rmsnorm(x, W["g_attn"], EPS, out=B["h1"]); end("rms1")
    begin("qkv"); bi.bi_addmm(W["b_qkv"], B["h1"], W["W_qkv"], "nk", out=B["qkv"]); end("qkv")
    begin("o"); bi.bi_addmm(x, B["qkv"][:, :HIDDEN], W["W_o"], "nk", out=B["o"]); end("o")
    begin("rms2"); bi.bi_rmsnorm(B["o"], W["g_mlp"], EPS, out=B["h2"]); end("rms2")
    if wl.fused:
        begin("gate_up_silu"); bi.bi_matmul_silu_mul(B["h2"], W["W_gu"], "nk", out=B["a"]); end("gate_up_silu")
    else:
        begin("gate_up"); bi.bi_matmul(B["h2"], W["W_gu"], "nk", out=B["gu"]); end("gate_up")
        begin("silu_mul"); bi.bi_silu_mul(B["gu"], out=B["a"]); end("silu_mul")
    begin("down"); bi.bi_addmm(B["o"], B["a"], W["W_down"], "nk", out=B["y"]); end("down")
    begin("rms3"); bi.bi_rmsnorm(B["y"], W["g_final"], EPS, out=B["hf"]); end("rms3")
    begin("lm_head"); bi.bi_matmul(B["hf"], W["W_lm"], "nk", out=B["lg"]); end("lm_head")
    begin("log_softmax"); bi.bi_log_softmax(B["lg"], out=B["lp"]); end("log_softmax")
    begin("mean"); bi.bi_mean(B["lp"], out=ce); end("mean")
    return ce


# ----------------------------------------------------------------------------- oracle leg

def oracle_step_rows(host: dict, x_rows, nthreads: int):
    """The same step in fp64 on the CPU oracle for a few rows (bf16 rounding between
    stages, as the device stores bf16 intermediates).  Returns the per-row mean log-prob."""
    import numpy as np
    import torch
    from invariant_bi_matmul_02_b200 import inputs
    from oracle import oracle

    b = inputs.bf16_bits
    to_bf16 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)
    h1 = to_bf16(oracle.rmsnorm(b(x_rows), b(host["g_attn"]), EPS, nthreads))
    q = to_bf16(oracle.addmm(b(host["b_q"]), b(h1), b(host["W_q"]), "nk", nthreads))
    oracle.matmul(b(h1), b(host["W_k"]), "nk", nthreads)
    oracle.matmul(b(h1), b(host["W_v"]), "nk", nthreads)
    o = to_bf16(oracle.addmm(b(x_rows), b(q), b(host["W_o"]), "nk", nthreads))
    h2 = to_bf16(oracle.rmsnorm(b(o), b(host["g_mlp"]), EPS, nthreads))
    gu = to_bf16(oracle.matmul(b(h2), b(host["W_gu"]), "nk", nthreads))
    a = to_bf16(oracle.silu_mul(b(gu), nthreads))
    y = to_bf16(oracle.addmm(b(o), b(a), b(host["W_down"]), "nk", nthreads))
    hf = to_bf16(oracle.rmsnorm(b(y), b(host["g_final"]), EPS, nthreads))
    lg = to_bf16(oracle.matmul(b(hf), b(host["W_lm"]), "nk", nthreads))
    lp = oracle.log_softmax(b(lg), nthreads).astype(np.float32)
    return oracle.mean(lp, nthreads)


def cpu_baseline(host: dict, x_host, budget_s: float = 15.0) -> dict:
    """Time the oracle on a bounded sample of the step (rank 0, N = 1)."""
    from oracle import oracle as orc
    cores = os.cpu_count() or 1
    orc.max_threads()
    t0 = time.perf_counter()
    oracle_step_rows(host, x_host[:1], cores)
    t1 = time.perf_counter() - t0
    rows = max(1, min(x_host.shape[0], int(budget_s / max(t1, 1e-3))))
    t0 = time.perf_counter()
    oracle_step_rows(host, x_host[:rows], cores)
    dt = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle_step_rows(host, x_host[:1], 1)  # the same oracle on one core
    dt1 = time.perf_counter() - t0
    return {"value": rows * gemm_flops_per_row() / dt / 1e12, "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{rows} of {x_host.shape[0]} rows through the whole step in fp64 "
                      f"({dt:.1f} s, after a 1-row calibration of {t1:.2f} s)",
            "value_1core": gemm_flops_per_row() / dt1 / 1e12,
            "sample_1core": f"1 row through the whole step in fp64 on one thread ({dt1:.2f} s)"}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self, window=None) -> dict:
        """Median SM clock and the throttle reasons seen.  With `window` = (t0, t1) host wall-clock
        seconds, only samples taken inside it count (the sampler starts before the timed region,
        and samples of an idle GPU would read its maximum clock)."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        from datetime import datetime
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                ts = None
            try:
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        inside = [r for r in rows if window and r[0] is not None and window[0] <= r[0] <= window[1]]
        use = inside if inside else rows
        sm, smax, reasons = [r[1] for r in use], (use[-1][2] if use else None), set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in use:
            for n, v in zip(names, r[3]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "window": "timed region" if inside else "whole sampling run"}


# ----------------------------------------------------------------------------- main arms

def physical_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            return int(vis.split(",")[local_rank])
        except (ValueError, IndexError):
            return local_rank
    return local_rank


def run_bi(args):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=device)

    from invariant_bi_matmul_02_b200.shard import weak_rows
    M = args.rows
    wl = Workload(M, weak_rows(M, rank)[0], device, fused_mlp=args.mlp == "fused")
    OPS = wl.ops
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        run_step(wl, wl.x)
    torch.cuda.synchronize()

    # Inside the timed region only the LM-head launch (the roofline kernel) is bracketed by
    # events; the per-op breakdown comes from a separate pass after it.
    lm_marks = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(physical_gpu_index(local_rank)) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)  # let nvidia-smi attach before the timed region
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    start.record(stream)
    for s in range(args.steps):
        run_step(wl, wl.x, lm_marks[s], only="lm_head")
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    clocks = sampler.stop((t_wall0, t_wall1)) if sampler else None
    barrier()
    elapsed_ms = start.elapsed_time(end)
    lm_ms = sum(m[0].elapsed_time(m[1]) for m in lm_marks) / args.steps

    bd_steps = max(1, min(args.steps, 50))
    marks = [[torch.cuda.Event(enable_timing=True) for _ in range(len(OPS) + 1)] for _ in range(bd_steps)]
    for s in range(bd_steps):
        run_step(wl, wl.x, marks[s])
    torch.cuda.synchronize()
    per_op = {op: 0.0 for op in OPS}
    for s in range(bd_steps):
        for i, op in enumerate(OPS):
            per_op[op] += marks[s][i].elapsed_time(marks[s][i + 1])
    per_op = {k: v / bd_steps for k, v in per_op.items()}

    # End to end through the public API: every step copies its input rows from pinned host
    # memory and the host reads the step's per-row result back.  Both copies run on a copy
    # stream, into and out of two alternating device buffers: the input for step s+1 while step s
    # computes, and step s's result once step s is done, so the compute stream holds only the
    # steps' kernels and the waits for their buffers.  The host reads step s's result while step
    # s+1 is queued, so the GPU is never left waiting on the host.
    x_pinned = wl.x_host.pin_memory()
    ce_pinned = [torch.empty(M, dtype=torch.float32).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(wl.x) for _ in range(2)]
    ce_dev = [torch.empty(M, dtype=torch.float32, device=device) for _ in range(2)]
    copy_stream = torch.cuda.Stream()
    e2e_steps = max(1, args.steps)  # as many steps as the timed region: the same power-capped regime
    host_sum = [0.0]

    def e2e_run(n, start_ev=None):
        copied = [torch.cuda.Event() for _ in range(2)]
        consumed = [torch.cuda.Event() for _ in range(2)]
        read = [torch.cuda.Event() for _ in range(2)]
        if start_ev is not None:
            copy_stream.wait_event(start_ev)
        with torch.cuda.stream(copy_stream):
            x_dev[0].copy_(x_pinned, non_blocking=True)
            copied[0].record(copy_stream)
        for s in range(n):
            i = s % 2
            if s + 1 < n:
                j = (s + 1) % 2
                with torch.cuda.stream(copy_stream):
                    if s >= 1:
                        copy_stream.wait_event(consumed[j])  # step s-1 is done with buffer j
                    x_dev[j].copy_(x_pinned, non_blocking=True)
                    copied[j].record(copy_stream)
            stream.wait_event(copied[i])
            if s >= 2:
                stream.wait_event(read[i])  # step s-2's result has left ce_dev[i]
            ce = run_step(wl, x_dev[i], ce=ce_dev[i])
            consumed[i].record(stream)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(consumed[i])  # step s is done
                ce_pinned[i].copy_(ce, non_blocking=True)  # the host read step s-2's value already
                read[i].record(copy_stream)
            if s >= 1:
                read[(s - 1) % 2].synchronize()  # the host reads step s-1's result
                host_sum[0] += float(ce_pinned[(s - 1) % 2][0])
        read[(n - 1) % 2].synchronize()
        host_sum[0] += float(ce_pinned[(n - 1) % 2][0])

    e2e_run(2)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(e2e_steps, e0)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)

    from invariant_bi_matmul_02_b200 import binding as bi
    status = bi.bi_get_device_status()

    if world > 1:
        t = torch.tensor([elapsed_ms, e2e_ms, float(status)], device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms, e2e_ms, status = float(t[0]), float(t[1]), int(t[2])

    flops_step = gemm_flops_per_row() * M
    value = world * flops_step * args.steps / (elapsed_ms / 1e3) / 1e12
    e2e_value = world * flops_step * e2e_steps / (e2e_ms / 1e3) / 1e12

    peaks, peak_src = load_peaks()
    long_run = elapsed_ms > 2000.0
    peak_tf = peaks["bf16_tflops_sustained" if long_run else "bf16_tflops"]
    lm_flops = 2 * M * HIDDEN * VOCAB
    achieved = lm_flops / (lm_ms / 1e3) / 1e12
    gemm_ms = sum(per_op[n] for n in ("qkv", "o", "gate_up", "gate_up_silu", "down", "lm_head")
                  if n in per_op)
    row_bytes = row_op_bytes_per_row()
    row_gbs = {op: round(b * M / (per_op[op] / 1e3) / 1e9, 1) for op, b in row_bytes.items()
               if op in per_op}

    # The per-kernel M sweep runs after every timed region, on this GPU alone (N = 1).
    sweep = metric_sweep(device, peaks) if world == 1 and not args.no_metric_sweep else None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(wl.host, wl.x_host, args.cpu_budget)
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(elapsed_ms / args.steps, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "rows_per_gpu": M, "global_rows": M * world,
                       "hidden": HIDDEN, "kv_out": KV, "ffn": FFN, "vocab": VOCAB,
                       "accumulate": "fp32", "parallelism": f"replicas x{world} (rows sharded)",
                       "mlp": "gate/up GEMM with SiLU*up in its epilogue" if wl.fused
                              else "gate/up GEMM, then bi_silu_mul",
                       "log_softmax": "bi_log_softmax after the LM head",
                       "l2": "working set ~3 GB > 126 MB L2; no flush",
                       # the tile each GEMM of the step runs, from its weight's rows alone
                       "gemm_tile": {op: bi.bi_gemm_config(rows) for op, rows in
                                     (("qkv", HIDDEN + 2 * KV), ("o", HIDDEN), ("gate_up", 2 * FFN),
                                      ("down", HIDDEN), ("lm_head", VOCAB))}},
            "roofline": {"kernel": "bi_matmul LM head launch [%d x 4096] x [4096 x 151936]" % M,
                         "bound": "tensor", "achieved": round(achieved, 1), "peak": peak_tf,
                         "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4),
                         "traffic": measured_traffic(M, "gemm_lm_head"),
                         "algorithmic_bytes": gemm_bytes(M, HIDDEN, VOCAB),
                         "peak_source": f"{peak_src} {'bf16_tflops_sustained' if long_run else 'bf16_tflops'}"},
            "gemm_all_launches_tflops": round(flops_step / (gemm_ms / 1e3) / 1e12, 1),
            "row_ops_gbs": row_gbs,
            "row_ops_hbm_peak_gbs": peaks["hbm_gbs"],
            "breakdown_ms": {k: round(v, 4) for k, v in per_op.items()},
            "breakdown_steps": bd_steps,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(wl.x.numel() * 2), "d2h_bytes_per_step": int(M * 4),
                    "steps": e2e_steps},
            "gpu_launches": len(OPS) * args.steps,
            "clocks": clocks,
            "device_status": status,
            "metric_sweep": sweep,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if status != 0:
        raise SystemExit(f"device status word set: {status}")


def run_reference(args):
    """The fp64 CPU oracle, timed on the host cores: each step is one row through the step."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import torch  # noqa: F401
    from invariant_bi_matmul_02_b200 import inputs
    M = args.rows
    hw = make_weights()
    cores = os.cpu_count() or 1
    x = inputs.rows_normal(10, 0, max(args.steps + args.warmup, 1), HIDDEN)
    for i in range(args.warmup):
        oracle_step_rows(hw, x[i:i + 1], cores)
    t0 = time.perf_counter()
    for s in range(args.steps):
        r = args.warmup + s
        oracle_step_rows(hw, x[r:r + 1], cores)
    dt = time.perf_counter() - t0
    value = args.steps * gemm_flops_per_row() / dt / 1e12
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / max(args.steps, 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "rows_per_gpu": M, "hidden": HIDDEN, "kv_out": KV,
                   "ffn": FFN, "vocab": VOCAB, "sample_rows_per_step": 1},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"1 of {M} rows through the whole step per timed step, fp64"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- sweep mode

SWEEP_M = [1, 2, 3, 4, 8, 16, 32, 64, 77, 128, 256, 512, 1000, 1024, 2048]
SWEEP_SHAPES = [("q/o", HIDDEN, HIDDEN), ("k/v", HIDDEN, KV), ("gate/up", HIDDEN, FFN),
                ("down", FFN, HIDDEN), ("lm_head", HIDDEN, VOCAB),
                # the step's stacked weights, which run the 256x192 tile
                ("qkv", HIDDEN, HIDDEN + 2 * KV), ("gate+up", HIDDEN, 2 * FFN)]


def _timed(fn, flush, reps):
    import torch
    times = []
    for _ in range(reps):
        flush()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        e.synchronize()
        times.append(s.elapsed_time(e))
    return statistics.median(times)


def _rows_differing(t, ref1):
    """Rows of t whose bits differ from the same rows computed alone (ref1)."""
    import torch
    n = ref1.shape[0]
    view = torch.int16 if t.element_size() == 2 else torch.int32
    return int((t[:n].contiguous().view(view) != ref1.contiguous().view(view)).any(dim=1).sum())


# ----------------------------------------------------------------------------- metric sweep (in the JSON line)

SWEEP_GEMMS = [("q/o", HIDDEN, HIDDEN), ("k/v", HIDDEN, KV), ("gate/up", HIDDEN, FFN), ("down", FFN, HIDDEN),
               ("lm_head", HIDDEN, VOCAB)]
METRIC_SWEEP_M = [1, 64, 256, 1024, 2048]
SWEEP_ROW_OPS = [("rmsnorm", HIDDEN, (1024, 16384)), ("mean", HIDDEN, (1024, 16384)),
                 ("log_softmax", VOCAB, (1, 64, 1024))]


def roofline_point(flop: float, nbytes: float, us: float, peaks: dict) -> dict:
    """Fraction of the roofline for one launch: the roofline time is the larger of the FLOPs at the
    tensor peak and the algorithmic bytes at the HBM peak; `bound` names the larger term."""
    t_tensor = flop / (peaks["bf16_tflops"] * 1e12) if flop else 0.0
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_roof = max(t_tensor, t_hbm)
    return {"bound": "tensor" if t_tensor >= t_hbm else "hbm", "roofline_frac": round(t_roof / (us * 1e-6), 3)}


def metric_sweep(device, peaks: dict, reps: int = 10) -> dict:
    """The metric's M sweep, per kernel, on synthetic inputs shaped like the workload: each bi
    kernel and torch's default kernel for the same op, timed alone (median of `reps` launches, a
    256 MB write before each to flush L2); TFLOP/s, algorithmic GB/s and the fraction of the
    roofline, and how many of the first 8 rows differ bit-wise from the same rows computed
    alone (M = 1)."""
    import torch
    import torch.nn.functional as F
    from invariant_bi_matmul_02_b200 import binding as bi
    g = torch.Generator(device=device)
    g.manual_seed(7)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    counter = [0]

    def flush():
        counter[0] += 1
        flush_buf.fill_(counter[0] & 0xFF)

    def us(fn):
        fn()
        return _timed(fn, flush, reps) * 1e3

    out = {"protocol": f"median of {reps} launches, 256 MB written before each (L2 flushed); inputs "
                       "N(0,1), weights N(0,0.02) [N,K]; peaks: burst", "gemm": [], "row_ops": []}
    for name, K, N in SWEEP_GEMMS:
        w = (torch.randn(N, K, generator=g, device=device) * 0.02).to(torch.bfloat16)
        a = torch.randn(max(METRIC_SWEEP_M), K, generator=g, device=device).to(torch.bfloat16)
        ref = torch.cat([bi.bi_matmul(a[i:i + 1], w) for i in range(8)])
        tref = torch.cat([F.linear(a[i:i + 1], w) for i in range(8)])
        for M in METRIC_SWEEP_M:
            am = a[:M]
            c = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            t_bi = us(lambda: bi.bi_matmul(am, w, out=c))
            t_t = us(lambda: F.linear(am, w))
            n = min(M, 8)
            flop, nbytes = 2.0 * M * N * K, float(gemm_bytes(M, K, N))
            out["gemm"].append({"shape": name, "M": M, "K": K, "N": N, "bi_us": round(t_bi, 1),
                                "tflops": round(flop / t_bi / 1e6, 1), "gbs": round(nbytes / t_bi / 1e3, 1),
                                **roofline_point(flop, nbytes, t_bi, peaks), "torch_us": round(t_t, 1),
                                "rows_differing_from_m1": _rows_differing(c, ref[:n]),
                                "torch_rows_differing_from_m1": _rows_differing(F.linear(am, w), tref[:n])})
        del w, a, ref, tref
    for op, H, ms in SWEEP_ROW_OPS:
        Mmax = max(ms)
        if op == "rmsnorm":
            x = torch.randn(Mmax, H, generator=g, device=device).to(torch.bfloat16)
            wn = (1 + 0.1 * torch.randn(H, generator=g, device=device)).to(torch.bfloat16)
            fb = lambda xm, y: bi.bi_rmsnorm(xm, wn, EPS, out=y)
            ft = lambda xm: F.rms_norm(xm, (H,), wn, EPS)
            y_of = lambda M: torch.empty(M, H, dtype=torch.bfloat16, device=device)
            per_row = 4 * H
        elif op == "mean":
            x = torch.randn(Mmax, H, generator=g, device=device)
            fb = lambda xm, y: bi.bi_mean(xm, out=y)
            ft = lambda xm: xm.mean(-1)
            y_of = lambda M: torch.empty(M, dtype=torch.float32, device=device)
            per_row = 4 * H + 4
        else:
            x = (1.3 * torch.randn(Mmax, H, generator=g, device=device)).to(torch.bfloat16)
            fb = lambda xm, y: bi.bi_log_softmax(xm, out=y)
            ft = lambda xm: torch.log_softmax(xm, -1, dtype=torch.float32)
            y_of = lambda M: torch.empty(M, H, dtype=torch.float32, device=device)
            per_row = 6 * H
        ref = torch.cat([fb(x[i:i + 1], y_of(1)).reshape(1, -1) for i in range(8)])
        tref = torch.cat([ft(x[i:i + 1]).reshape(1, -1) for i in range(8)])
        for M in ms:
            xm, y = x[:M], y_of(M)
            t_bi = us(lambda: fb(xm, y))
            t_t = us(lambda: ft(xm))
            n = min(M, 8)
            nbytes = float(per_row * M)
            out["row_ops"].append({"op": op, "M": M, "H": H, "bi_us": round(t_bi, 1),
                                   "gbs": round(nbytes / t_bi / 1e3, 1),
                                   "hbm_frac": round(nbytes / t_bi / 1e3 / peaks["hbm_gbs"], 3),
                                   "torch_us": round(t_t, 1),
                                   "rows_differing_from_m1": _rows_differing(y.reshape(M, -1), ref[:n]),
                                   "torch_rows_differing_from_m1": _rows_differing(ft(xm).reshape(M, -1),
                                                                                   tref[:n])})
        del x, ref, tref
    # Decode attention (f2) at the Qwen3-8B decode shape, B = 64 sequences of L = 4096 cached
    # tokens, 32 query / 8 kv heads, head sizes 128 and 64, against torch SDPA; the first 8
    # sequences are also decoded alone, for both.
    out["attention"] = []
    for D in (128, 64):
        B, L, Hq, Hkv = 64, 4096, 32, 8
        q = torch.randn(B, Hq, D, generator=g, device=device).to(torch.bfloat16)
        k = torch.randn(B, L, Hkv, D, generator=g, device=device).to(torch.bfloat16)
        v = torch.randn(B, L, Hkv, D, generator=g, device=device).to(torch.bfloat16)
        sl = torch.full((B,), L, dtype=torch.int32, device=device)
        scr = torch.empty(bi.bi_decode_attention_scratch_bytes(B, Hq, D, L), dtype=torch.uint8, device=device)
        o = torch.empty_like(q)
        sdpa = lambda qq, kk, vv: F.scaled_dot_product_attention(qq.view(qq.shape[0], Hq, 1, D), kk.permute(0, 2, 1, 3),
                                                                 vv.permute(0, 2, 1, 3), enable_gqa=True).view(qq.shape)
        t_bi = us(lambda: bi.bi_decode_attention(q, k, v, sl, scratch=scr, out=o))
        t_t = us(lambda: sdpa(q, k, v))
        alone = torch.cat([bi.bi_decode_attention(q[i:i + 1], k[i:i + 1], v[i:i + 1], sl[i:i + 1]) for i in range(8)])
        talone = torch.cat([sdpa(q[i:i + 1], k[i:i + 1], v[i:i + 1]) for i in range(8)])
        nbytes = 2.0 * B * L * Hkv * D * 2
        out["attention"].append({"op": "decode_attention", "B": B, "L": L, "Hq": Hq, "Hkv": Hkv, "D": D,
                                 "bi_us": round(t_bi, 1), "gbs": round(nbytes / t_bi / 1e3, 1),
                                 "hbm_frac": round(nbytes / t_bi / 1e3 / peaks["hbm_gbs"], 3),
                                 "torch_sdpa_us": round(t_t, 1),
                                 "rows_differing_from_alone": _rows_differing(o.reshape(B, -1), alone.reshape(8, -1)),
                                 "torch_rows_differing_from_alone": _rows_differing(sdpa(q, k, v).reshape(B, -1),
                                                                                    talone.reshape(8, -1))})
        del q, k, v, scr, o, alone, talone
    del flush_buf
    torch.cuda.empty_cache()
    return out


def run_mma_probe(args):
    """Cycles per back-to-back tcgen05.mma for several instruction shapes (the stand-alone probe
    built by csrc/build.py); one JSON line per shape."""
    from invariant_bi_matmul_02_b200.csrc import build as libbuild
    exe = libbuild.build_probe()
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    print(out, end="", flush=True)


def run_host_overhead(args):
    """Host time per bi_matmul call at M = 1 (K = N = 256) through the binding, with the tensor-map
    cache hitting (the same buffers every call) and missing (a new activation address each call,
    so one of the two maps is encoded), and the device time of the same launch for scale."""
    import torch
    from invariant_bi_matmul_02_b200 import binding as bi
    dev = torch.device("cuda", 0)
    K = N = 256
    w = torch.randn(N, K, device=dev).to(torch.bfloat16)
    pool = torch.randn(4096, K, device=dev).to(torch.bfloat16)  # 4096 distinct row addresses
    c = torch.empty(1, N, dtype=torch.bfloat16, device=dev)
    calls = 4000

    def host_us(rows):
        for i in range(50):
            bi.bi_matmul(rows(i), w, out=c)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for i in range(calls):
            bi.bi_matmul(rows(i), w, out=c)
        t = (time.perf_counter() - t0) / calls * 1e6
        torch.cuda.synchronize()
        return t

    h0, m0 = bi.bi_tensor_map_cache_stats()
    hit = host_us(lambda i: pool[:1])
    h1, m1 = bi.bi_tensor_map_cache_stats()
    miss = host_us(lambda i: pool[(i * 7) % 4096:(i * 7) % 4096 + 1])
    h2, m2 = bi.bi_tensor_map_cache_stats()
    # The C entry point alone (ctypes call with prepared arguments, maps cached): what the
    # binding's checks add is the difference.
    lib = bi.load()
    c_args = (pool.data_ptr(), K, w.data_ptr(), K, bi.BI_B_NK, c.data_ptr(), N, bi.BI_BF16, 1, N, K,
              torch.cuda.current_stream().cuda_stream)
    for _ in range(50):
        lib.bi_matmul(*c_args)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(calls):
        lib.bi_matmul(*c_args)
    c_abi = (time.perf_counter() - t0) / calls * 1e6
    torch.cuda.synchronize()
    print(json.dumps({"host_overhead": "bi_matmul M=1 K=N=256 through the binding",
                      "host_us_per_call_cache_hit": round(hit, 2), "host_us_per_call_one_miss": round(miss, 2),
                      "host_us_per_call_c_abi_only": round(c_abi, 2),
                      "hits_misses_hit_loop": [h1 - h0, m1 - m0], "hits_misses_miss_loop": [h2 - h1, m2 - m1]}))


def run_sweep(args):
    """Per-kernel M sweeps: bi kernels vs torch defaults, L2 flushed before every rep.
    For the first 64 rows of every M, both bi's and torch's outputs are compared bit for bit
    with the same rows computed alone (M = 1): bi must differ in none (invariance), torch's
    count is the negative control.  With --sweep-out the JSON is rewritten after every point,
    and --resume skips the points already in it."""
    import torch
    import torch.nn.functional as F
    from invariant_bi_matmul_02_b200 import binding as bi
    from invariant_bi_matmul_02_b200 import inputs

    dev = torch.device("cuda", 0)
    peaks, src = load_peaks()
    scratch = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush = lambda: scratch.fill_(1.0)
    reps = max(5, min(args.steps, 30))
    out = {"peaks": peaks, "peak_source": src, "gemm": [], "rows": []}
    if args.resume and args.sweep_out and os.path.exists(args.sweep_out):
        with open(args.sweep_out) as f:
            prev = json.load(f)
        out["gemm"], out["rows"] = prev.get("gemm", []), prev.get("rows", [])
    have = {("gemm", r["shape"], r["M"]) for r in out["gemm"]} | {("rows", r["op"], r["M"]) for r in out["rows"]}

    def save():
        if args.sweep_out:
            tmp = args.sweep_out + ".tmp"
            with open(tmp, "w") as f:
                json.dump(out, f, indent=1)
            os.replace(tmp, args.sweep_out)

    def row_rec(op, M, t_bi, by, t_t, bi_diff, t_diff, n):
        rec = {"op": op, "M": M, "bi_us": t_bi * 1e3, "bi_gbs": by / t_bi / 1e6,
               "bi_frac_hbm": by / t_bi / 1e6 / peaks["hbm_gbs"], "torch_us": t_t * 1e3,
               "torch_gbs": by / t_t / 1e6, "bi_rows_differing_from_m1": bi_diff,
               "torch_rows_differing_from_m1": t_diff, "rows_compared": n}
        out["rows"].append(rec)
        save()
        print(f"{op:20s} {M:6d} {t_bi*1e3:9.1f} {by/t_bi/1e6:8.0f} {100*by/t_bi/1e6/peaks['hbm_gbs']:5.1f}% "
              f"{t_t*1e3:9.1f} {by/t_t/1e6:10.0f} {bi_diff:>5d}/{n} {t_diff:>5d}/{n}", flush=True)

    print(f"peaks ({src}): {peaks}")
    print(f"{'shape':9s} {'M':>5s} {'bi us':>9s} {'bi TF/s':>8s} {'%pk':>6s} {'GB/s':>7s} "
          f"{'torch us':>9s} {'torch TF/s':>10s} {'bi != M=1':>10s} {'torch != M=1':>12s}")
    for name, K, N in SWEEP_SHAPES:
        if args.sweep_shapes and name not in args.sweep_shapes.split(","):
            continue
        if all(("gemm", name, M) in have for M in SWEEP_M):
            continue
        w = inputs.weight_normal(40, (N, K)).to(dev)
        pool = inputs.rows_normal(41, 0, max(SWEEP_M), K).to(dev)
        ref1 = torch.cat([F.linear(pool[i:i + 1], w) for i in range(64)])  # torch's rows at M = 1
        ref1_bi = torch.cat([bi.bi_matmul(pool[i:i + 1], w, "nk") for i in range(64)])
        for M in SWEEP_M:
            if ("gemm", name, M) in have:
                continue
            a = pool[:M]
            c = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            t_bi = _timed(lambda: bi.bi_matmul(a, w, "nk", out=c), flush, reps)
            n = min(M, 64)
            bi_diff = _rows_differing(c, ref1_bi[:n])
            t_t = _timed(lambda: torch.mm(a, w.t(), out=c), flush, reps)
            diff = _rows_differing(F.linear(a, w), ref1[:n])
            fl = 2 * M * N * K
            by = gemm_bytes(M, K, N)
            rec = {"shape": name, "K": K, "N": N, "M": M, "bi_us": t_bi * 1e3,
                   "bi_tflops": fl / t_bi / 1e9, "bi_frac_tensor": fl / t_bi / 1e9 / peaks["bf16_tflops"],
                   "bi_gbs": by / t_bi / 1e6, "bi_frac_hbm": by / t_bi / 1e6 / peaks["hbm_gbs"],
                   "torch_us": t_t * 1e3, "torch_tflops": fl / t_t / 1e9,
                   "bi_rows_differing_from_m1": bi_diff,
                   "torch_rows_differing_from_m1": diff, "rows_compared": n}
            out["gemm"].append(rec)
            save()
            print(f"{name:9s} {M:5d} {t_bi*1e3:9.1f} {rec['bi_tflops']:8.1f} "
                  f"{100*rec['bi_frac_tensor']:5.1f}% {rec['bi_gbs']:7.0f} {t_t*1e3:9.1f} "
                  f"{rec['torch_tflops']:10.1f} {bi_diff:>7d}/{n} {diff:>9d}/{n}", flush=True)
        del w, pool, ref1, ref1_bi
        torch.cuda.empty_cache()
    if not args.sweep_shapes or "rows" in args.sweep_shapes.split(","):
        print(f"{'op':20s} {'M':>6s} {'bi us':>9s} {'GB/s':>8s} {'%HBM':>6s} {'torch us':>9s} {'torch GB/s':>10s} "
              f"{'bi!=M=1':>7s} {'torch!=M=1':>10s}")
        g = inputs.gain(42, HIDDEN).to(dev)
        x64 = inputs.rows_normal_outliers(43, 0, 64, HIDDEN, torch.bfloat16).to(dev)  # rows are seed-keyed
        ones = {
            "rmsnorm": (torch.cat([bi.bi_rmsnorm(x64[i:i + 1], g, EPS) for i in range(64)]),
                        torch.cat([F.rms_norm(x64[i:i + 1], (HIDDEN,), g, EPS) for i in range(64)])),
            "mean": (torch.cat([bi.bi_mean(x64[i:i + 1].float()) for i in range(64)])[:, None],
                     torch.cat([x64[i:i + 1].float().mean(-1) for i in range(64)])[:, None]),
        }
        for M in [1, 8, 64, 148, 256, 1024, 4096, 8192, 16384, 3, 77, 1000]:
            if ("rows", "rmsnorm", M) in have and ("rows", "mean", M) in have:
                continue
            x = inputs.rows_normal_outliers(43, 0, M, HIDDEN, torch.bfloat16).to(dev)
            xf = x.float()
            y = torch.empty_like(x)
            ym = torch.empty(M, dtype=torch.float32, device=dev)
            n = min(M, 64)
            for op, fn, tfn, by in (
                ("rmsnorm", lambda: bi.bi_rmsnorm(x, g, EPS, out=y),
                 lambda: F.rms_norm(x, (HIDDEN,), g, EPS), 4 * HIDDEN * M),
                ("mean", lambda: bi.bi_mean(xf, out=ym), lambda: xf.mean(-1), (4 * HIDDEN + 4) * M)):
                t_bi = _timed(fn, flush, reps)
                bi_out = (y if op == "rmsnorm" else ym[:, None])
                bi_diff = _rows_differing(bi_out, ones[op][0][:n])
                t_t = _timed(tfn, flush, reps)
                t_out = tfn()
                t_diff = _rows_differing(t_out if op == "rmsnorm" else t_out[:, None], ones[op][1][:n])
                row_rec(op, M, t_bi, by, t_t, bi_diff, t_diff, n)
        xv64 = inputs.rows_normal(44, 0, 64, VOCAB, std=1.3).to(dev)
        one_v = {"log_softmax": torch.cat([bi.bi_log_softmax(xv64[i:i + 1]) for i in range(64)]),
                 "log_softmax_cluster": torch.cat([bi.bi_log_softmax_cluster(xv64[i:i + 1]) for i in range(64)]),
                 "log_softmax_split": torch.cat([bi.bi_log_softmax_split(xv64[i:i + 1]) for i in range(64)]),
                 "torch": torch.cat([torch.log_softmax(xv64[i:i + 1], -1, dtype=torch.float32) for i in range(64)])}
        lp64 = one_v["log_softmax"]  # the step's mean runs over log-probs
        one_m = (torch.cat([bi.bi_mean(lp64[i:i + 1]) for i in range(64)])[:, None],
                 torch.cat([lp64[i:i + 1].mean(-1) for i in range(64)])[:, None])
        for M in [1, 8, 64, 256, 1024]:
            ops_v = ("log_softmax", "log_softmax_cluster", "log_softmax_split", "mean_vocab")
            if all(("rows", op, M) in have for op in ops_v):
                continue
            x = inputs.rows_normal(44, 0, M, VOCAB, std=1.3).to(dev)
            y = torch.empty(M, VOCAB, dtype=torch.float32, device=dev)
            by = 6 * VOCAB * M
            n = min(M, 64)
            t_t = _timed(lambda: torch.log_softmax(x, -1, dtype=torch.float32), flush, reps)
            t_diff = _rows_differing(torch.log_softmax(x, -1, dtype=torch.float32), one_v["torch"][:n])
            t_bi = _timed(lambda: bi.bi_log_softmax(x, out=y), flush, reps)
            row_rec("log_softmax", M, t_bi, by, t_t, _rows_differing(y, one_v["log_softmax"][:n]), t_diff, n)
            lp = y.clone()
            t_cl = _timed(lambda: bi.bi_log_softmax_cluster(x, out=y), flush, reps)
            row_rec("log_softmax_cluster", M, t_cl, by, t_t,
                    _rows_differing(y, one_v["log_softmax_cluster"][:n]), t_diff, n)
            scr = torch.empty(bi.bi_log_softmax_split_scratch_bytes(M, VOCAB), dtype=torch.uint8, device=dev)
            t_sp = _timed(lambda: bi.bi_log_softmax_split(x, scr, out=y), flush, reps)
            row_rec("log_softmax_split", M, t_sp, by, t_t, _rows_differing(y, one_v["log_softmax_split"][:n]),
                    t_diff, n)
            ym = torch.empty(M, dtype=torch.float32, device=dev)
            t_m = _timed(lambda: bi.bi_mean(lp, out=ym), flush, reps)
            t_mt = _timed(lambda: lp.mean(-1), flush, reps)
            row_rec("mean_vocab", M, t_m, (4 * VOCAB + 4) * M, t_mt, _rows_differing(ym[:, None], one_m[0][:n]),
                    _rows_differing(lp.mean(-1)[:, None], one_m[1][:n]), n)
            del x, y, lp
            torch.cuda.empty_cache()
    if args.sweep_shapes and "attention" in args.sweep_shapes.split(","):
        # decode attention, Qwen3-8B heads: bi_decode_attention against torch's SDPA (GQA), L2
        # flushed before every call; caches [B, L, 8, 128] (SDPA gets them as [B, 8, L, 128])
        Hq, Hkv, D = 32, 8, 128
        out.setdefault("attention", [])
        print(f"{'B':>4s} {'L':>6s} {'bi us':>9s} {'GB/s':>7s} {'%HBM':>6s} {'sdpa us':>9s}")
        for B, L in [(1, 1024), (8, 1024), (32, 2048), (64, 4096), (128, 2048)]:
            g = torch.Generator(device=dev)
            g.manual_seed(58)
            q = torch.randn(B, Hq, D, generator=g, device=dev).to(torch.bfloat16)
            k = torch.randn(B, L, Hkv, D, generator=g, device=dev).to(torch.bfloat16)
            v = torch.randn(B, L, Hkv, D, generator=g, device=dev).to(torch.bfloat16)
            sl = torch.full((B,), L, dtype=torch.int32, device=dev)
            scr = torch.empty(bi.bi_decode_attention_scratch_bytes(B, Hq, D, L), dtype=torch.uint8, device=dev)
            o = torch.empty_like(q)
            t_bi = _timed(lambda: bi.bi_decode_attention(q, k, v, sl, scratch=scr, out=o), flush, reps)
            qt, kt, vt = q.view(B, Hq, 1, D), k.permute(0, 2, 1, 3).contiguous(), v.permute(0, 2, 1, 3).contiguous()
            t_t = _timed(lambda: F.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True), flush, reps)
            by = 2 * B * L * Hkv * D * 2
            out["attention"].append({"B": B, "L": L, "bi_us": t_bi * 1e3, "bi_gbs": by / t_bi / 1e6,
                                     "bi_frac_hbm": by / t_bi / 1e6 / peaks["hbm_gbs"], "sdpa_us": t_t * 1e3})
            save()
            print(f"{B:4d} {L:6d} {t_bi*1e3:9.1f} {by/t_bi/1e6:7.0f} {100*by/t_bi/1e6/peaks['hbm_gbs']:5.1f}% "
                  f"{t_t*1e3:9.1f}", flush=True)
            del q, k, v, kt, vt, scr, o
            torch.cuda.empty_cache()
    save()


# ----------------------------------------------------------------------------- single-kernel cases

KERNEL_CASES = {
    # name: (description, bytes in + out) -- inputs larger than L2, a few hundred MB on the device
    "gemm_gate_up": "bi_matmul M=1024 K=4096 N=24576 (B [N, K])",
    "gemm_lm_head": "bi_matmul M=1024 K=4096 N=151936 (B [N, K])",
    "gemm_qo_m256": "bi_matmul M=256 K=4096 N=4096 (B [N, K])",
    "gemm_kv_m1": "bi_matmul M=1 K=4096 N=1024 (B [N, K])",
    "gemm_down_m64": "bi_matmul M=64 K=12288 N=4096 (B [N, K])",
    "gemm_gate_up_silu": "bi_matmul_silu_mul M=1024 K=4096 F=12288 (B [2F, K])",
    "rmsnorm": "bi_rmsnorm M=16384 H=4096 bf16",
    "mean": "bi_mean M=16384 H=4096 fp32",
    "mean_vocab": "bi_mean M=1024 H=151936 fp32 (the step's mean over log-probs)",
    "log_softmax": "bi_log_softmax M=1024 V=151936 bf16 -> fp32",
    "log_softmax_cluster": "bi_log_softmax_cluster M=1024 V=151936 bf16 -> fp32 (4 CTAs per row)",
    "silu_mul": "bi_silu_mul M=1024 F=12288",
    "decode_attention": "bi_decode_attention B=64 L=4096, 32 q / 8 kv heads of 128",
    "decode_attention_sdpa": "torch scaled_dot_product_attention on the decode_attention case's inputs "
                             "(a library reference for profiles; not batch-invariant)",
}


def run_kernel_case(args):
    """Launch one kernel `warmup + steps` times on a fixed case (for profiler captures);
    prints the mean device time of the timed launches."""
    import torch
    from invariant_bi_matmul_02_b200 import binding as bi
    from invariant_bi_matmul_02_b200 import inputs
    dev = torch.device("cuda", 0)
    name = args.kernel_case
    if name == "gemm_gate_up_silu":
        a = inputs.rows_normal(50, 0, 1024, HIDDEN).to(dev)
        w = inputs.weight_normal(51, (2 * FFN, HIDDEN)).to(dev)
        h = torch.empty(1024, FFN, dtype=torch.bfloat16, device=dev)
        fn = lambda: bi.bi_matmul_silu_mul(a, w, "nk", out=h)
        work, unit = 2 * 1024 * 2 * FFN * HIDDEN, "TFLOP/s"
    elif name.startswith("gemm"):
        M, K, N = {"gemm_gate_up": (1024, HIDDEN, 2 * FFN), "gemm_lm_head": (1024, HIDDEN, VOCAB),
                   "gemm_qo_m256": (256, HIDDEN, HIDDEN), "gemm_kv_m1": (1, HIDDEN, KV),
                   "gemm_down_m64": (64, FFN, HIDDEN)}[name]
        a = inputs.rows_normal(50, 0, M, K).to(dev)
        w = inputs.weight_normal(51, (N, K)).to(dev)
        c = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        fn = lambda: bi.bi_matmul(a, w, "nk", out=c)
        work, unit = 2 * M * N * K, "TFLOP/s"
    elif name in ("rmsnorm", "mean"):
        x = inputs.rows_normal_outliers(52, 0, 16384, HIDDEN, torch.bfloat16).to(dev)
        if name == "rmsnorm":
            g = inputs.gain(53, HIDDEN).to(dev)
            y = torch.empty_like(x)
            fn = lambda: bi.bi_rmsnorm(x, g, EPS, out=y)
            work = 4 * HIDDEN * 16384
        else:
            xf = x.float()
            y = torch.empty(16384, dtype=torch.float32, device=dev)
            fn = lambda: bi.bi_mean(xf, out=y)
            work = (4 * HIDDEN + 4) * 16384
        unit = "GB/s"
    elif name == "mean_vocab":
        xf = inputs.rows_normal(57, 0, 1024, VOCAB, dtype=torch.float32).to(dev)
        y = torch.empty(1024, dtype=torch.float32, device=dev)
        fn = lambda: bi.bi_mean(xf, out=y)
        work, unit = (4 * VOCAB + 4) * 1024, "GB/s"
    elif name == "log_softmax":
        x = inputs.rows_normal(54, 0, 1024, VOCAB, std=1.3).to(dev)
        y = torch.empty(1024, VOCAB, dtype=torch.float32, device=dev)
        fn = lambda: bi.bi_log_softmax(x, out=y)
        work, unit = 6 * VOCAB * 1024, "GB/s"
    elif name == "log_softmax_cluster":
        x = inputs.rows_normal(54, 0, 1024, VOCAB, std=1.3).to(dev)
        y = torch.empty(1024, VOCAB, dtype=torch.float32, device=dev)
        fn = lambda: bi.bi_log_softmax_cluster(x, out=y)
        work, unit = 6 * VOCAB * 1024, "GB/s"
    elif name == "silu_mul":
        gu = inputs.rows_normal(55, 0, 1024, 2 * FFN, std=2.0).to(dev)
        h = torch.empty(1024, FFN, dtype=torch.bfloat16, device=dev)
        fn = lambda: bi.bi_silu_mul(gu, out=h)
        work, unit = 6 * FFN * 1024, "GB/s"
    elif name in ("decode_attention", "decode_attention_sdpa"):
        B, L, Hq, Hkv, D = 64, 4096, 32, 8, 128
        g = torch.Generator(device=dev)
        g.manual_seed(56)
        q = torch.randn(B, Hq, D, generator=g, device=dev).to(torch.bfloat16)
        k = torch.randn(B, L, Hkv, D, generator=g, device=dev).to(torch.bfloat16)
        v = torch.randn(B, L, Hkv, D, generator=g, device=dev).to(torch.bfloat16)
        sl = torch.full((B,), L, dtype=torch.int32, device=dev)
        scr = torch.empty(bi.bi_decode_attention_scratch_bytes(B, Hq, D, L), dtype=torch.uint8, device=dev)
        o = torch.empty_like(q)
        fn = lambda: bi.bi_decode_attention(q, k, v, sl, scratch=scr, out=o)
        if name == "decode_attention_sdpa":
            import torch.nn.functional as F
            qs, ks, vs = q.view(B, Hq, 1, D), k.permute(0, 2, 1, 3), v.permute(0, 2, 1, 3)
            fn = lambda: F.scaled_dot_product_attention(qs, ks, vs, enable_gqa=True)
        work, unit = 2 * B * L * Hkv * D * 2, "GB/s"
    else:
        raise SystemExit(f"unknown kernel case {name}; choose from {sorted(KERNEL_CASES)}")
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / args.steps
    rate = work / (ms / 1e3) / (1e12 if unit == "TFLOP/s" else 1e9)
    print(json.dumps({"kernel_case": name, "what": KERNEL_CASES[name], "launches": args.warmup + args.steps,
                      "mean_ms": ms, "rate": rate, "unit": unit,
                      "status": bi.bi_get_device_status()}), flush=True)


# ----------------------------------------------------------------------------- uniqueness experiment

class ToyDecoder:
    """A random-weight decoder (Qwen-style blocks without position encoding) used to repeat the
    pages' experiment in miniature: greedy decoding of one prompt inside many different batch
    compositions.  `impl` "bi" runs every reduction through libbi.so; "torch" uses torch's
    default kernels for the same arithmetic."""

    HIDDEN, HQ, HKV, HEAD, FFN_T, VOC, LAYERS = 1024, 8, 2, 128, 2816, 32000, 4

    def __init__(self, device, seed: int = 900):
        import torch
        from invariant_bi_matmul_02_b200 import inputs
        H, F = self.HIDDEN, self.FFN_T
        w = lambda i, shape, std=0.02: inputs.weight_normal(seed + i, shape, std=std).to(device)
        self.emb = w(0, (self.VOC, H), std=1.0)
        self.layers = []
        for l in range(self.LAYERS):
            b = 10 * (l + 1)
            self.layers.append(dict(
                g1=inputs.gain(seed + b, H).to(device), g2=inputs.gain(seed + b + 1, H).to(device),
                wq=w(b + 2, (self.HQ * self.HEAD, H)), wk=w(b + 3, (self.HKV * self.HEAD, H)),
                wv=w(b + 4, (self.HKV * self.HEAD, H)), wo=w(b + 5, (H, self.HQ * self.HEAD)),
                wgu=w(b + 6, (2 * F, H)), wd=w(b + 7, (H, F))))
        self.gf = inputs.gain(seed + 99, H).to(device)
        self.wlm = w(98, (self.VOC, H))
        self.device = device

    def step(self, impl, tokens, kcache, vcache, pos):
        """One decode step for a batch: tokens [B] -> next tokens [B]; writes position `pos`
        of every sequence's cache and attends over positions 0..pos."""
        import torch
        import torch.nn.functional as Fn
        from invariant_bi_matmul_02_b200 import binding as bi
        B = tokens.shape[0]
        x = self.emb.index_select(0, tokens)
        lens = torch.full((B,), pos + 1, dtype=torch.int32, device=self.device)
        for l, L in enumerate(self.layers):
            if impl == "bi":
                h = bi.bi_rmsnorm(x, L["g1"], EPS)
                q, k, v = (bi.bi_matmul(h, L["wq"]), bi.bi_matmul(h, L["wk"]), bi.bi_matmul(h, L["wv"]))
            else:
                h = Fn.rms_norm(x, (self.HIDDEN,), L["g1"], EPS)
                q, k, v = Fn.linear(h, L["wq"]), Fn.linear(h, L["wk"]), Fn.linear(h, L["wv"])
            kcache[l][:, pos] = k.view(B, self.HKV, self.HEAD)
            vcache[l][:, pos] = v.view(B, self.HKV, self.HEAD)
            if impl == "bi":
                a = bi.bi_decode_attention(q.view(B, self.HQ, self.HEAD), kcache[l], vcache[l], lens)
                x = bi.bi_addmm(x, a.view(B, -1), L["wo"])
                m = bi.bi_matmul_silu_mul(bi.bi_rmsnorm(x, L["g2"], EPS), L["wgu"])
                x = bi.bi_addmm(x, m, L["wd"])
            else:
                kk = kcache[l][:, :pos + 1].transpose(1, 2)
                vv = vcache[l][:, :pos + 1].transpose(1, 2)
                a = Fn.scaled_dot_product_attention(q.view(B, self.HQ, 1, self.HEAD), kk, vv, enable_gqa=True)
                x = x + Fn.linear(a.reshape(B, -1), L["wo"])
                gu = Fn.linear(Fn.rms_norm(x, (self.HIDDEN,), L["g2"], EPS), L["wgu"])
                g_, u_ = gu.chunk(2, dim=-1)
                x = x + Fn.linear(Fn.silu(g_) * u_, L["wd"])
        if impl == "bi":
            lp = bi.bi_log_softmax(bi.bi_matmul(bi.bi_rmsnorm(x, self.gf, EPS), self.wlm))
        else:
            lp = torch.log_softmax(Fn.linear(Fn.rms_norm(x, (self.HIDDEN,), self.gf, EPS), self.wlm), -1,
                                   dtype=torch.float32)
        return lp.argmax(-1), lp

    def generate(self, impl, prompts, new_tokens, watch=None, digest=None, context=0, context_seeds=None):
        """Greedy decoding of a batch of equal-length prompts [B, P]: returns [B, new_tokens].
        With `context` > 0 every sequence starts from `context` cached positions of random keys
        and values (N(0, 1), drawn on the device from the sequence's seed in `context_seeds`).
        With `watch` (a row index) and `digest` (a hashlib object), the bits of that row's
        log-prob vector at every step are fed to the digest."""
        import torch
        B, P = prompts.shape
        T = context + P + new_tokens
        kc = [torch.zeros(B, T, self.HKV, self.HEAD, dtype=torch.bfloat16, device=self.device)
              for _ in range(self.LAYERS)]
        vc = [torch.zeros_like(kc[0]) for _ in range(self.LAYERS)]
        for b in range(B if context else 0):
            g = torch.Generator(device=self.device)
            g.manual_seed(int(context_seeds[b]))
            for l in range(self.LAYERS):
                for cache in (kc[l], vc[l]):
                    cache[b, :context] = torch.randn(context, self.HKV, self.HEAD, generator=g,
                                                     device=self.device).to(torch.bfloat16)

        def step(tok, pos):
            nxt, lp = self.step(impl, tok, kc, vc, pos)
            if digest is not None:
                digest.update(lp[watch].contiguous().view(torch.int32).cpu().numpy().tobytes())
            return nxt

        out = []
        tok = prompts[:, 0]
        for i in range(P + new_tokens - 1):
            pos = context + i
            nxt = step(tok, pos)
            if i + 1 < P:
                tok = prompts[:, i + 1]
            else:
                out.append(nxt)
                tok = nxt
        out.append(step(tok, T - 1))
        return torch.stack(out, 1)[:, -new_tokens:]


def uniqueness(trials: int, new_tokens: int = 32, prompt_len: int = 16, max_batch: int = 64, seed: int = 950,
               device="cuda", context: int = 0):
    """Decode one fixed prompt greedily inside `trials` random batch compositions (random batch
    size 1..max_batch, random position, random other prompts) with each implementation, and
    count the distinct completions of the fixed prompt and the distinct bit patterns of its
    log-prob vectors over all steps."""
    import hashlib
    import torch
    from invariant_bi_matmul_02_b200 import inputs
    model = ToyDecoder(device)
    g = torch.Generator().manual_seed(seed)
    target = torch.randint(0, ToyDecoder.VOC, (prompt_len,), generator=g)
    sizes = inputs.batch_sizes(seed, trials, 1, max_batch)
    result = {}
    for impl in ("bi", "torch"):
        seen, bits = {}, set()
        for t, b in enumerate(sizes):
            gt = torch.Generator().manual_seed(seed * 1000 + t)
            others = torch.randint(0, ToyDecoder.VOC, (b, prompt_len), generator=gt)
            at = int(torch.randint(0, b, (1,), generator=gt))
            others[at] = target
            ctx_seeds = torch.randint(1, 2 ** 31 - 1, (b,), generator=gt)
            ctx_seeds[at] = seed  # the fixed prompt always sees the same context
            h = hashlib.sha256()
            comp = model.generate(impl, others.to(device), new_tokens, watch=at, digest=h, context=context,
                                  context_seeds=ctx_seeds)[at].tolist()
            key = tuple(comp)
            seen[key] = seen.get(key, 0) + 1
            bits.add(h.hexdigest())
        result[impl] = {"unique": len(seen), "most_common": max(seen.values()),
                        "unique_logprob_bits": len(bits), "trials": trials}
    return result


def run_uniqueness(args):
    import torch
    t0 = time.perf_counter()
    res = uniqueness(args.uniqueness, context=args.context)
    print(json.dumps({"experiment": "greedy completions of one prompt over random batch compositions",
                      "context_tokens": args.context,
                      "model": "random-weight 4-layer decoder, hidden 1024, 8 q / 2 kv heads of 128, "
                               "ffn 2816, vocab 32000",
                      "new_tokens": 32, "prompt_len": 16, "batch_sizes": "1..64",
                      "bi": res["bi"], "torch_default": res["torch"],
                      "seconds": round(time.perf_counter() - t0, 1),
                      "status": __import__("invariant_bi_matmul_02_b200").bi_get_device_status()}),
          flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--rows", type=int, default=1024, help="token rows per GPU per step")
    ap.add_argument("--impl", choices=["bi", "reference"], default="bi")
    ap.add_argument("--mlp", choices=["fused", "unfused"], default="fused",
                    help="gate/up + SiLU*up as one fused GEMM (default) or GEMM then bi_silu_mul")
    ap.add_argument("--cpu-budget", type=float, default=25.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mma-probe", action="store_true",
                    help="cycles per tcgen05.mma for several instruction shapes")
    ap.add_argument("--host-overhead", action="store_true",
                    help="host time per small GEMM call with and without tensor-map cache hits")
    ap.add_argument("--no-metric-sweep", action="store_true",
                    help="leave out the per-kernel M sweep that the JSON line carries at N=1")
    ap.add_argument("--sweep", action="store_true", help="per-kernel M sweeps (table, not JSON line)")
    ap.add_argument("--sweep-shapes", default="",
                    help="comma list of sweep groups (q/o,k/v,gate/up,down,lm_head,rows; attention only when named)")
    ap.add_argument("--sweep-out", default="", help="write the sweep as JSON to this path (after every point)")
    ap.add_argument("--resume", action="store_true", help="with --sweep-out: skip the points already there")
    ap.add_argument("--uniqueness", type=int, default=0,
                    help="run the batch-composition uniqueness experiment with this many trials")
    ap.add_argument("--context", type=int, default=4096,
                    help="cached context positions per sequence in the uniqueness experiment")
    ap.add_argument("--kernel-case", default="", help="launch one kernel on a fixed case: "
                    + ", ".join(sorted(KERNEL_CASES)))
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.sweep:
        run_sweep(args)
        return
    if args.kernel_case:
        run_kernel_case(args)
        return
    if args.host_overhead:
        run_host_overhead(args)
        return
    if args.mma_probe:
        run_mma_probe(args)
        return
    if args.uniqueness:
        run_uniqueness(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_bi(args)


if __name__ == "__main__":
    main()
