"""Benchmark of the quantized linear layer on B200.

Workload (the headline): dense decode W8A8 int8 g128 in the Hadamard domain,
N = 21504, K = 5376, tokens M in {1, 4, 8, 16}.  One step = the whole hot path
once per M: rotate + quantise the activations, then the skinny GEMM over the
packed weight.  Metric: decode qGEMV HBM GB/s, counted from the algorithmic
bytes (packed codes + scales + bf16 x read + fp32 y written).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]

Timing: W eager warm-up steps, then the K timed steps replayed from a CUDA
graph, bracketed by a barrier and device synchronisation, measured with CUDA
events on the launching stream; max over ranks.  Four packed copies of the
weight (470 MB, more than the 126 MB L2) rotate between the forward calls, so
no call finds its weight in L2.  The timed graph holds only the library's
kernels; the per-kernel durations for the roofline come from one more replay
of the same steps with the library's launch trace (CUDA events around each of
its kernels, on the launching stream) captured into the graph.
Multi-GPU: replicas only -- the layer does not shard in this workload, every
rank runs the same step on its own GPU and value sums the ranks' bytes.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import re
import subprocess
import sys
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

N_FULL, K_FULL = 21504, 5376
MS = (1, 4, 8, 16)
COPIES = 4
METRIC = "decode qGEMV HBM GB/s (% of peak); prefill qGEMM TOPS (% of int8/fp8 peak)"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-extras", action="store_true", help="skip the secondary workloads")
    p.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    p.add_argument("--extras", default=None,
                   help="comma-separated extras sections to run (decode, moe_decode, moe_prefill, moe_fp8a8_down, "
                        "prefill); default all")
    p.add_argument("--extras-only", action="store_true",
                   help="run only the extras and print them as one JSON line (the main run starts this as a "
                        "child process, so a fault in a secondary workload cannot take the headline line with it)")
    p.add_argument("--ncu-case", choices=["skinny_w8a8", "prefill_w8a8", "prefill_fp8", "prefill_fp8a8", "prefill_w5a8",
                                          "moe_decode", "moe_decode_t1", "moe_prefill", "act_quant", "decode_w4a16",
                                          "decode_w5a16", "decode_w8a16", "decode_fp8", "moe_down"],
                   default=None,
                   help="run only a small fixed case for an ncu capture (2 warm-up + 2 profiled launches)")
    return p.parse_args()


def step_bytes():
    """Algorithmic bytes of one step: per M, codes + scales + x (bf16) + y (fp32)."""
    G = K_FULL // 128
    w = N_FULL * K_FULL + N_FULL * G * 2
    return sum(w + m * K_FULL * 2 + m * N_FULL * 4 for m in MS)


def skinny_bytes(m):
    """Algorithmic bytes of one skinny-GEMM launch: codes + scales + int8 x + fp32 x scales + fp32 y."""
    G = K_FULL // 128
    return N_FULL * K_FULL + N_FULL * G * 2 + m * K_FULL + m * G * 4 + m * N_FULL * 4


def replicas_time(ms_local: float, world: int, device) -> float:
    """The job's time for a replicated step: the slowest rank's (max over ranks)."""
    if world <= 1:
        return ms_local
    import torch
    import torch.distributed as dist

    t = torch.tensor([ms_local], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replicas_value(ms_job: float, world: int, steps: int, bytes_per_step: int) -> float:
    """Whole-job GB/s of N replicas: every rank moved bytes_per_step per step."""
    return world * steps * bytes_per_step / (ms_job * 1e-3) / 1e9


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


def kernel_traffic(name: str, src: Path):
    """Per-launch DRAM bytes of a kernel from its committed ncu summary, if the
    summary was taken on the current source (matching sha256 of the .cu file)."""
    md = ROOT / "profiles" / f"{name}.md"
    if not md.exists():
        return None
    text = md.read_text()
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_tr:
        return None
    if hashlib.sha256(src.read_bytes()).hexdigest() != m_sha.group(1):
        return None
    return float(m_tr.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [r.split(",") for r in (self.out or "").strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i] and "Not" not in r[5 + i]})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------
# CPU oracle arm
# --------------------------------------------------------------------------
def oracle_sample(rows: int):
    """Inputs of a bounded sample of the workload: the first `rows` weight rows,
    quantised by the oracle, and the activations of each M."""
    from moe_hadamard128_act_b200 import synth
    from oracle import oracle as O

    W = synth.weight_rows(0, "W", K_FULL, 0, rows)
    q, s = O.quant_i8_g128(W, hadamard=True)
    xs = {m: synth.activations(0, f"x_M{m}", m, K_FULL, outlier_frac=0.01) for m in MS}
    return q.view(np.uint8), s, xs


def oracle_step(q, s, xs, rows):
    from oracle import oracle as O

    t0 = time.perf_counter()
    for m in MS:
        O.forward(xs[m], q, s, None, O.I8A8_G128_BF16, O.HADAMARD, rows)
    return time.perf_counter() - t0


def sample_bytes(rows):
    G = K_FULL // 128
    return sum(rows * (K_FULL + G * 2) + m * K_FULL * 2 + m * rows * 4 for m in MS)


def cpu_baseline(target_s: float = 10.0):
    """The oracle on the host cores: whole steps (or a row slice of one, when a
    step alone takes longer than target_s) repeated for about target_s."""
    rows = 512
    q, s, xs = oracle_sample(rows)
    t = oracle_step(q, s, xs, rows)
    rows = int(min(N_FULL, max(64, rows * target_s / max(t, 1e-3))))
    q, s, xs = oracle_sample(rows)
    reps, tot = 0, 0.0
    while tot < target_s or reps == 0:
        tot += oracle_step(q, s, xs, rows)
        reps += 1
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": reps * sample_bytes(rows) / tot / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 oracle (OpenMP over rows), W8A8 Hadamard forward of {rows} of {N_FULL} weight rows "
                      f"for M in {list(MS)}, repeated {reps}x, {tot:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    from oracle import oracle as O

    O.build()
    rows = 512
    q, s, xs = oracle_sample(rows)
    t = oracle_step(q, s, xs, rows)
    budget = 120.0 / max(1, args.steps + args.warmup)  # whole run within a few minutes
    rows = int(min(N_FULL, max(32, rows * budget / max(t, 1e-3))))
    q, s, xs = oracle_sample(rows)
    for _ in range(args.warmup):
        oracle_step(q, s, xs, rows)
    tot = sum(oracle_step(q, s, xs, rows) for _ in range(args.steps))
    value = args.steps * sample_bytes(rows) / tot / 1e9
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "dense decode W8A8 int8 g128 Hadamard, N=21504 K=5376, M in [1,4,8,16]",
                   "sample_rows": rows},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {rows} of {N_FULL} weight rows per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# --------------------------------------------------------------------------
# Secondary workloads (reported under "extras"; the headline is the W8A8 step)
# --------------------------------------------------------------------------
def _graph_call_us(torch, fn, stream, calls=64, reps=10):
    """Mean us per fn(i) call, fn(0 .. calls-1) captured once in a CUDA graph and
    replayed reps times on `stream` (CUDA events on that stream)."""
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(gr, stream=stream):
            for i in range(calls):
                fn(i)
        gr.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            gr.replay()
        e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) / (reps * calls) * 1e3


def _traced(Q, fn, iters, kind):
    """Run fn(i) iters times with the library trace on; mean ms of `kind` launches."""
    Q.ql_trace_enable(64 * iters)
    for i in range(iters):
        fn(i)
    tr = Q.ql_trace_read(64 * iters)
    Q.ql_trace_enable(0)
    ks = [t for k, t in tr if k == kind and t >= 0]
    return float(np.mean(ks)) if ks else None, len(tr) / iters


def _mark(torch, section, stream):
    """Synchronise after a section of the extras and say so on stderr, so that a device fault
    is reported against the section that raised it."""
    stream.synchronize()
    torch.cuda.synchronize()
    print(f"[bench] section done: {section}", file=sys.stderr, flush=True)


def run_extras(torch, Q, synth, dev, stream, hbm, sections=None):
    """The secondary workloads; `sections` (a set of names, None = all) limits which run:
    decode, moe_decode, moe_prefill, moe_fp8a8_down, prefill."""
    want = lambda name: sections is None or name in sections  # noqa: E731
    out = {}
    G = K_FULL // 128
    bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    with torch.cuda.stream(stream):
        if want("decode"):
            # weight-only decode: int4 g64, int5 + zero point g128, int8 g128 bf16, fp8 128x128; and
            # format 7 (the fp8 weight with E4M3 activations) on the same decode kernel.
            # "us" is the whole forward (activation prologue + decode GEMM) replayed from a
            # CUDA graph, the rate it gives is over the forward's bytes; "us_gemm" is the
            # traced decode kernel alone.
            Wd = None
            for name, fmt in (("w4a16_decode", Q.I4_G64_BF16), ("w5a16_decode", Q.I5Z_G128_F16),
                              ("w8a16_decode", Q.I8_G128_BF16), ("fp8_decode", Q.FP8_B128_BF16),
                              ("fp8a8_decode", Q.FP8A8_B128_BF16)):
                if fmt in (Q.I4_G64_BF16, Q.I5Z_G128_F16):
                    d = synth.w4a16(16) if fmt == Q.I4_G64_BF16 else synth.w5a16(16)
                    z = torch.from_numpy(d["zeros"]).to(dev) if "zeros" in d else None
                    c, s, zz = Q.qlinear_pack(fmt, N_FULL, K_FULL, codes=torch.from_numpy(d["codes"]).to(dev),
                                              scales=torch.from_numpy(d["scales"].view(np.int16)).to(dev), zeros=z)
                else:
                    if Wd is None:
                        Wd = torch.from_numpy(synth.weight_rows(0, "W", K_FULL, 0, N_FULL)).to(dev)
                    c, s, zz = Q.qlinear_pack(fmt, N_FULL, K_FULL, W=Wd)
                cp = [(c, s, zz)] + [(c.clone(), s.clone(), None if zz is None else zz.clone()) for _ in range(3)]
                res = {}
                # above 16 rows int4 (and int5 up to 64) has no tensor-core prefill path: the decode
                # kernel runs once per 16 rows, streaming the weight again each time
                ms = {Q.I4_G64_BF16: (1, 5, 16, 64, 256), Q.I5Z_G128_F16: (1, 4, 16, 64)}.get(fmt, (1, 4, 16))
                for m in ms:
                    x = bf(synth.activations(0, f"x_M{m}", m, K_FULL))
                    y = torch.empty((m, N_FULL), dtype=torch.float32, device=dev)
                    ws = torch.empty(Q.qlinear_workspace_size(fmt, 0, m, N_FULL, K_FULL), dtype=torch.uint8, device=dev)
                    run = lambda i: Q.qlinear_forward(x, cp[i % 4][0], cp[i % 4][1], cp[i % 4][2], fmt, N_FULL,  # noqa
                                                      y=y, ws=ws, stream=stream)
                    for i in range(8):
                        run(i)
                    t, per = _traced(Q, run, 40, "skinny")
                    us = _graph_call_us(torch, run, stream)
                    cb, sb, zb = Q.qlinear_packed_sizes(fmt, N_FULL, K_FULL)
                    byts = cb + sb + zb + m * K_FULL * 2 + m * N_FULL * 4
                    res[str(m)] = {"us": us, "GB/s": byts / (us * 1e-6) / 1e9, "frac": byts / (us * 1e-6) / 1e9 / hbm,
                                   "us_gemm": 1e3 * t, "launches_per_call": per}
                    if m > 16:
                        res[str(m)]["TFLOPS"] = 2.0 * m * N_FULL * K_FULL / (us * 1e-6) / 1e12
                out[name] = res
                del cp, c, s, zz
            del Wd
            _mark(torch, "decode", stream)
        if want("moe_decode") or want("moe_prefill"):
            # MoE gate_up, int8 Hadamard-domain experts, decode batches
            E, topk, Ke, Ne = 128, 8, 2816, 1408
            Ws = synth.moe_gate_up(1, experts=range(E))["W"]
            codes = torch.empty((E, Ne, Ke), dtype=torch.int8, device=dev)
            scales = torch.empty((E, Ne, Ke // 128), dtype=torch.int16, device=dev)
            for e in range(E):
                c, s, _ = Q.qlinear_pack(Q.I8_G128_BF16, Ne, Ke, W=torch.from_numpy(Ws[e]).to(dev), flags=Q.HADAMARD)
                codes[e] = c.view(torch.int8).reshape(Ne, Ke)
                scales[e] = s.view(torch.int16).reshape(Ne, Ke // 128)
            del Ws
        if want("moe_decode"):
            res = {}
            for T in (1, 8, 16):
                batches = []
                for b in range(8):
                    ids, w = synth.routing(100 + b, T, E, topk)
                    batches.append((bf(synth.activations(b, f"x_T{T}", T, Ke)), torch.from_numpy(ids).to(dev),
                                    len(set(ids.ravel().tolist()))))
                y = torch.empty((T, topk, Ne), dtype=torch.float32, device=dev)
                wsm = torch.empty(Q.moe_workspace_size(E, Ne, Ke, Q.I8_G128_BF16, Q.HADAMARD, T, topk), dtype=torch.uint8,
                                  device=dev)
                run = lambda i: Q.moe_gate_up(batches[i % 8][0], batches[i % 8][1], codes, scales, E, Ne, y=y,  # noqa
                                              ws=wsm, stream=stream)
                for i in range(8):
                    run(i)
                t, per = _traced(Q, run, 40, "moe_gemm")
                us_call = _graph_call_us(torch, run, stream)
                touched = float(np.mean([b[2] for b in batches]))
                byts = touched * (Ne * Ke + Ne * (Ke // 128) * 2) + T * Ke * 2 + T * topk * Ne * 4
                res[str(T)] = {"us_gemm": 1e3 * t, "touched_experts": touched, "GB/s": byts / (t * 1e-3) / 1e9,
                               "frac": byts / (t * 1e-3) / 1e9 / hbm, "launches_per_call": per,
                               "us_call_graph": us_call, "GB/s_call": byts / (us_call * 1e-6) / 1e9}
            out["moe_gate_up_decode"] = res
            _mark(torch, "moe_decode", stream)
        if want("moe_prefill"):
            # the same experts at prefill size, T = 2048 (every expert touched)
            T = 2048
            ids, _ = synth.routing(200, T, E, topk)
            xT = bf(synth.activations(0, "x_T2048", T, Ke))
            idsT = torch.from_numpy(ids).to(dev)
            yT = torch.empty((T, topk, Ne), dtype=torch.float32, device=dev)
            wsT = torch.empty(Q.moe_workspace_size(E, Ne, Ke, Q.I8_G128_BF16, Q.HADAMARD, T, topk), dtype=torch.uint8,
                              device=dev)
            run = lambda i: Q.moe_gate_up(xT, idsT, codes, scales, E, Ne, y=yT, ws=wsT, stream=stream)  # noqa: E731
            for i in range(2):
                run(i)
            t, per = _traced(Q, run, 5, "moe_gemm")
            us_call = _graph_call_us(torch, run, stream, calls=8, reps=3)
            touched = len(set(ids.ravel().tolist()))
            byts = touched * (Ne * Ke + Ne * (Ke // 128) * 2) + T * Ke * 2 + T * topk * Ne * 4
            flops = 2.0 * T * topk * Ne * Ke
            bf16_peak = peaks()[1]
            t_roof = max(byts / (hbm * 1e9), flops / (bf16_peak * 1e12))
            out["moe_gate_up_prefill"] = {"T": T, "us_gemm": 1e3 * t, "touched_experts": touched, "GB/s": byts / (t * 1e-3) / 1e9,
                                          "TFLOPS": flops / (t * 1e-3) / 1e12, "roofline_us": 1e6 * t_roof,
                                          "frac": 1e6 * t_roof / (1e3 * t), "launches_per_call": per,
                                          "us_call_graph": us_call,
                                          "roofline": "max(bytes / measured HBM, flops / measured bf16 peak)"}
            _mark(torch, "moe_prefill", stream)
        if want("moe_decode") or want("moe_prefill"):
            del codes, scales
        if want("moe_fp8a8_down"):
            out.update(moe_extras(torch, Q, synth, dev, stream, hbm))
            _mark(torch, "moe_fp8a8_down", stream)
        if want("prefill"):
            # prefill W8A8 at M = 2048 (tcgen05 kind::i8 GEMM with per-group fp32 promotion)
            M = 2048
            d = synth.prefill(M=M)
            c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N_FULL, K_FULL, W=torch.from_numpy(d["W"]).to(dev))
            x = bf(d["x"])
            y = torch.empty((M, N_FULL), dtype=torch.float32, device=dev)
            ws = torch.empty(Q.qlinear_workspace_size(Q.I8A8_G128_BF16, 0, M, N_FULL, K_FULL), dtype=torch.uint8,
                             device=dev)
            run = lambda i: Q.qlinear_forward(x, c, s, None, Q.I8A8_G128_BF16, N_FULL, y=y, ws=ws,  # noqa: E731
                                              stream=stream)
            for i in range(3):
                run(i)
            t, _ = _traced(Q, run, 10, "prefill")
            tq, _ = _traced(Q, run, 10, "act_quant")
            tp, _ = _traced(Q, run, 10, "prefill_prep")
            ops = 2.0 * M * N_FULL * K_FULL
            peak_i8 = 2.0 * peaks()[1]  # measured bf16 dense burst x the nominal int8 / bf16 ratio of 2
            out["prefill_w8a8"] = {"M": M, "us_gemm": 1e3 * t, "us_act_quant": 1e3 * tq, "us_scale_prep": 1e3 * tp, "TOPS": ops / (t * 1e-3) / 1e12,
                                   "peak_TOPS": peak_i8, "frac": ops / (t * 1e-3) / 1e12 / peak_i8,
                                   "peak_source": "MEASURED_PEAKS.json bf16_tflops x 2 (nominal int8/bf16 ratio)"}
            del c, s, y, ws
            # prefill with 16-bit activations: fp8 128x128 and int8 g128 bf16 weights (tcgen05 kind::f16)
            for name, fmt in (("prefill_fp8", Q.FP8_B128_BF16), ("prefill_w8a16", Q.I8_G128_BF16)):
                c, s, _ = Q.qlinear_pack(fmt, N_FULL, K_FULL, W=torch.from_numpy(d["W"]).to(dev))
                y = torch.empty((M, N_FULL), dtype=torch.float32, device=dev)
                ws = torch.empty(Q.qlinear_workspace_size(fmt, 0, M, N_FULL, K_FULL), dtype=torch.uint8, device=dev)
                run = lambda i: Q.qlinear_forward(x, c, s, None, fmt, N_FULL, y=y, ws=ws, stream=stream)  # noqa: E731
                for i in range(3):
                    run(i)
                t, _ = _traced(Q, run, 10, "prefill")
                tq, _ = _traced(Q, run, 10, "prep_a16")
                tf = ops / (t * 1e-3) / 1e12
                out[name] = {"M": M, "us_gemm": 1e3 * t, "us_prep_a16": 1e3 * tq, "TFLOPS": tf,
                             "frac_of_fp8_peak": tf / peak_i8, "frac_of_bf16_peak": tf / peaks()[1],
                             "peak_source": "MEASURED_PEAKS.json bf16_tflops (x 2 for fp8, nominal ratio)",
                             "mma": "kind::f16 (exact f16 codes x token-scaled f16 activations)"}
                del c, s, y, ws
            # format 7: the fp8 weights with E4M3 activations (tcgen05 kind::f8f6f4, fp8 rate)
            c, s, _ = Q.qlinear_pack(Q.FP8A8_B128_BF16, N_FULL, K_FULL, W=torch.from_numpy(d["W"]).to(dev))
            y = torch.empty((M, N_FULL), dtype=torch.float32, device=dev)
            ws = torch.empty(Q.qlinear_workspace_size(Q.FP8A8_B128_BF16, 0, M, N_FULL, K_FULL), dtype=torch.uint8,
                             device=dev)
            run = lambda i: Q.qlinear_forward(x, c, s, None, Q.FP8A8_B128_BF16, N_FULL, y=y, ws=ws,  # noqa: E731
                                              stream=stream)
            for i in range(3):
                run(i)
            t, _ = _traced(Q, run, 10, "prefill")
            tq, _ = _traced(Q, run, 10, "act_quant")
            tp, _ = _traced(Q, run, 10, "prefill_prep")
            tf = ops / (t * 1e-3) / 1e12
            out["prefill_fp8a8"] = {"M": M, "us_gemm": 1e3 * t, "us_act_quant": 1e3 * tq, "us_scale_prep": 1e3 * tp,
                                    "TFLOPS": tf, "frac_of_fp8_peak": tf / peak_i8,
                                    "peak_source": "MEASURED_PEAKS.json bf16_tflops x 2 (nominal fp8/bf16 ratio)",
                                    "mma": "kind::f8f6f4 (E4M3 x E4M3, fp32 group sums)"}
            del c, s, y, ws
            # int5 with a zero point from 65 rows on (W5A8): int8 activations, the codes converted to
            # int8 q - z in the workspace, the W8A8 tensor-core GEMM
            d5 = synth.w5a16(M)
            c, s, z = Q.qlinear_pack(Q.I5Z_G128_F16, N_FULL, K_FULL, codes=torch.from_numpy(d5["codes"]).to(dev),
                                     scales=torch.from_numpy(d5["scales"]).to(dev),
                                     zeros=torch.from_numpy(d5["zeros"]).to(dev))
            x5 = bf(d5["x"])
            y = torch.empty((M, N_FULL), dtype=torch.float32, device=dev)
            ws = torch.empty(Q.qlinear_workspace_size(Q.I5Z_G128_F16, 0, M, N_FULL, K_FULL), dtype=torch.uint8,
                             device=dev)
            run = lambda i: Q.qlinear_forward(x5, c, s, z, Q.I5Z_G128_F16, N_FULL, y=y, ws=ws,  # noqa: E731
                                              stream=stream)
            for i in range(3):
                run(i)
            t, _ = _traced(Q, run, 10, "prefill")
            tq, _ = _traced(Q, run, 10, "act_quant")
            tp, _ = _traced(Q, run, 10, "prefill_prep")
            out["prefill_w5a8"] = {"M": M, "us_gemm": 1e3 * t, "us_act_quant": 1e3 * tq,
                                   "us_scale_prep_and_code_conversion": 1e3 * tp, "TOPS": ops / (t * 1e-3) / 1e12,
                                   "frac": ops / (t * 1e-3) / 1e12 / peak_i8,
                                   "peak_source": "MEASURED_PEAKS.json bf16_tflops x 2 (nominal int8/bf16 ratio)"}
            del c, s, z, y, ws, d5
            _mark(torch, "prefill", stream)
    torch.cuda.synchronize()
    return out


def moe_extras(torch, Q, synth, dev, stream, hbm):
    """The fp8 experts with E4M3 activations (format 7) at the MoE workload's decode and prefill batch
    sizes, and the bf16 down projection with its routing-weighted combine: whole calls replayed from a
    CUDA graph, and the expert GEMM alone from the launch trace."""
    out = {}
    E, topk, Ke, Ne, I = 128, 8, 2816, 1408, 704
    bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    Ws = synth.moe_gate_up(1, experts=range(E))["W"]
    sb = (Ne + 127) // 128 * (Ke // 128)
    codes = torch.empty((E, Ne, Ke), dtype=torch.uint8, device=dev)
    scales = torch.empty((E, sb), dtype=torch.int16, device=dev)
    for e in range(E):
        c, s, _ = Q.qlinear_pack(Q.FP8A8_B128_BF16, Ne, Ke, W=torch.from_numpy(Ws[e]).to(dev), flags=Q.HADAMARD)
        codes[e] = c.reshape(Ne, Ke)
        scales[e] = s.view(torch.int16)
    del Ws
    res = {}
    for T in (1, 16, 2048):
        ids, _ = synth.routing(300 + T, T, E, topk)
        x = bf(synth.activations(0, f"x_T{T}", T, Ke))
        idt = torch.from_numpy(ids).to(dev)
        y = torch.empty((T, topk, Ne), dtype=torch.float32, device=dev)
        ws = torch.empty(Q.moe_workspace_size(E, Ne, Ke, Q.FP8A8_B128_BF16, Q.HADAMARD, T, topk), dtype=torch.uint8,
                         device=dev)
        run = lambda i: Q.moe_gate_up(x, idt, codes, scales, E, Ne, fmt=Q.FP8A8_B128_BF16,  # noqa: E731
                                      flags=Q.HADAMARD, y=y, ws=ws, stream=stream)
        for i in range(3):
            run(i)
        t, per = _traced(Q, run, 10, "moe_gemm")
        us_call = _graph_call_us(torch, run, stream, calls=16 if T == 2048 else 64, reps=3 if T == 2048 else 10)
        touched = len(set(ids.ravel().tolist()))
        byts = touched * (Ne * Ke + sb * 2) + T * Ke * 2 + T * topk * Ne * 4
        flops = 2.0 * T * topk * Ne * Ke
        r = {"us_gemm": 1e3 * t, "us_call_graph": us_call, "touched_experts": touched,
             "GB/s": byts / (t * 1e-3) / 1e9, "frac_hbm": byts / (t * 1e-3) / 1e9 / hbm, "launches_per_call": per}
        if T == 2048:
            r["TFLOPS"] = flops / (t * 1e-3) / 1e12
            r["frac_of_fp8_peak"] = r["TFLOPS"] / (2.0 * peaks()[1])
        res[str(T)] = r
    out["moe_gate_up_fp8a8"] = res
    del codes, scales
    # down projection: bf16 [128][2816][704] (507 MB), routing-weighted combine into [T, 2816]
    wd = torch.empty((E, Ke, I), dtype=torch.int16, device=dev)
    dd = synth.moe_down(1, experts=range(E))
    for e in range(E):
        wd[e] = torch.from_numpy(dd["Wd"][e].view(np.int16)).to(dev)
    del dd
    res = {}
    for T in (1, 16, 2048):
        d = synth.moe_down(T, experts=[])
        h = torch.from_numpy(d["h"]).to(dev)
        idt = torch.from_numpy(d["ids"]).to(dev)
        wt = torch.from_numpy(d["weights"]).to(dev)
        o = torch.empty((T, Ke), dtype=torch.float32, device=dev)
        ws = torch.empty(Q.moe_down_workspace_size(E, Ke, I, T, topk), dtype=torch.uint8, device=dev)
        run = lambda i: Q.moe_down_combine(h, idt, wt, wd, E, out=o, ws=ws, stream=stream)  # noqa: E731
        for i in range(3):
            run(i)
        t, per = _traced(Q, run, 10 if T < 2048 else 3, "moe_down")
        us_call = _graph_call_us(torch, run, stream, calls=16 if T == 2048 else 64, reps=2 if T == 2048 else 10)
        touched = len(set(d["ids"].ravel().tolist()))
        byts = touched * Ke * I * 2 + T * topk * 2 * I * 4 + T * Ke * 4
        flops = 2.0 * T * topk * Ke * I
        res[str(T)] = {"us_gemm": 1e3 * t, "us_call_graph": us_call, "touched_experts": touched,
                       "GB/s": byts / (t * 1e-3) / 1e9, "frac_hbm": byts / (t * 1e-3) / 1e9 / hbm,
                       "TFLOPS": flops / (t * 1e-3) / 1e12, "launches_per_call": per}
    out["moe_down_combine"] = res
    del wd
    torch.cuda.synchronize()
    return out


def ncu_case(name):
    """A small, fixed launch sequence for one ncu capture.
    skinny_w8a8: the W8A8 weight at full size (117 MB codes, two copies so each
    launch misses L2), M = 16, two warm-up forwards then two more; the skinny
    GEMM is launch 1..4 of its name.
    prefill_w8a8 / prefill_fp8 / prefill_fp8a8: the prefill workload (M = 2048,
    N = 21504, K = 5376; about 0.6 GB on the device), four forwards; the tcgen05
    GEMM (k_prefill_w8a8, which also runs format 7, / k_prefill_a16) is launch
    1..4 of its name.
    act_quant: the rotation + int8 quantiser on 16384 x 5376 bf16 (176 MB, more
    than L2), four calls.
    decode_w4a16 / decode_w5a16 / decode_w8a16 / decode_fp8: a weight-only
    decode forward at M = 1 on the full 21504 x 5376 weight of that format (two
    packed copies, alternating), four forwards; the decode GEMM is launch 1..4 of
    k_skinny_tma.
    prefill_w5a8: the int5 weight of the W5A16 workload with M = 2048 tokens
    (int8 activations), four forwards: act quant, scale prep, int5 -> int8 code
    conversion (k_prefill_i5_codes) and the W8A8 GEMM each launch four times.
    moe_decode / moe_decode_t1 / moe_prefill: the MoE gate_up experts (128 x
    [1408, 2816] int8 g128 bf16, Hadamard domain; about 0.5 GB), top-8 routing
    of T = 16 / 1 / 2048 tokens, four calls of moe_gate_up (activation
    prologue and expert GEMM; the permute too at T = 2048).
    moe_down: the bf16 down projection (128 x [2816, 704], 507 MB) with its
    routing-weighted combine for T = 2048 tokens, top-8, four calls of
    moe_down_combine (permute, activation planes, grouped tensor-core GEMM)."""
    import torch

    from moe_hadamard128_act_b200 import qlinear as Q
    from moe_hadamard128_act_b200 import synth

    dev = torch.device("cuda", 0)
    if name.startswith("decode_"):
        # a weight-only decode forward at M = 1 on the full 21504 x 5376 weight (two packed copies,
        # so no launch finds its weight in L2): two warm-up forwards, then two more
        fmt = {"decode_w4a16": Q.I4_G64_BF16, "decode_w5a16": Q.I5Z_G128_F16, "decode_w8a16": Q.I8_G128_BF16,
               "decode_fp8": Q.FP8_B128_BF16}[name]
        if fmt in (Q.I4_G64_BF16, Q.I5Z_G128_F16):
            d = synth.w4a16(1) if fmt == Q.I4_G64_BF16 else synth.w5a16(1)
            z = torch.from_numpy(d["zeros"]).to(dev) if "zeros" in d else None
            c, s, zz = Q.qlinear_pack(fmt, N_FULL, K_FULL, codes=torch.from_numpy(d["codes"]).to(dev),
                                      scales=torch.from_numpy(d["scales"].view(np.int16)).to(dev), zeros=z)
        else:
            W = torch.from_numpy(synth.weight_rows(0, "W", K_FULL, 0, N_FULL)).to(dev)
            c, s, zz = Q.qlinear_pack(fmt, N_FULL, K_FULL, W=W)
            del W
        cp = [(c, s, zz), (c.clone(), s.clone(), None if zz is None else zz.clone())]
        x = torch.from_numpy(synth.activations(0, "x_M1", 1, K_FULL).view(np.int16)).view(torch.bfloat16).to(dev)
        y = torch.empty((1, N_FULL), dtype=torch.float32, device=dev)
        for i in range(4):
            Q.qlinear_forward(x, cp[i % 2][0], cp[i % 2][1], cp[i % 2][2], fmt, N_FULL, y=y)
        torch.cuda.synchronize()
        st, bits = Q.ql_get_device_error()
        assert st == 0, bits
        print(f"ncu case {name} done")
        return
    if name == "act_quant":
        # the fused rotation + int8 quantiser on 16384 tokens of K = 5376 (176 MB of bf16 in, more
        # than L2), four calls
        M = 16384
        x = torch.from_numpy(synth.activations(0, "x_aq", M, K_FULL).view(np.int16)).view(torch.bfloat16).to(dev)
        for i in range(4):
            Q.act_quant_i8_g128(x, rotate=True)
        torch.cuda.synchronize()
        st, bits = Q.ql_get_device_error()
        assert st == 0, bits
        print(f"ncu case {name} done")
        return
    if name == "moe_down":
        E, topk, Ke, I, T = 128, 8, 2816, 704, 2048
        wd = torch.empty((E, Ke, I), dtype=torch.int16, device=dev)
        dd = synth.moe_down(1, experts=range(E))
        for e in range(E):
            wd[e] = torch.from_numpy(dd["Wd"][e].view(np.int16)).to(dev)
        del dd
        d = synth.moe_down(T, experts=[])
        h = torch.from_numpy(d["h"]).to(dev)
        idt = torch.from_numpy(d["ids"]).to(dev)
        wt = torch.from_numpy(d["weights"]).to(dev)
        o = torch.empty((T, Ke), dtype=torch.float32, device=dev)
        for i in range(4):
            Q.moe_down_combine(h, idt, wt, wd, E, out=o)
        torch.cuda.synchronize()
        st, bits = Q.ql_get_device_error()
        assert st == 0, bits
        print(f"ncu case {name} done")
        return
    if name.startswith("moe"):
        E, topk, Ke, Ne = 128, 8, 2816, 1408
        T = {"moe_decode": 16, "moe_decode_t1": 1}.get(name, 2048)
        Ws = synth.moe_gate_up(1, experts=range(E))["W"]
        codes = torch.empty((E, Ne, Ke), dtype=torch.int8, device=dev)
        scales = torch.empty((E, Ne, Ke // 128), dtype=torch.int16, device=dev)
        for e in range(E):
            c, s, _ = Q.qlinear_pack(Q.I8_G128_BF16, Ne, Ke, W=torch.from_numpy(Ws[e]).to(dev), flags=Q.HADAMARD)
            codes[e] = c.view(torch.int8).reshape(Ne, Ke)
            scales[e] = s.view(torch.int16).reshape(Ne, Ke // 128)
        del Ws
        ids, _ = synth.routing(200, T, E, topk)
        x = torch.from_numpy(synth.activations(0, f"x_T{T}", T, Ke).view(np.int16)).view(torch.bfloat16).to(dev)
        idt = torch.from_numpy(ids).to(dev)
        y = torch.empty((T, topk, Ne), dtype=torch.float32, device=dev)
        for i in range(4):
            Q.moe_gate_up(x, idt, codes, scales, E, Ne, y=y)
        torch.cuda.synchronize()
        st, bits = Q.ql_get_device_error()
        assert st == 0, bits
        print(f"ncu case {name} done")
        return
    if name == "prefill_w5a8":
        d = synth.w5a16(2048)
        c, s, z = Q.qlinear_pack(Q.I5Z_G128_F16, N_FULL, K_FULL, codes=torch.from_numpy(d["codes"]).to(dev),
                                 scales=torch.from_numpy(d["scales"]).to(dev), zeros=torch.from_numpy(d["zeros"]).to(dev))
        x = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16).to(dev)
        y = torch.empty((2048, N_FULL), dtype=torch.float32, device=dev)
        for i in range(4):
            Q.qlinear_forward(x, c, s, z, Q.I5Z_G128_F16, N_FULL, y=y)
        torch.cuda.synchronize()
        st, bits = Q.ql_get_device_error()
        assert st == 0, bits
        print(f"ncu case {name} done")
        return
    if name.startswith("prefill"):
        fmt = {"prefill_w8a8": Q.I8A8_G128_BF16, "prefill_fp8a8": Q.FP8A8_B128_BF16}.get(name, Q.FP8_B128_BF16)
        d = synth.prefill(M=2048)
        c, s, _ = Q.qlinear_pack(fmt, N_FULL, K_FULL, W=torch.from_numpy(d["W"]).to(dev))
        x = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16).to(dev)
        y = torch.empty((2048, N_FULL), dtype=torch.float32, device=dev)
        for i in range(4):
            Q.qlinear_forward(x, c, s, None, fmt, N_FULL, y=y)
        torch.cuda.synchronize()
        st, bits = Q.ql_get_device_error()
        assert st == 0, bits
        print(f"ncu case {name} done")
        return
    W = torch.from_numpy(synth.weight_rows(0, "W", K_FULL, 0, N_FULL)).to(dev)
    c, s, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N_FULL, K_FULL, W=W, flags=Q.HADAMARD)
    del W
    cp = [(c, s), (c.clone(), s.clone())]
    x = torch.from_numpy(synth.activations(0, "x_M16", 16, K_FULL, outlier_frac=0.01).view(np.int16)).view(
        torch.bfloat16).to(dev)
    y = torch.empty((16, N_FULL), dtype=torch.float32, device=dev)
    for i in range(4):
        Q.qlinear_forward(x, cp[i % 2][0], cp[i % 2][1], None, Q.I8A8_G128_BF16, N_FULL, flags=Q.HADAMARD, y=y)
    torch.cuda.synchronize()
    st, bits = Q.ql_get_device_error()
    assert st == 0, bits
    print(f"ncu case {name} done")


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------
def run_extras_child(args):
    """Runs `bench.py --extras-only` as a child process and returns its extras dict, or
    {"error": ...} when the child fails (its stderr, with the section markers, passes through)."""
    import subprocess
    cmd = [sys.executable, str(Path(__file__).resolve()), "--extras-only"]
    if args.extras is not None:
        cmd += ["--extras", args.extras]
    try:
        r = subprocess.run(cmd, stdout=subprocess.PIPE, stderr=None, text=True, timeout=1800)
    except subprocess.TimeoutExpired:
        return {"error": "extras child process timed out"}
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    if r.returncode != 0 or not lines:
        print(f"[bench] extras failed: child exit code {r.returncode}", file=sys.stderr, flush=True)
        return {"error": f"extras child process exited with code {r.returncode}"}
    return json.loads(lines[-1])


def extras_only(args):
    """The secondary workloads alone (one GPU), printed as one JSON line."""
    import torch

    from moe_hadamard128_act_b200 import build as qbuild
    from moe_hadamard128_act_b200 import qlinear as Q
    from moe_hadamard128_act_b200 import synth

    torch.cuda.set_device(0)
    qbuild.build()
    Q.lib()
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=dev)
    hbm = peaks()[0]
    sections = None if args.extras is None else set(args.extras.split(","))
    try:
        extras = run_extras(torch, Q, synth, dev, stream, hbm, sections)
    except Exception as ex:  # report what failed; the parent keeps its headline line either way
        extras = {"error": f"{type(ex).__name__}: {ex}"}
        print(f"[bench] extras failed: {extras['error']}", file=sys.stderr, flush=True)
    st, bits = Q.ql_get_device_error(stream)
    if st != 0 or bits:
        extras["device_error"] = {"status": st, "bits": bits}
    print(json.dumps(extras), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.ncu_case:
        return ncu_case(args.ncu_case)
    if args.extras_only:
        return extras_only(args)

    import torch
    import torch.distributed as dist

    from moe_hadamard128_act_b200 import build as qbuild
    from moe_hadamard128_act_b200 import qlinear as Q
    from moe_hadamard128_act_b200 import synth

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    if rank == 0:
        qbuild.build()
    if world > 1:
        dist.barrier()
    Q.lib()
    dev = torch.device("cuda", local)
    assert args.warmup >= 3, "at least 3 warm-up steps"

    # ---- inputs: the weight packed on the GPU from the seeded fp32 draw ----
    W = torch.from_numpy(synth.weight_rows(0, "W", K_FULL, 0, N_FULL)).to(dev)
    codes0, scales0, _ = Q.qlinear_pack(Q.I8A8_G128_BF16, N_FULL, K_FULL, W=W, flags=Q.HADAMARD)
    del W
    copies = [(codes0, scales0)] + [(codes0.clone(), scales0.clone()) for _ in range(COPIES - 1)]
    xs_host = {m: synth.activations(0, f"x_M{m}", m, K_FULL, outlier_frac=0.01) for m in MS}
    xs = {m: torch.from_numpy(xs_host[m].view(np.int16)).view(torch.bfloat16).to(dev) for m in MS}
    ys = {m: torch.empty((m, N_FULL), dtype=torch.float32, device=dev) for m in MS}
    ws = torch.empty(Q.qlinear_workspace_size(Q.I8A8_G128_BF16, Q.HADAMARD, 16, N_FULL, K_FULL), dtype=torch.uint8,
                     device=dev)
    L = Q.lib()
    stream = torch.cuda.Stream(device=dev)

    def forward_args(i, m, s):
        c, sc = copies[i % COPIES]
        return (ctypes.c_void_p(xs[m].data_ptr()), ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(sc.data_ptr()),
                None, Q.I8A8_G128_BF16, Q.HADAMARD, m, N_FULL, K_FULL, ctypes.c_void_p(ys[m].data_ptr()),
                ctypes.c_void_p(ws.data_ptr()), ws.numel(), ctypes.c_void_p(s.cuda_stream))

    calls = [forward_args(i, m, stream) for i, m in enumerate(MS)]

    def step():
        for a in calls:
            st = L.qlinear_forward(*a)
            if st:
                raise Q.QLError("qlinear_forward", st)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()

    # ---- timed region: a graph of S steps, replayed R times (no trace nodes) ----
    S = max(d for d in range(1, min(args.steps, 50) + 1) if args.steps % d == 0)
    R = args.steps // S
    launches_per_step = 2 * len(MS)

    def capture(trace: bool):
        if trace:
            Q.ql_trace_enable(S * launches_per_step)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(gr, stream=stream):
                for _ in range(S):
                    step()
            gr.replay()  # untimed graph warm-up, on the launching stream
        stream.synchronize()
        return gr

    g = capture(trace=False)
    # clocks pre-roll: about a second of the same load while nvidia-smi samples
    with ClockSampler(local) as clk, torch.cuda.stream(stream):  # every replay goes to `stream`
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < 1.0:
            g.replay()
            n += 1
            if n % 10 == 0:
                stream.synchronize()
        stream.synchronize()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(R):
            g.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    ms = replicas_time(ev0.elapsed_time(ev1), world, dev)
    value = replicas_value(ms, world, args.steps, step_bytes())

    # ---- roofline of the dominant kernel (the skinny GEMM), untraced: the same
    # GEMM launches on activations quantised beforehand (qlinear_gemm_a8, adding
    # into y), S steps of the four M captured in a graph and replayed on the
    # launching stream between CUDA events.  Launch gaps stay in the time, so
    # this is a lower bound of the kernel's own rate. ----
    hbm, bf16_tf, peak_src = peaks()
    qxs = {m: Q.act_quant_i8_g128(xs[m], rotate=True, stream=stream) for m in MS}
    stream.synchronize()
    gemm_calls = []
    for i in range(S * len(MS)):
        m = MS[i % len(MS)]
        c, sc = copies[i % COPIES]
        gemm_calls.append((ctypes.c_void_p(qxs[m][0].data_ptr()), ctypes.c_void_p(qxs[m][1].data_ptr()),
                           ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(sc.data_ptr()), Q.I8A8_G128_BF16, m,
                           N_FULL, K_FULL, ctypes.c_void_p(ys[m].data_ptr()), 1, ctypes.c_void_p(stream.cuda_stream)))

    def gemm_only():
        for a in gemm_calls:
            st = L.qlinear_gemm_a8(*a)
            if st:
                raise Q.QLError("qlinear_gemm_a8", st)

    gg = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(gg, stream=stream):
            gemm_only()
        gg.replay()
    stream.synchronize()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g0.record(stream)
        for _ in range(R):
            gg.replay()
        g1.record(stream)
    stream.synchronize()
    del gg
    gemm_ms_step = g0.elapsed_time(g1) / (R * S)  # four GEMM launches
    sk_bytes_step = float(sum(skinny_bytes(m) for m in MS))
    achieved = sk_bytes_step / (gemm_ms_step * 1e-3) / 1e9

    # ---- per-kernel durations for context: the same S steps replayed once more with
    # the library's launch trace (CUDA events around each of its kernels, recorded on
    # the launching stream) captured into the graph; the events split the programmatic
    # overlap of each forward's two kernels, so these durations run long ----
    gt = capture(trace=True)
    with torch.cuda.stream(stream):
        gt.replay()
    stream.synchronize()
    trace = Q.ql_trace_read(S * launches_per_step)
    Q.ql_trace_enable(0)
    del gt
    sk = [t for k, t in trace if k == "skinny" and t >= 0]
    traffic = kernel_traffic("skinny_w8a8_decode", ROOT / "moe_hadamard128_act_b200" / "csrc" / "k_skinny.cu")
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": traffic,
                "kernel": "k_skinny_tma<W8A8>", "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)",
                "timing": f"CUDA events around {R} replays of a graph of {S} x {len(MS)} GEMM-only launches "
                          "(qlinear_gemm_a8 on pre-quantised activations), launch gaps included",
                "gemm_us_per_step": 1e3 * gemm_ms_step, "gemm_share_of_step": gemm_ms_step / (ms / args.steps),
                "bytes_per_step": sk_bytes_step,
                "traced_us_per_m": {str(m): 1e3 * float(np.mean(sk[i::len(MS)])) for i, m in enumerate(MS)}}

    # ---- end to end through the C ABI with host buffers ----
    e2e_steps = min(args.steps, 200)
    xh = {m: torch.from_numpy(xs_host[m].view(np.int16)).view(torch.bfloat16).pin_memory() for m in MS}
    yh = {m: torch.empty((m, N_FULL), dtype=torch.float32).pin_memory() for m in MS}
    h2d = sum(m * K_FULL * 2 for m in MS)
    d2h = sum(m * N_FULL * 4 for m in MS)
    # Copies run on their own streams (uploads and downloads apart: the host link
    # is full duplex) and overlap the forwards, as an application would pipeline
    # them: x of forward j goes up ahead of it, y of forward j comes back while
    # forward j + 1 computes.  Events keep each device buffer's reuse in
    # order (the next upload of x[m] after its forward has read it, the next
    # forward into y[m] after its previous download).  The steps are captured as
    # a CUDA graph, as for the device-only number: every replayed step performs
    # all of its uploads, forwards (C-ABI calls) and downloads.
    cu = torch.cuda.Stream(device=dev)  # uploads
    cd = torch.cuda.Stream(device=dev)  # downloads
    x_up = {m: torch.cuda.Event() for m in MS}
    x_used = {m: torch.cuda.Event() for m in MS}
    y_done = {m: torch.cuda.Event() for m in MS}
    y_down = {m: torch.cuda.Event() for m in MS}

    def e2e_step(first):
        for j, m in enumerate(MS):
            with torch.cuda.stream(cu):
                if not first:
                    cu.wait_event(x_used[m])
                xs[m].copy_(xh[m], non_blocking=True)
                x_up[m].record(cu)
            with torch.cuda.stream(stream):
                stream.wait_event(x_up[m])
                if not first:
                    stream.wait_event(y_down[m])
                st = L.qlinear_forward(*calls[j])
                if st:
                    raise Q.QLError("qlinear_forward", st)
                x_used[m].record(stream)
                y_done[m].record(stream)
            with torch.cuda.stream(cd):
                cd.wait_event(y_done[m])
                yh[m].copy_(ys[m], non_blocking=True)
                y_down[m].record(cd)

    S_e = max(d for d in range(1, min(e2e_steps, 20) + 1) if e2e_steps % d == 0)
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(ge, stream=stream):
            cu.wait_stream(stream)
            cd.wait_stream(stream)
            for i in range(S_e):
                e2e_step(first=i == 0)
            stream.wait_stream(cu)
            stream.wait_stream(cd)
        ge.replay()  # untimed warm-up
    stream.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps // S_e):
            ge.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    del ge
    e2e_ms = replicas_time(e0.elapsed_time(e1), world, dev)
    e2e = {"value": replicas_value(e2e_ms, world, e2e_steps, step_bytes()), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps}

    st, bits = Q.ql_get_device_error(stream)
    if st != 0:
        raise RuntimeError(f"ql_get_device_error: status {st} ({Q.STATUS.get(st, st)}), bits {bits}, "
                           f"last CUDA error: {Q.lib().ql_last_cuda_error().decode()}")

    extras = None
    if not args.no_extras and world == 1:
        # The secondary workloads run in a child process with its own CUDA context, after this
        # one has released its buffers: whatever happens there, the headline line below stands.
        del copies, codes0, scales0
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        extras = run_extras_child(args)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline()

    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8 x int8 -> int32 (fp32 scales)", "data": "synthetic",
            "config": {"workload": "dense decode W8A8 int8 g128 Hadamard, N=21504 K=5376, M in [1,4,8,16]",
                       "parallelism": f"replicas x{world}", "l2": f"{COPIES} rotating weight copies (470 MB > L2)",
                       "graph_steps": S, "frac_of_hbm": value / world / hbm},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * launches_per_step,
            "clocks": clk.summary(),
            "extras": extras,
        }
        print(json.dumps(out), flush=True)
    del g
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
