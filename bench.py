"""Benchmark of the W4A4 quantized linear layer on B200.

One step = the five linears of one Llama-2-70B decoder layer (qkv 8192->10240,
o 8192->8192, w1/w3 8192->28672, w2 28672->8192) at M tokens, each a fused
W4A4 linear: per-token NVFP4 quantization of the bf16 activations followed by
the block-scaled NVFP4 GEMM against NVFP4 weights quantized once beforehand.
Metric: TFLOPS (2*M*N*K summed over the layer / time), whole job.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun) every rank runs its own replica on its own
tokens ("weak" scaling, no collective).  Also measured in the same run and
reported under "rows": the activation quantizer (GB/s), the small-M decode
variant (GB/s), the INT4-g128 path (Qwen2.5-7B shapes, TOPS), the residual
augmentation (Qwen2.5-3B shapes) and MXFP4.  `--impl reference` times the C
oracle on the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from w4a4_quantized_gemm_token_b200 import synth  # noqa: E402

LLAMA = synth.SHAPES["llama2_70b"]
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FP4_PER_BF16 = 4.0        # nominal dense FP4 / BF16 tensor throughput (9 / 2.25 PFLOP/s)
INT8_PER_BF16 = 2.0       # nominal dense INT8 / BF16 (4.5 / 2.25)
NOMINAL_FP4_TFLOPS = 9000.0  # B200 dense FP4, nominal
NOMINAL_INT8_TOPS = 4500.0   # B200 dense INT8, nominal
# FP4 MMA issue rate per SM: one 128x256x64 NVFP4 MMA (2 * 128 * 256 * 64 FLOP)
# every 128 cycles, measured back to back on one SM
MMA_FLOP_PER_CYCLE = 2 * 128 * 256 * 64 // 128


def mma_issue_peak_tflops(dev, sm_mhz: float) -> float:
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    return sms * MMA_FLOP_PER_CYCLE * sm_mhz * 1e6 / 1e12


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# dominant kernel, averaged over the five GEMM launches of one step, from an ncu
# capture of the pair GEMM on this workload; valid only for the kernel source it
# was measured on (else reported as null).
PROFILED_TRAFFIC = {"sources": ("gemm_fp4_pair.cu", "ptx.cuh"), "sha256_16": "1c98d42c0906a8c3",
                    "bytes_per_launch": 303.7e6}


def profiled_traffic():
    import hashlib
    h = hashlib.sha256()
    for f in PROFILED_TRAFFIC["sources"]:
        with open(os.path.join(ROOT, "w4a4_quantized_gemm_token_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return PROFILED_TRAFFIC["bytes_per_launch"] if h.hexdigest()[:16] == PROFILED_TRAFFIC["sha256_16"] else None


def peaks():
    try:
        p = json.load(open(PEAKS_FILE))
        return {"hbm": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
                "bf16_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "src": "measured",
                "sm_max_mhz": float(p.get("sm_max_mhz", 1965.0))}
    except Exception:
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "src": "fallback", "sm_max_mhz": 1965.0}


# ----------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0=None, t1=None, t2=None):
        """Samples taken in the timed region [t0, t1] (host clock); if it was
        too short to hold one, those of [t1, t2], a window right after it in
        which the same steps keep running untimed."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 10:
                rows.append(f)
        os.unlink(self.path)
        return summarize_clocks(rows, t0, t1, t2)


def _sample_time(stamp):
    import datetime
    try:
        return datetime.datetime.strptime(stamp, "%Y/%m/%d %H:%M:%S.%f").timestamp()
    except ValueError:
        return None


def summarize_clocks(rows, t0=None, t1=None, t2=None):
    """rows: nvidia-smi CSV fields in ClockSampler.QUERY order."""
    if not rows:
        return None
    window = "sampler run"
    if t0 is not None:
        ts = [_sample_time(r[0]) for r in rows]
        inside = [r for r, t in zip(rows, ts) if t is not None and t0 <= t <= t1]
        after = [r for r, t in zip(rows, ts) if t is not None and t1 < t <= t2]
        n_in = len(inside)
        if inside:
            rows, window = inside, "timed region"
        elif after:
            rows, window = after, "the same steps, untimed, right after the timed region (it was shorter than the sampling period)"
    sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
    mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
    out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
           "reasons": reasons, "samples": len(rows), "window": window}
    if t0 is not None:
        out["samples_in_timed_region"] = n_in
    return out


# ----------------------------------------------------------------------------------------------
# the reference arm and the CPU baseline: the oracle on a bounded sample
# ----------------------------------------------------------------------------------------------
_ORACLE_W = {}


def _oracle_weights(li, n):
    import oracle
    key = (li, n)
    if key not in _ORACLE_W:
        name, K, N = LLAMA[li]
        W = synth.weights("llama2_70b", N, K, seed=0, tensor_id=100 + li)[:n]
        _ORACLE_W[key] = oracle.quant_nvfp4(W, mode=0)
    return _ORACLE_W[key]


def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(M_rows: int, n_cols: int, threads: int = 1):
    """Time the C oracle (as it stands) on the layer's five linears for
    `M_rows` tokens and the first `n_cols` output columns of each: per-token
    NVFP4 quantization of those rows plus the exact block-scaled GEMM.  With
    threads > 1 the GEMM's output columns are split into `threads` contiguous
    parts computed at once (the oracle's C calls release the interpreter lock).
    The weights' quantization is offline on both arms and is not timed.
    Returns (TFLOPS, seconds, flops)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    oracle.build()
    t_total, flops = 0.0, 0.0
    pool = ThreadPoolExecutor(threads) if threads > 1 else None
    try:
        for li, (name, K, N) in enumerate(LLAMA):
            n = min(N, n_cols)
            cw, sw, s2w = _oracle_weights(li, n)
            X = synth.activations("llama2_70b", M_rows, K, seed=0, tensor_id=200 + li)
            t0 = time.perf_counter()
            ca, sa, s2a = oracle.quant_nvfp4(X, mode=1)
            if pool is None:
                oracle.gemm_nvfp4(ca, sa, s2a, 1, cw, sw, s2w, want_ref=False)
            else:
                cuts = [n * i // threads for i in range(threads + 1)]
                parts = [(cuts[i], cuts[i + 1]) for i in range(threads) if cuts[i + 1] > cuts[i]]
                list(pool.map(lambda r: oracle.gemm_nvfp4(ca, sa, s2a, 1, cw[r[0]:r[1]], sw[r[0]:r[1]], s2w,
                                                          want_ref=False), parts))
            t_total += time.perf_counter() - t0
            flops += 2.0 * M_rows * n * K
    finally:
        if pool is not None:
            pool.shutdown()
    return flops / t_total / 1e12, t_total, flops


def mxfp4_small_parity(Y_gpu_bits):
    """The MXFP4 16x256x256 workload (X ~ N(0,1), W ~ N(0,0.02), seed 0) by the
    oracle, compared with the GPU's output: every element within 1 bf16 ulp +
    1e-5 * sum|a w| of the exact product.  Returns (ok, oracle seconds)."""
    import oracle
    Xa = synth.activations("mxfp4_small", 16, 256, seed=0)
    Xw = synth.weights("mxfp4_small", 256, 256, seed=0)
    t0 = time.perf_counter()
    ca, sa = oracle.quant_mxfp4(Xa)
    cw, sw = oracle.quant_mxfp4(Xw)
    _, yref, absd = oracle.gemm_mxfp4(ca, sa, cw, sw)
    dt = time.perf_counter() - t0
    y = (np.asarray(Y_gpu_bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    a = np.abs(yref)
    ulp = np.exp2(np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), -126) - 7)
    ok = bool((np.abs(y - yref) <= ulp + 1e-5 * absd).all())
    return ok, dt


def run_reference(args, rank, world):
    if rank != 0:
        return
    K, W = args.steps, args.warmup
    rows, cols = args.ref_rows, args.ref_cols
    threads = host_threads()
    for _ in range(W):
        oracle_sample(1, cols, threads)
    vals, secs = [], []
    for _ in range(K):
        v, s, _ = oracle_sample(rows, cols, threads)
        vals.append(v)
        secs.append(s)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": "W4A4 linear TFLOPS (Llama-2-70B layer, NVFP4 per-token)",
        "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": statistics.median(secs) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": {"workload": f"llama2_70b layer linears (qkv,o,w1,w3,w2), oracle on {rows} tokens x "
                               f"{cols} output columns per linear per step", "tokens": rows},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} tokens x {cols} output columns of each of the 5 layer linears "
                                   f"(full K), GEMM columns split over {threads} host threads"},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------------------
def to_dev(bits, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def time_loop(fn, iters, stream, flush=None):
    """Average device time (ms) of fn() over iters launches, CUDA events on `stream`.

    With `flush` (a device buffer larger than L2) each launch is timed on its
    own between events, after the buffer has been read through, so inputs
    that would fit in L2 are read from HBM every time (reading leaves clean
    lines in L2: the timed kernel pays no write-back of the flush)."""
    import torch
    torch.cuda.synchronize()
    if flush is None:
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(iters):
            fn()
        e.record(stream)
        e.synchronize()
        return s.elapsed_time(e) / iters
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for (s, e) in evs:
        flush.max()
        s.record(stream)
        fn()
        e.record(stream)
    torch.cuda.synchronize()
    return sum(s.elapsed_time(e) for (s, e) in evs) / iters


def l2_flush_buffer(dev):
    """A buffer twice the size of L2 (read between timed launches)."""
    import torch
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    return torch.ones(2 * l2 // 4, dtype=torch.int32, device=dev)


def max_over_ranks(x: float, device, world: int) -> float:
    """The largest of every rank's x (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_ours(args, rank, world):
    import torch
    import torch.distributed as dist
    import w4a4_quantized_gemm_token_b200 as w4

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    P = peaks()
    fp4_peak = P["bf16"] * FP4_PER_BF16
    M = args.tokens
    if args.only is not None:
        rows = extra_rows(args, dev, stream, P)
        for v in rows.values():
            if isinstance(v, dict):
                v.pop("_y", None)
        print(json.dumps({"only": args.only, "rows": rows}), flush=True)
        return

    # ---- workload: Llama-2-70B layer linears, NVFP4 weights quantized once ----
    layers = []
    for li, (name, K, N) in enumerate(LLAMA):
        Wd = to_dev(synth.weights("llama2_70b", N, K, seed=0, tensor_id=100 + li), dev)
        Wq = w4.quantize_weight(Wd, w4.NVFP4)
        del Wd
        X = to_dev(synth.activations("llama2_70b", M, K, seed=rank, tensor_id=200 + li), dev)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w4.linear_workspace(M, N, K, w4.NVFP4), dtype=torch.uint8, device=dev)
        layers.append((name, K, N, Wq, X, Y, ws))
    torch.cuda.synchronize()
    flops_step = sum(2.0 * M * N * K for (_, K, N, *_r) in layers)

    def step():
        for (_, K, N, Wq, X, Y, ws) in layers:
            w4.linear(X, Wq, w4.SCALE_TOKEN, Y=Y, ws=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK

    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_clk0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    t_clk1 = time.time()
    if world > 1:
        dist.barrier()
    # the clock window after the timed region: the same steps for 0.4 s,
    # untimed (used only when the timed region held no clock sample)
    t_clk2 = time.time() + 0.4
    while time.time() < t_clk2:
        step()
        torch.cuda.synchronize()
    clocks = sampler.stop(t_clk0, t_clk1, t_clk2)
    ms = ev0.elapsed_time(ev1) / args.steps
    ms = max_over_ranks(ms, dev, world)
    value = flops_step * world / (ms * 1e-3) / 1e12
    assert w4.device_status() == w4.OK
    launches = 2 * len(layers) * args.steps

    # ---- end to end through the public API with host buffers ----
    hX = [torch.empty(X.shape, dtype=torch.bfloat16, pin_memory=True) for (_, _, _, _, X, _, _) in layers]
    hY = [torch.empty(Y.shape, dtype=torch.bfloat16, pin_memory=True) for (_, _, _, _, _, Y, _) in layers]
    for h, (_, _, _, _, X, _, _) in zip(hX, layers):
        h.copy_(X)
    h2d = sum(h.numel() * 2 for h in hX)
    d2h = sum(h.numel() * 2 for h in hY)

    # Copies overlap the compute: a copy-in stream brings X of linear i + 1
    # while linear i runs, a copy-out stream returns Y of linear i - 1 (PCIe is
    # full duplex); events order each buffer's reuse across steps.
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    nl = len(layers)
    ev_in = [torch.cuda.Event() for _ in range(nl)]
    ev_comp = [torch.cuda.Event() for _ in range(nl)]
    ev_out = [torch.cuda.Event() for _ in range(nl)]
    for i in range(nl):  # every buffer starts free
        ev_comp[i].record(stream)
        ev_out[i].record(stream)

    def e2e_step():
        for i, (_, K, N, Wq, X, Y, ws) in enumerate(layers):
            s_in.wait_event(ev_comp[i])       # X_i no longer read by the previous step
            with torch.cuda.stream(s_in):
                X.copy_(hX[i], non_blocking=True)
            ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            stream.wait_event(ev_out[i])      # Y_i of the previous step has left
            w4.linear(X, Wq, w4.SCALE_TOKEN, Y=Y, ws=ws)
            ev_comp[i].record(stream)
            s_out.wait_event(ev_comp[i])
            with torch.cuda.stream(s_out):
                hY[i].copy_(Y, non_blocking=True)
            ev_out[i].record(s_out)

    def e2e_timed(iters):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        for _ in range(iters):
            e2e_step()
        for i in range(nl):  # the last outputs are home
            stream.wait_event(ev_out[i])
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / iters

    e2e_iters = max(3, min(args.steps, 10))
    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e2e_ms = e2e_timed(e2e_iters)
    e2e_ms = max_over_ranks(e2e_ms, dev, world)
    e2e_value = flops_step * world / (e2e_ms * 1e-3) / 1e12

    # ---- dominant kernel: the block-scaled GEMM alone, per shape ----
    gemm_ms, gemm_flops = 0.0, 0.0
    per_shape = {}
    for (name, K, N, Wq, X, Y, ws) in layers:
        Xq = w4.quantize_act(X, w4.NVFP4, w4.SCALE_TOKEN)
        w4.gemm(Xq, Wq, Y)
        t_ms = time_loop(lambda: w4.gemm(Xq, Wq, Y), max(5, args.steps), stream)
        f = 2.0 * M * N * K
        per_shape[name] = round(f / (t_ms * 1e-3) / 1e12, 1)
        gemm_ms += t_ms
        gemm_flops += f
        del Xq
    gemm_tflops = gemm_flops / (gemm_ms * 1e-3) / 1e12
    sm_mhz = (clocks or {}).get("sm_mhz") or P["sm_max_mhz"]
    issue_peak = mma_issue_peak_tflops(dev, sm_mhz)
    roofline = {"bound": "tensor", "achieved": round(gemm_tflops, 1), "peak": round(fp4_peak, 1),
                "unit": "TFLOP/s", "frac": round(gemm_tflops / fp4_peak, 4), "traffic": profiled_traffic(),
                "peak_src": f"{P['src']} bf16 burst x {FP4_PER_BF16:g} (nominal fp4/bf16)",
                "kernel": "gemm_fp4_pair_kernel (NVFP4, 256x256 tile on a CTA pair)", "per_shape_tflops": per_shape,
                "frac_of_nominal_9pf": round(gemm_tflops / NOMINAL_FP4_TFLOPS, 4),
                "frac_of_mma_issue_peak": round(gemm_tflops / issue_peak, 4),
                "mma_issue_peak": round(issue_peak, 1),
                "mma_issue_peak_src": f"SMs x {MMA_FLOP_PER_CYCLE} FLOP/cycle (back-to-back 128x256x64 NVFP4 MMA "
                                      f"every 128 cycles) x median SM clock {sm_mhz:.0f} MHz"}

    rows = {} if args.no_rows else extra_rows(args, dev, stream, P)

    if rank == 0:
        line = {
            "metric": "W4A4 linear TFLOPS (Llama-2-70B layer, NVFP4 per-token)",
            "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
            "config": {"workload": f"llama2_70b layer linears (qkv,o,w1,w3,w2), fused per-token NVFP4 "
                                   f"W4A4 linear, M={M} tokens per GPU",
                       "tokens_per_gpu": M, "l2": "inputs larger than L2 (0.47 GB of weights per step)",
                       "parallelism": f"replicas x{world}"},
            "frac_of_fp4_peak": round(value / world / fp4_peak, 4),
            "frac_of_nominal_fp4_9pf": round(value / world / NOMINAL_FP4_TFLOPS, 4),
            "frac_of_mma_issue_peak": round(value / world / issue_peak, 4),
            "roofline": roofline,
            "e2e": {"value": round(e2e_value, 3), "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": clocks,
            "rows": rows,
        }
        if world == 1 and not args.no_cpu:
            threads = host_threads()
            v1, s1, _ = oracle_sample(args.cpu_rows, args.cpu_cols, 1)
            vn, sn, _ = oracle_sample(args.cpu_rows, args.cpu_cols, threads)
            line["cpu_baseline"] = {
                "value": vn, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                "sample": f"{args.cpu_rows} tokens x {args.cpu_cols} output columns of each of the 5 layer "
                          f"linears (full K); GEMM columns split over {threads} host threads, {sn:.1f} s",
                "single_thread": {"value": v1, "cores": 1, "seconds": round(s1, 2)},
                "host_cores": os.cpu_count()}
            small = rows.get("mxfp4_small_16x256x256") if isinstance(rows, dict) else None
            if small is not None and "_y" in small:
                ok, dt = mxfp4_small_parity(small.pop("_y"))
                small["parity_vs_oracle"] = ok
                small["oracle_us"] = round(dt * 1e6, 1)
        if isinstance(rows, dict) and isinstance(rows.get("mxfp4_small_16x256x256"), dict):
            rows["mxfp4_small_16x256x256"].pop("_y", None)
        print(json.dumps(line), flush=True)


def extra_rows(args, dev, stream, P):
    """The other hot-path rows, each timed with CUDA events on the launching stream."""
    import torch
    import w4a4_quantized_gemm_token_b200 as w4
    out = {}
    hbm = P["hbm"]
    it = max(5, args.steps)
    want = lambda name: args.only is None or args.only == name

    # the block-scaled GEMM alone on the Llama shapes (the profiling case)
    for li, (name, K, N) in enumerate(LLAMA if args.only == "gemm" else []):
        if args.shape and name != args.shape:
            continue
        M = args.tokens
        Wq = w4.quantize_weight(to_dev(synth.weights("llama2_70b", N, K, seed=0, tensor_id=100 + li), dev), w4.NVFP4)
        X = to_dev(synth.activations("llama2_70b", M, K, seed=0, tensor_id=200 + li), dev)
        Xq = w4.quantize_act(X, w4.NVFP4, w4.SCALE_TOKEN)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        for _ in range(args.warmup):
            w4.gemm(Xq, Wq, Y)
        ms = time_loop(lambda: w4.gemm(Xq, Wq, Y), args.steps, stream)
        out[f"gemm_nvfp4_{name}_m{M}"] = {"TFLOPS": round(2.0 * M * N * K / (ms * 1e-3) / 1e12, 1),
                                          "us": round(ms * 1e3, 2)}
        del Wq, X, Xq, Y

    # activation quantizer, per-token NVFP4 (and MXFP4 / INT4), Llama qkv and w2 inputs
    # (each launch timed after an L2 flush: the qkv input alone would fit in L2)
    flush = l2_flush_buffer(dev) if want("quant") else None
    for (name, M, K) in [] if not want("quant") else [("qkv_in", args.tokens, 8192), ("w2_in", args.tokens, 28672)]:
        X = to_dev(synth.activations("llama2_70b", M, K, seed=3), dev)
        for fmt, g, sb in [(w4.NVFP4, 16, 1), (w4.MXFP4, 32, 1), (w4.INT4, 128, 4)]:
            q = w4.QTensor(fmt, M, K, w4.SCALE_TOKEN if fmt == w4.NVFP4 else 0, dev)
            f = lambda: w4.quantize_act(X, fmt, w4.SCALE_TOKEN, out=q)
            f()
            ms = time_loop(f, it, stream, flush)
            byts = 2 * M * K + M * K / 2 + M * K / g * sb + (4 * M if fmt == w4.NVFP4 else 0)
            key = {w4.NVFP4: "nvfp4_token", w4.MXFP4: "mxfp4", w4.INT4: "int4"}[fmt]
            out[f"quant_{key}_{name}"] = {"GB/s": round(byts / ms / 1e6, 1), "frac_hbm": round(byts / ms / 1e6 / hbm, 3),
                                          "us": round(ms * 1e3, 2)}
        q = w4.QTensor(w4.NVFP4, M, K, w4.SCALE_TENSOR, dev)
        f = lambda: w4.quantize_act(X, w4.NVFP4, w4.SCALE_TENSOR, out=q)
        f()
        ms = time_loop(f, it, stream, flush)
        byts = 4 * M * K + M * K / 2 + M * K / 16
        out[f"quant_nvfp4_tensor_2pass_{name}"] = {"GB/s": round(byts / ms / 1e6, 1), "us": round(ms * 1e3, 2)}
        del X
    del flush

    # decode: M = 1 and 16 over the layer (weights streamed from HBM)
    Ws = []
    if not want("decode"):
        Ws = None
    for li, (name, K, N) in enumerate(LLAMA if Ws is not None else []):
        Wd = to_dev(synth.weights("llama2_70b", N, K, seed=0, tensor_id=100 + li), dev)
        Ws.append((K, N, w4.quantize_weight(Wd, w4.NVFP4)))
        del Wd
    for Md in ((1, 16) if Ws is not None else ()):
        bufs = []
        for (K, N, Wq) in Ws:
            X = to_dev(synth.activations("llama2_70b", Md, K, seed=5), dev)
            Y = torch.empty(Md, N, dtype=torch.bfloat16, device=dev)
            ws = torch.empty(w4.linear_workspace(Md, N, K, w4.NVFP4), dtype=torch.uint8, device=dev)
            bufs.append((X, Wq, Y, ws))

        def dec():
            for (X, Wq, Y, ws) in bufs:
                w4.linear(X, Wq, w4.SCALE_TOKEN, Y=Y, ws=ws)
        dec()
        ms = time_loop(dec, it, stream)
        byts = sum(N * K * 0.5625 + 2 * Md * K + 2 * Md * N for (K, N, _) in Ws)
        # the same layer as one CUDA graph (ten kernels, PDL edges kept): the
        # difference to the eager stream is what host launches cost
        t0 = time.perf_counter()
        for _ in range(it):
            dec()
        host_us = (time.perf_counter() - t0) / (it * 2 * len(bufs)) * 1e6
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            dec()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            dec()
        g.replay()
        ms_g = time_loop(g.replay, it, stream)
        out[f"decode_m{Md}_llama_layer"] = {
            "GB/s": round(byts / ms / 1e6, 1), "frac_hbm": round(byts / ms / 1e6 / hbm, 3), "us": round(ms * 1e3, 2),
            "graph_GB/s": round(byts / ms_g / 1e6, 1), "graph_frac_hbm": round(byts / ms_g / 1e6 / hbm, 3),
            "graph_us": round(ms_g * 1e3, 2), "host_launch_us_per_kernel": round(host_us, 2),
            "launch_overhead_us_per_layer": round((ms - ms_g) * 1e3, 2)}
        del g
    del Ws

    # INT4, Qwen2.5-7B shapes at M = 2048: groups of 128, and of 512 (the
    # rho-aware choice for this device's tensor / CUDA-core ratio)
    i8_peak = P["bf16"] * INT8_PER_BF16
    for G in ((128, w4.int4_group_for_rho(60.0)) if want("int4") else ()):
        tot_ms, tot_ops = 0.0, 0.0
        for li, (name, K, N) in enumerate(synth.SHAPES["qwen25_7b_int4"]):
            M = 2048
            Wq = w4.quantize_weight(to_dev(synth.weights("qwen25_7b_int4", N, K, tensor_id=300 + li), dev), w4.INT4,
                                    group=G)
            X = to_dev(synth.activations("qwen25_7b_int4", M, K), dev)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            ws = torch.empty(w4.linear_workspace(M, N, K, w4.INT4), dtype=torch.uint8, device=dev)
            f = lambda: w4.linear(X, Wq, 0, Y=Y, ws=ws)
            f()
            ms = time_loop(f, it, stream)
            tot_ms += ms
            tot_ops += 2.0 * M * N * K
        v = tot_ops / (tot_ms * 1e-3) / 1e12
        out[f"int4_g{G}_qwen25_7b_m2048"] = {"TOPS": round(v, 1), "frac_int8_peak": round(v / i8_peak, 3),
                                             "frac_of_nominal_int8_4p5": round(v / NOMINAL_INT8_TOPS, 3)}

    # dual-stage residual augmentation, Qwen2.5-3B shapes at M = 8192
    tot_ms, tot_f, tot_fk = 0.0, 0.0, 0.0
    for li, (name, K, N) in enumerate(synth.SHAPES["qwen25_3b_aug"] if want("aug") else []):
        M, nS = 8192, 256
        Xc = to_dev(synth.calibration("qwen25_3b_aug", K), dev)
        S = w4.select_channels(Xc, nS)
        Wq = w4.quantize_weight(to_dev(synth.weights("qwen25_3b_aug", N, K, tensor_id=400 + li), dev), w4.NVFP4, S=S)
        X = to_dev(synth.activations("qwen25_3b_aug", M, K), dev)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(w4.linear_workspace(M, N, K, w4.NVFP4, nS), dtype=torch.uint8, device=dev)
        f = lambda: w4.linear(X, Wq, w4.SCALE_TOKEN, S=S, Y=Y, ws=ws)
        f()
        ms = time_loop(f, it, stream)
        tot_ms += ms
        tot_f += 2.0 * M * N * (K + nS)
        tot_fk += 2.0 * M * N * K
    if tot_ms > 0:
        out["aug_nvfp4_qwen25_3b_m8192"] = {"TFLOPS_exec": round(tot_f / (tot_ms * 1e-3) / 1e12, 1),
                                            "TFLOPS_effective_K": round(tot_fk / (tot_ms * 1e-3) / 1e12, 1)}
    # fused qkv with one weight scale per module (q | k | v segments): the
    # linear at M = 4096 and the M = 1 decode, beside the one-scale weights
    if want("segments"):
        K = 8192
        rows, gains = synth.FUSED["llama2_70b"]["qkv"]
        Wb, seg = synth.fused_weights(rows, gains, K, seed=0, tensor_id=100)
        Wd = to_dev(Wb, dev)
        del Wb
        N = seg[-1]
        variants = {"segments": w4.quantize_weight_segments(Wd, seg), "one_scale": w4.quantize_weight(Wd, w4.NVFP4)}
        del Wd
        fl = l2_flush_buffer(dev)  # the M = 1 weights (47 MB) would stay in L2
        for Ms in (args.tokens, 1):
            X = to_dev(synth.activations("llama2_70b", Ms, K, seed=9), dev)
            Y = torch.empty(Ms, N, dtype=torch.bfloat16, device=dev)
            ws = torch.empty(w4.linear_workspace(Ms, N, K, w4.NVFP4), dtype=torch.uint8, device=dev)
            for vname, Wq in variants.items():
                f = lambda: w4.linear(X, Wq, w4.SCALE_TOKEN, Y=Y, ws=ws)
                for _ in range(max(3, args.warmup)):
                    f()
                ms = time_loop(f, it, stream, None if Ms > 16 else fl)
                if Ms > 16:
                    out[f"qkv_{vname}_m{Ms}"] = {"TFLOPS": round(2.0 * Ms * N * K / (ms * 1e-3) / 1e12, 1),
                                                 "us": round(ms * 1e3, 2)}
                else:
                    byts = N * K * 0.5625 + 2 * Ms * K + 2 * Ms * N + (4 * N if vname == "segments" else 0)
                    out[f"qkv_{vname}_m{Ms}"] = {"GB/s": round(byts / ms / 1e6, 1), "us": round(ms * 1e3, 2)}
            del X, Y, ws
        del variants, fl

    # the fused per-token NVFP4 linear over the Llama layer at other token
    # counts: 128 on the one-CTA kernel (128 x 256 tiles, N / 256 of them);
    # 256 and 1024 on the CTA pair, few waves of 256 x 256 tiles streaming the
    # weights from memory once; 16384 runs many waves
    for Ms in ((128, 256, 1024, 16384) if want("tokens") else ()):
        lay = []
        for li, (name, K, N) in enumerate(LLAMA):
            Wq = w4.quantize_weight(to_dev(synth.weights("llama2_70b", N, K, seed=0, tensor_id=100 + li), dev),
                                    w4.NVFP4)
            X = to_dev(synth.activations("llama2_70b", Ms, K, seed=0, tensor_id=200 + li), dev)
            Y = torch.empty(Ms, N, dtype=torch.bfloat16, device=dev)
            ws = torch.empty(w4.linear_workspace(Ms, N, K, w4.NVFP4), dtype=torch.uint8, device=dev)
            lay.append((K, N, Wq, X, Y, ws))

        def layer_step():
            for (K, N, Wq, X, Y, ws) in lay:
                w4.linear(X, Wq, w4.SCALE_TOKEN, Y=Y, ws=ws)
        for _ in range(max(3, args.warmup)):
            layer_step()
        ms = time_loop(layer_step, max(3, min(args.steps, 10)), stream)
        fl = sum(2.0 * Ms * N * K for (K, N, *_r) in lay)
        out[f"linear_nvfp4_llama_layer_m{Ms}"] = {"TFLOPS": round(fl / (ms * 1e-3) / 1e12, 1),
                                                  "ms": round(ms, 3)}
        del lay

    # the same layer at M = 4096 as a deployment runs it: gate and up (w1, w3)
    # read the same normalized input, so they are one module of N = 2 x 28672
    # with one NVFP4 weight scale per segment, quantized once per call (the
    # FLOPs are those of the five-linear headline; the headline keeps the five)
    if want("tokens"):
        Ms = args.tokens
        lay = []
        for li in (0, 1, 4):  # qkv, o, w2
            name, K, N = LLAMA[li]
            Wq = w4.quantize_weight(to_dev(synth.weights("llama2_70b", N, K, seed=0, tensor_id=100 + li), dev),
                                    w4.NVFP4)
            X = to_dev(synth.activations("llama2_70b", Ms, K, seed=0, tensor_id=200 + li), dev)
            lay.append((K, N, Wq, X))
        _, K13, N1 = LLAMA[2]
        W13 = torch.cat([to_dev(synth.weights("llama2_70b", N1, K13, seed=0, tensor_id=100 + li), dev) for li in (2, 3)])
        Wq13 = w4.quantize_weight_segments(W13, [0, N1, 2 * N1])
        del W13
        X13 = to_dev(synth.activations("llama2_70b", Ms, K13, seed=0, tensor_id=202), dev)
        lay.insert(2, (K13, 2 * N1, Wq13, X13))
        lay = [(K, N, Wq, X, torch.empty(Ms, N, dtype=torch.bfloat16, device=dev),
                torch.empty(w4.linear_workspace(Ms, N, K, w4.NVFP4), dtype=torch.uint8, device=dev))
               for (K, N, Wq, X) in lay]

        def fused_step():
            for (K, N, Wq, X, Y, ws) in lay:
                w4.linear(X, Wq, w4.SCALE_TOKEN, Y=Y, ws=ws)
        for _ in range(max(3, args.warmup)):
            fused_step()
        ms = time_loop(fused_step, max(3, min(args.steps, 10)), stream)
        fl = sum(2.0 * Ms * N * K for (K, N, *_r) in lay)
        out[f"linear_nvfp4_llama_layer_gate_up_fused_m{Ms}"] = {
            "TFLOPS": round(fl / (ms * 1e-3) / 1e12, 1), "ms": round(ms, 3),
            "linears": "qkv, o, w1|w3 as one module (per-segment weight scales), w2"}
        del lay

    # the 300M SwiGLU decoder layer at M = 4096, NVFP4 with a tensor scale on
    # both sides (the activation scale from an amax pass on every call)
    if want("swiglu"):
        lay = []
        for li, (name, K, N) in enumerate(synth.SHAPES["swiglu300m"]):
            Wq = w4.quantize_weight(to_dev(synth.weights("swiglu300m", N, K, seed=0, tensor_id=100 + li), dev),
                                    w4.NVFP4)
            X = to_dev(synth.activations("swiglu300m", args.tokens, K, seed=0, tensor_id=200 + li), dev)
            Y = torch.empty(args.tokens, N, dtype=torch.bfloat16, device=dev)
            ws = torch.empty(w4.linear_workspace(args.tokens, N, K, w4.NVFP4), dtype=torch.uint8, device=dev)
            lay.append((K, N, Wq, X, Y, ws))

        def sw_step():
            for (K, N, Wq, X, Y, ws) in lay:
                w4.linear(X, Wq, w4.SCALE_TENSOR, Y=Y, ws=ws)
        for _ in range(max(3, args.warmup)):
            sw_step()
        ms = time_loop(sw_step, max(5, min(args.steps, 20)), stream)
        fl = sum(2.0 * args.tokens * N * K for (K, N, *_r) in lay)
        out[f"linear_nvfp4_tensor_swiglu300m_m{args.tokens}"] = {"TFLOPS": round(fl / (ms * 1e-3) / 1e12, 1),
                                                                 "ms": round(ms, 3)}
        # static activation scale (a calibrated constant per linear, here the
        # tensor's own amax / 2688 taken once outside the timed region): the
        # quantizer with the caller's s2, then the GEMM; and the quantizers
        # alone, dynamic (amax inside the call) against static
        qs, sts = [], []
        for (K, N, Wq, X, Y, ws) in lay:
            sts.append((X.float().abs().max() / 2688.0).reshape(1).contiguous())
            qs.append(w4.QTensor(w4.NVFP4, args.tokens, K, w4.SCALE_TENSOR, dev))

        def st_step():
            for (K, N, Wq, X, Y, ws), q, st in zip(lay, qs, sts):
                w4.quantize_act(X, w4.NVFP4, w4.SCALE_TENSOR, static_s2=st, out=q)
                w4.gemm(q, Wq, Y)

        def q_dyn():
            for (K, N, Wq, X, Y, ws), q in zip(lay, qs):
                w4.quantize_act(X, w4.NVFP4, w4.SCALE_TENSOR, out=q)

        def q_st():
            for (K, N, Wq, X, Y, ws), q, st in zip(lay, qs, sts):
                w4.quantize_act(X, w4.NVFP4, w4.SCALE_TENSOR, static_s2=st, out=q)
        for _ in range(max(3, args.warmup)):
            st_step()
        ms_s = time_loop(st_step, max(5, min(args.steps, 20)), stream)
        out[f"linear_nvfp4_static_s2_swiglu300m_m{args.tokens}"] = {"TFLOPS": round(fl / (ms_s * 1e-3) / 1e12, 1),
                                                                    "ms": round(ms_s, 3)}
        q_dyn()
        q_st()
        ms_qd = time_loop(q_dyn, max(5, min(args.steps, 20)), stream)
        ms_qs = time_loop(q_st, max(5, min(args.steps, 20)), stream)
        out[f"quant_nvfp4_tensor_swiglu300m_layer_inputs_m{args.tokens}"] = {
            "dynamic_us": round(ms_qd * 1e3, 2), "static_us": round(ms_qs * 1e3, 2),
            "amax_cost_us": round((ms_qd - ms_qs) * 1e3, 2)}
        del lay, qs, sts

    # multi-pass MXFP4 (two passes) on the Llama qkv shape: the quantizer alone
    # (L2 flushed before each launch) and the linear, beside one-pass MXFP4
    if want("msd"):
        K, N, M = 8192, 10240, args.tokens
        Wd = to_dev(synth.weights("llama2_70b", N, K, tensor_id=100), dev)
        W1, W2 = w4.quantize_weight(Wd, w4.MXFP4), w4.quantize_weight_msd(Wd, 2)
        del Wd
        X = to_dev(synth.activations("llama2_70b", M, K, seed=7), dev)
        q = w4.QTensor(w4.MXFP4, M, 2 * K, 0, dev)
        fl = l2_flush_buffer(dev)
        f = lambda: w4.quantize_act_msd(X, 2, out=q)
        for _ in range(max(3, args.warmup)):
            f()
        ms = time_loop(f, it, stream, fl)
        byts = 2 * M * K + 2 * (M * K / 2 + M * K / 32)
        out["msd2_quant_llama_qkv_in"] = {"GB/s": round(byts / ms / 1e6, 1), "frac_hbm": round(byts / ms / 1e6 / hbm, 3),
                                          "us": round(ms * 1e3, 2)}
        del fl
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        for name, fn, passes in (("mxfp4_1pass", lambda: w4.linear(X, W1, 0, Y=Y), 1),
                                 ("msd2", lambda: w4.linear_msd(X, W2, 2, Y=Y), 2)):
            for _ in range(max(3, args.warmup)):
                fn()
            ms = time_loop(fn, it, stream)
            out[f"{name}_linear_llama_qkv_m{M}"] = {
                "TFLOPS_exec": round(2.0 * M * N * K * passes / (ms * 1e-3) / 1e12, 1),
                "TFLOPS_effective_K": round(2.0 * M * N * K / (ms * 1e-3) / 1e12, 1), "us": round(ms * 1e3, 2)}
        del W1, W2, X, q, Y

    # block-local Hadamard rotation, NVFP4 per token, Llama qkv shape: the
    # rotating quantizer alone (L2 flushed) and the linear, beside the plain ones
    if want("hadamard"):
        K, N, M = 8192, 10240, args.tokens
        Wd = to_dev(synth.weights("llama2_70b", N, K, tensor_id=100), dev)
        Wp, Wr = w4.quantize_weight(Wd, w4.NVFP4), w4.quantize_weight(Wd, w4.NVFP4, hadamard=True)
        del Wd
        X = to_dev(synth.activations("llama2_70b", M, K, seed=8), dev)
        fl = l2_flush_buffer(dev)
        byts = 2 * M * K + M * K / 2 + M * K / 16 + 4 * M
        for name, rot in (("plain", False), ("hadamard", True)):
            q = w4.QTensor(w4.NVFP4, M, K, w4.SCALE_TOKEN, dev, w4.FLAG_HADAMARD if rot else 0)
            f = lambda: w4.quantize_act(X, w4.NVFP4, w4.SCALE_TOKEN, out=q)
            for _ in range(max(3, args.warmup)):
                f()
            ms = time_loop(f, it, stream, fl)
            out[f"quant_nvfp4_token_{name}_llama_qkv_in"] = {"GB/s": round(byts / ms / 1e6, 1),
                                                              "frac_hbm": round(byts / ms / 1e6 / hbm, 3),
                                                              "us": round(ms * 1e3, 2)}
        del fl
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        for name, Wq in (("plain", Wp), ("hadamard", Wr)):
            fn = lambda: w4.linear(X, Wq, w4.SCALE_TOKEN, Y=Y)
            for _ in range(max(3, args.warmup)):
                fn()
            ms = time_loop(fn, it, stream)
            out[f"linear_nvfp4_{name}_llama_qkv_m{M}"] = {"TFLOPS": round(2.0 * M * N * K / (ms * 1e-3) / 1e12, 1),
                                                          "us": round(ms * 1e3, 2)}
        del Wp, Wr, X, Y

    # the MXFP4 16 x 256 x 256 workload (X ~ N(0,1), W ~ N(0,0.02), seed 0):
    # the fused linear's time, eager and as a CUDA graph; its output is kept
    # for the oracle comparison of the CPU-baseline leg
    if want("small"):
        Xs = to_dev(synth.activations("mxfp4_small", 16, 256, seed=0), dev)
        Wsm = w4.quantize_weight(to_dev(synth.weights("mxfp4_small", 256, 256, seed=0), dev), w4.MXFP4)
        Ysm = torch.empty(16, 256, dtype=torch.bfloat16, device=dev)
        wss = torch.empty(w4.linear_workspace(16, 256, 256, w4.MXFP4), dtype=torch.uint8, device=dev)
        f = lambda: w4.linear(Xs, Wsm, 0, Y=Ysm, ws=wss)
        for _ in range(10):
            f()
        ms = time_loop(f, 200, stream)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            f()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            f()
        g.replay()
        ms_g = time_loop(g.replay, 200, stream)
        torch.cuda.synchronize()
        out["mxfp4_small_16x256x256"] = {"us": round(ms * 1e3, 2), "graph_us": round(ms_g * 1e3, 2),
                                         "_y": Ysm.view(torch.int16).cpu().numpy().view(np.uint16)}
        del g

    if not want("mxfp4"):
        torch.cuda.synchronize()
        assert w4.device_status() == w4.OK
        return out

    # MXFP4 GEMM on the Llama qkv shape, M = 4096
    K, N, M = 8192, 10240, args.tokens
    Wq = w4.quantize_weight(to_dev(synth.weights("llama2_70b", N, K, tensor_id=100), dev), w4.MXFP4)
    X = to_dev(synth.activations("llama2_70b", M, K), dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(w4.linear_workspace(M, N, K, w4.MXFP4), dtype=torch.uint8, device=dev)
    f = lambda: w4.linear(X, Wq, 0, Y=Y, ws=ws)
    f()
    ms = time_loop(f, it, stream)
    out["mxfp4_linear_llama_qkv"] = {"TFLOPS": round(2.0 * M * N * K / (ms * 1e-3) / 1e12, 1)}
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--tokens", type=int, default=4096)
    ap.add_argument("--ref-rows", type=int, default=2, help="reference arm: tokens per step")
    ap.add_argument("--ref-cols", type=int, default=2048, help="reference arm: output columns per linear")
    ap.add_argument("--cpu-rows", type=int, default=8, help="cpu_baseline sample: tokens")
    ap.add_argument("--cpu-cols", type=int, default=4096, help="cpu_baseline sample: output columns")
    ap.add_argument("--no-rows", action="store_true", help="skip the secondary rows")
    ap.add_argument("--only", choices=["gemm", "quant", "decode", "int4", "aug", "mxfp4", "segments", "msd", "hadamard",
                                       "tokens", "swiglu", "small"], default=None,
                    help="run only one secondary row (for profiling) and print it")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--shape", default=None, help="--only gemm: one Llama linear (qkv, o, w1, w3, w2)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores alone; no collective is needed
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
