"""Benchmark: one streaming denoise step of a 30-layer 5B-style video DiT on the
NVFP4 W4A4 path (libnvfp4), on synthetic seeded inputs.

Step (per layer, on a 3-frame chunk of 2640 tokens; dim 3072, 24 heads x 128,
FFN 14336): quantize the layer input -> QKV GEMM (N=9216) -> kv_quant_chunk of
the 3 new frames' K and V straight out of the QKV output -> kv_dequant_window
over 12 cached frames (3 sinks + 9 window) -> quantize the attention-output
stand-in -> out-proj GEMM -> quantize -> FFN-up GEMM (N=14336) with the GELU
(tanh form) in its epilogue -> requantize the intermediate -> FFN-down GEMM;
the down output feeds the next layer.  Attention, norms and residuals are not
part of the NVFP4 path and are not run; the attention output is a fixed seeded
tensor; attention straight from the NVFP4 cache (nvfp4_window_attention) is
timed separately on layer 0's window.  Weights are pre-quantized
(outside the timed region).  The whole step is captured once as a CUDA graph.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own step (independent chunks, weak
scaling); ranks only synchronise for the barrier and the max-over-ranks timing.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import nvfp4_w4a4_quantized_08_b200 as nv  # noqa: E402
from nvfp4_w4a4_quantized_08_b200 import workloads as wl  # noqa: E402

from nvfp4_w4a4_quantized_08_b200.dit_step import (D, F, GEMM_FLOPS_LAYER, GEMM_SHAPES,  # noqa: E402
                                                   M, NEW_FRAMES, POOL, QKV, TPF, WINDOW,
                                                   DiTStep)

Q_BYTES_PER_ELEM = 2 + 0.5625     # bf16 in, 4-bit code + 1/16 E4M3 scale out
KV_ELEMS_FRAME = TPF * wl.HEADS * wl.HEAD_DIM
CODEC_BYTES = {
    "quant_act": 3 * M * D * Q_BYTES_PER_ELEM + 3 * 4,
    "requant_ffn": M * F * Q_BYTES_PER_ELEM + 4,
    "kv_quant": 2 * NEW_FRAMES * KV_ELEMS_FRAME * Q_BYTES_PER_ELEM + 2 * 4,
    "kv_dequant": 2 * WINDOW * KV_ELEMS_FRAME * Q_BYTES_PER_ELEM,
}
GEMM_SRC = os.path.join(ROOT, "nvfp4_w4a4_quantized_08_b200", "csrc", "gemm.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "nvfp4_gemm_dit_step_traffic.txt")


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def max_over_ranks(value: float, dist, device) -> float:
    """The largest `value` over all ranks (identity without a process group)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank runs its own step (weak scaling)."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = [s for s in sm if mx and s > 0.3 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def gemm_traffic_per_launch():
    """DRAM bytes per GEMM launch from the committed ncu summary, or None when
    the summary is missing or was taken on a different gemm.cu."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    src_hash = hashlib.sha256(open(GEMM_SRC, "rb").read()).hexdigest()[:16]
    vals = {}
    for line in open(TRAFFIC_FILE):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("gemm_cu_sha256_16") != src_hash:
        return None
    try:
        return float(vals["traffic_bytes_per_launch_avg"])
    except (KeyError, ValueError):
        return None


class CpuSample:
    """The CPU oracle on a bounded sample of the step: `rows` token rows through
    one layer's four activation quantizations and four FP64 GEMMs (that layer's
    weights pre-quantized by the oracle once, not timed), and the K + V codec
    (quantize + dequantize) of one latent frame."""

    def __init__(self, rows: int = 16, seed_layer: int = 0, threads: int = 0):
        import oracle
        self.oracle = oracle
        self.cores = oracle.set_threads(threads)
        self.rows = rows
        if torch.cuda.is_available():
            wts = [t.cpu() for t in wl.layer_weights_cuda(seed_layer, device="cuda")]
        else:
            wts = [wl.weights(n, k, c=5, i=10 + j) for j, (n, k) in
                   enumerate([(QKV, D), (D, D), (F, D), (D, F)])]
        self.wq = [oracle.quantize(self.bits(t)) for t in wts]
        self.x = self.bits(wl.activations(rows=rows, c=5, i=0))
        self.attn = self.bits(wl.randn((rows, D), 5, 1))
        self.kv = self.bits(wl.kv_tensor(seed=20, tokens=TPF)).reshape(-1)

    @staticmethod
    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    def run(self):
        """Returns dict(tflops, kv_gbs, cores, sample, seconds)."""
        o = self.oracle

        def to_bf16_bits(y):
            return self.bits(torch.from_numpy(np.ascontiguousarray(y, np.float32))
                             .to(torch.bfloat16))

        t0 = time.perf_counter()
        o.gemm(o.quantize(self.x), self.wq[0])
        y, _ = o.gemm(o.quantize(self.attn), self.wq[1])
        u, _ = o.gemm(o.quantize(to_bf16_bits(y)), self.wq[2])
        # the FFN GELU on the bf16 up-projection output, as the GPU step computes it
        u16 = (to_bf16_bits(u).astype(np.uint32) << 16).view(np.float32)
        o.gemm(o.quantize(to_bf16_bits(o.gelu_tanh(u16))), self.wq[3])
        t_rows = time.perf_counter() - t0
        t0 = time.perf_counter()
        ck, sk, tk = o.kv_quant_chunk(self.kv, 1, TPF, wl.HEADS, wl.HEAD_DIM)
        cv, sv, tv = o.kv_quant_chunk(self.kv, 1, TPF, wl.HEADS, wl.HEAD_DIM)
        o.kv_dequant_window(ck, sk, tk, [0], TPF, wl.HEADS, wl.HEAD_DIM)
        o.kv_dequant_window(cv, sv, tv, [0], TPF, wl.HEADS, wl.HEAD_DIM)
        t_kv = time.perf_counter() - t0
        flops = self.rows * GEMM_FLOPS_LAYER / M
        kv_bytes = 2 * 2 * KV_ELEMS_FRAME * Q_BYTES_PER_ELEM
        desc = (f"CPU oracle, {self.rows} of {M} token rows through one layer (4 activation "
                f"quantizations, the FFN GELU + 4 FP64 GEMMs: {flops / 1e9:.2f} GFLOP in "
                f"{t_rows:.2f} s) and "
                f"the K+V codec of one 880-token frame ({kv_bytes / 1e6:.1f} MB in {t_kv:.2f} s)")
        return {"tflops": flops / t_rows / 1e12, "kv_gbs": kv_bytes / t_kv / 1e9,
                "cores": self.cores, "sample": desc, "seconds": t_rows + t_kv}


# ---------------------------------------------------------------- arms
def run_reference(args):
    rank = env_int("RANK", 0)
    if rank != 0:
        return 0
    res = []
    sample = CpuSample(rows=args.ref_rows)
    for i in range(args.warmup + args.steps):
        r = sample.run()
        if i >= args.warmup:
            res.append(r)
    value = statistics.median(r["tflops"] for r in res)
    secs = statistics.median(r["seconds"] for r in res)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(args),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": res[-1]["cores"],
                         "kind": "oracle", "sample": res[-1]["sample"],
                         "kv_codec_gbs": statistics.median(r["kv_gbs"] for r in res)},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


METRIC = "W4A4 NVFP4 GEMM TFLOP/s & KV quant/dequant GB/s, % of B200 roofline"


def config_block(args):
    return {"workload": f"dit_denoise_step_{args.layers}L_{M}tok", "layers": args.layers,
            "tokens": M, "dim": D, "ffn": F, "heads": wl.HEADS, "head_dim": wl.HEAD_DIM,
            "kv_window_frames": WINDOW, "kv_new_frames": NEW_FRAMES,
            "global_batch": M * max(1, args.gpus), "seq_len": M,
            "parallelism": f"replica{args.gpus}" if args.gpus > 1 else "single",
            "l2": "inputs larger than L2 (2.1 GB NVFP4 weights + 1.4 GB KV pools per step)",
            "stand_ins": "attention output fixed seeded tensor; attention, norm, residual "
                         "not run (outside the NVFP4 path); FFN GELU (tanh form) fused in the "
                         "up-projection epilogue"}


ATTN_FLOPS = 4 * M * WINDOW * TPF * wl.HEAD_DIM * wl.HEADS  # QK^T and PV, one layer


def time_window_attention(step: DiTStep, dev, reps: int = 10) -> float:
    """Device ms of one nvfp4_window_attention: the chunk's 2640 queries (the Q
    third of the QKV output) over layer 0's 12-slot window read from the NVFP4
    pools, graph-replayed."""
    cache = step.cache[0]
    q = step.qkv_out[:, :D]
    out = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        for _ in range(2):
            cache.window_attention(q, step.window, out=out)
        with torch.cuda.graph(g, stream=s):
            for _ in range(reps):
                cache.window_attention(q, step.window, out=out)
    torch.cuda.current_stream(dev).wait_stream(s)
    g.replay()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    del g
    return e0.elapsed_time(e1) / reps


def time_kv_four_over_six(step: DiTStep, dev, reps: int = 20) -> float:
    """Device ms of one nvfp4_kv_quant_chunk (3 frames of K and V read from a
    QKV output, amax pass included) with the Four Over Six scale rule."""
    cache = nv.KVCache(POOL, TPF, wl.HEADS, wl.HEAD_DIM, device=dev,
                       scale_rule=nv.SCALE_FOUR_OVER_SIX)
    k, v = step.qkv_out[:, D:2 * D], step.qkv_out[:, 2 * D:]
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        for _ in range(2):
            cache.quant_chunk(k, v, step.new_slots, ws=nv.workspace(dev))
        with torch.cuda.graph(g, stream=s):
            for _ in range(reps):
                cache.quant_chunk(k, v, step.new_slots, ws=nv.workspace(dev))
    torch.cuda.current_stream(dev).wait_stream(s)
    g.replay()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    del g
    return e0.elapsed_time(e1) / reps


class L2Flush:
    """Writes a buffer twice the size of L2 so the next timed call starts with
    its inputs in HBM only."""

    def __init__(self, dev):
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.buf = torch.empty(2 * max(l2, 64 << 20), dtype=torch.uint8, device=dev)

    def __call__(self):
        self.buf.zero_()


def time_flushed(fn, flush, reps: int = 20, warmup: int = 3) -> float:
    """Median device ms of fn() over `reps` calls, L2 flushed before each one;
    CUDA events on the launching stream bracket fn() alone."""
    cur = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    times = []
    for _ in range(reps):
        flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        fn()
        e1.record(cur)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def time_configs(dev, peaks) -> dict:
    """The four single-call workloads, each timed on its own with L2 flushed
    before every call (median of 20):
      tiny: A and B fp32 256x256 with 2% x50 outliers -- quantize (amax pass
        included), dequantize, FP4 GEMM 256^3 (fp32 out): microseconds;
      qkv: activation quantization (amax pass included) + QKV GEMM
        2640x9216x3072 (bf16 out): TFLOP/s of the pair;
      ffn: quantize X, FFN-up 2640x14336x3072 with the GELU epilogue and its
        amax hand-off, requantize the intermediate, FFN-down 2640x3072x14336:
        TFLOP/s of the chain;
      kv: K and V [10560, 24, 128] quantized in chunks of 8 and 4 frames (amax
        pass included), then the 12-slot window rebuilt to bf16: GB/s."""
    flush = L2Flush(dev)
    ws = nv.workspace(dev)
    out = {}
    hbm = peaks["hbm_gbs"]

    a, b = wl.tiny_pair()
    a, b = a.to(dev), b.to(dev)
    qa, qb = nv.empty(256, 256, device=dev), nv.empty(256, 256, device=dev)
    y = torch.empty(256, 256, dtype=torch.float32, device=dev)
    dq = torch.empty(256, 256, dtype=torch.bfloat16, device=dev)
    t_q = time_flushed(lambda: nv.quantize(a, out=qa, ws=ws), flush)
    nv.quantize(b, out=qb, ws=ws)
    t_dq = time_flushed(lambda: nv.dequantize(qa, out=dq), flush)
    t_g = time_flushed(lambda: nv.gemm(qa, qb, out=y, ws=ws), flush)

    def tiny_all():
        nv.quantize(a, out=qa, ws=ws)
        nv.quantize(b, out=qb, ws=ws)
        nv.dequantize(qa, out=dq)
        nv.dequantize(qb, out=dq)
        nv.gemm(qa, qb, out=y, ws=ws)
    t_all = time_flushed(tiny_all, flush)
    out["tiny_256"] = {"quantize_us": t_q * 1e3, "dequantize_us": t_dq * 1e3,
                       "gemm_us": t_g * 1e3, "round_trip_and_gemm_us": t_all * 1e3,
                       "note": "latency-bound: 2 quantizations, 2 dequantizations, one GEMM"}

    w = wl.qkv()
    x, wq = w.a.to(dev), nv.quantize(w.w.to(dev))
    del w
    qx = nv.empty(M, D, device=dev)
    yq = torch.empty(M, QKV, dtype=torch.bfloat16, device=dev)
    flops = 2 * M * QKV * D
    qbytes = M * D * Q_BYTES_PER_ELEM + 4
    t_q = time_flushed(lambda: nv.quantize(x, out=qx, ws=ws), flush)
    t_g = time_flushed(lambda: nv.gemm(qx, wq, out=yq, ws=ws), flush)
    t_all = time_flushed(lambda: (nv.quantize(x, out=qx, ws=ws), nv.gemm(qx, wq, out=yq, ws=ws)),
                         flush)
    out["qkv_projection"] = {"tflops": flops / (t_all * 1e-3) / 1e12, "us": t_all * 1e3,
                             "gemm_tflops": flops / (t_g * 1e-3) / 1e12, "gemm_us": t_g * 1e3,
                             "quantize_gb_s": qbytes / (t_q * 1e-3) / 1e9,
                             "quantize_frac_hbm": qbytes / (t_q * 1e-3) / 1e9 / hbm,
                             "quantize_us": t_q * 1e3}
    del x, wq, qx, yq

    f = wl.ffn()
    x, wu, wd = f.x.to(dev), nv.quantize(f.w_up.to(dev)), nv.quantize(f.w_down.to(dev))
    del f
    qx, qh = nv.empty(M, D, device=dev), nv.empty(M, F, device=dev)
    h = torch.empty(M, F, dtype=torch.bfloat16, device=dev)
    yd = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
    amax = torch.zeros(1, dtype=torch.float32, device=dev)

    def ffn_chain():
        nv.quantize(x, out=qx, ws=ws)
        nv.gemm(qx, wu, out=h, ws=ws, c_amax=amax, act=nv.ACT_GELU_TANH)
        nv.quantize(h, out=qh, ws=ws, amax_in=amax)
        nv.gemm(qh, wd, out=yd, ws=ws)
    flops = 2 * 2 * M * F * D
    t_all = time_flushed(ffn_chain, flush)
    rq_bytes = M * F * Q_BYTES_PER_ELEM + 4
    t_rq = time_flushed(lambda: nv.quantize(h, out=qh, ws=ws), flush)
    out["ffn_pair"] = {"tflops": flops / (t_all * 1e-3) / 1e12, "us": t_all * 1e3,
                       "requant_gb_s": rq_bytes / (t_rq * 1e-3) / 1e9,
                       "requant_frac_hbm": rq_bytes / (t_rq * 1e-3) / 1e9 / hbm,
                       "requant_us_with_amax_pass": t_rq * 1e3}
    del x, wu, wd, qx, qh, h, yd

    k, v = wl.kv_window()
    k, v = k.to(dev), v.to(dev)
    cache = nv.KVCache(WINDOW, TPF, wl.HEADS, wl.HEAD_DIM, device=dev)
    kw, vw = torch.empty_like(k), torch.empty_like(v)
    slots = list(range(WINDOW))

    def kv_quant():
        cache.quant_chunk(k[:8 * TPF], v[:8 * TPF], slots[:8], ws=ws)
        cache.quant_chunk(k[8 * TPF:], v[8 * TPF:], slots[8:], ws=ws)

    elems = 2 * WINDOW * KV_ELEMS_FRAME
    qb_ = elems * Q_BYTES_PER_ELEM + 2 * 2 * 4
    db_ = elems * Q_BYTES_PER_ELEM
    t_q = time_flushed(kv_quant, flush)
    t_d = time_flushed(lambda: cache.dequant_window(slots, kw, vw), flush)
    t_all = time_flushed(lambda: (kv_quant(), cache.dequant_window(slots, kw, vw)), flush)
    out["kv_codec"] = {"gb_s": (qb_ + db_) / (t_all * 1e-3) / 1e9,
                       "frac_hbm": (qb_ + db_) / (t_all * 1e-3) / 1e9 / hbm, "us": t_all * 1e3,
                       "quant_gb_s": qb_ / (t_q * 1e-3) / 1e9,
                       "quant_frac_hbm": qb_ / (t_q * 1e-3) / 1e9 / hbm,
                       "dequant_gb_s": db_ / (t_d * 1e-3) / 1e9,
                       "dequant_frac_hbm": db_ / (t_d * 1e-3) / 1e9 / hbm,
                       "note": "quant: 2 chunks (8 + 4 frames) x K,V with amax passes"}
    out["timing"] = "each workload alone, L2 flushed before every call, median of 20"
    return out


def library_fp4_gemm(dev) -> dict:
    """Context only: cuBLASLt's NVFP4 GEMM (through torch) on the step's four
    GEMM shapes, fed the same NVFP4 operands as nvfp4_gemm (tensor-core scale
    layout), timed back to back like the step's launches (30 calls, same
    operands).  Never on the path; a yardstick for the FP4 tensor peak."""
    import torch.nn.functional as Fn
    res = {}
    g = torch.Generator(device=dev).manual_seed(1)
    for name, (m, n, k) in GEMM_SHAPES.items():
        try:
            qa = nv.quantize(torch.randn(m, k, device=dev, generator=g).to(torch.bfloat16))
            qw = nv.quantize((torch.randn(n, k, device=dev, generator=g) * 0.02)
                             .to(torch.bfloat16))
            out = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
            ws = nv.workspace(dev)
            a4 = qa.codes.view(torch.float4_e2m1fn_x2)
            w4 = qw.codes.view(torch.float4_e2m1fn_x2)
            sa, sw = qa.sf.view(torch.float8_e4m3fn), qw.sf.view(torch.float8_e4m3fn)

            def lib():
                return Fn.scaled_mm(a4, w4.t(), sa, Fn.ScalingType.BlockWise1x16, sw,
                                    Fn.ScalingType.BlockWise1x16,
                                    swizzle_a=Fn.SwizzleType.SWIZZLE_32_4_4,
                                    swizzle_b=Fn.SwizzleType.SWIZZLE_32_4_4,
                                    output_dtype=torch.bfloat16)

            def ours():
                nv.gemm(qa, qw, out=out, ws=ws)
            r = {}
            for tag, fn in (("cublaslt", lib), ("nvfp4_gemm", ours)):
                for _ in range(3):
                    fn()
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(30):
                    fn()
                e1.record()
                torch.cuda.synchronize()
                us = e0.elapsed_time(e1) / 30 * 1e3
                r[tag] = {"us": us, "tflops": 2 * m * n * k / us / 1e6}
            res[name] = r
        except Exception as e:  # a library without the NVFP4 path: report, do not fail
            res[name] = {"unavailable": str(e)[:200]}
    return res


def run_case(args) -> int:
    """One kernel on one step-shaped case, `reps` times, for profilers:
    ncu -k <kernel> -s <launches to skip> -c <n> python bench.py --case <name>."""
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(7)
    ws = nv.workspace(dev)
    case, reps = args.case, args.reps
    gemm_cases = {"gemm_qkv": ("qkv", nv.ACT_NONE), "gemm_out": ("out", nv.ACT_NONE),
                  "gemm_up": ("up", nv.ACT_GELU_TANH), "gemm_down": ("down", nv.ACT_NONE)}
    if case in gemm_cases:
        shape, act = gemm_cases[case]
        m, n, k = GEMM_SHAPES[shape]
        qa = nv.quantize(torch.randn(m, k, device=dev, generator=g).to(torch.bfloat16))
        qw = nv.quantize((torch.randn(n, k, device=dev, generator=g) * 0.02).to(torch.bfloat16))
        out = torch.empty(m, n, dtype=torch.bfloat16, device=dev)
        run = lambda: nv.gemm(qa, qw, out=out, ws=ws, act=act)  # noqa: E731
    elif case == "quant_amax":
        x = torch.randn(M, D, device=dev, generator=g).to(torch.bfloat16)
        q = nv.empty(M, D, device=dev)
        # no tensor scale handed in: the amax pass, then the encode
        run = lambda: nv.quantize(x, out=q, ws=ws)  # noqa: E731
    elif case in ("quant_act", "quant_ffn"):
        cols = D if case == "quant_act" else F
        x = torch.randn(M, cols, device=dev, generator=g).to(torch.bfloat16)
        q = nv.empty(M, cols, device=dev)
        st = nv.quantize(x).s_t.clone()
        # the encode pass alone, as in the step (tensor scale handed in)
        run = lambda: nv.quantize(x, out=q, ws=ws, s_t=st)  # noqa: E731
    elif case in ("kv_quant", "kv_quant_fos", "kv_dequant", "attention"):
        rule = nv.SCALE_FOUR_OVER_SIX if case == "kv_quant_fos" else nv.SCALE_ONTO_6
        cache = nv.KVCache(POOL, TPF, wl.HEADS, wl.HEAD_DIM, device=dev, scale_rule=rule)
        qkv = torch.randn(M, QKV, device=dev, generator=g).to(torch.bfloat16)
        for s0 in (0, 3, 6, 9):
            cache.quant_chunk(qkv[:, D:2 * D], qkv[:, 2 * D:], [s0, s0 + 1, s0 + 2], ws=ws)
        window = [0, 1, 2, 6, 7, 8, 9, 10, 11, 12, 13, 14]
        kw = torch.empty(WINDOW * TPF, wl.HEADS, wl.HEAD_DIM, dtype=torch.bfloat16, device=dev)
        vw = torch.empty_like(kw)
        o = torch.empty(M, D, dtype=torch.bfloat16, device=dev)
        if case in ("kv_quant", "kv_quant_fos"):
            run = lambda: cache.quant_chunk(qkv[:, D:2 * D], qkv[:, 2 * D:],  # noqa: E731
                                            [12, 13, 14], ws=ws)
        elif case == "kv_dequant":
            cache.quant_chunk(qkv[:, D:2 * D], qkv[:, 2 * D:], [12, 13, 14], ws=ws)
            run = lambda: cache.dequant_window(window, kw, vw)  # noqa: E731
        else:
            cache.quant_chunk(qkv[:, D:2 * D], qkv[:, 2 * D:], [12, 13, 14], ws=ws)
            run = lambda: cache.window_attention(qkv[:, :D], window, out=o)  # noqa: E731
    else:
        raise SystemExit(f"unknown case {case!r}")
    torch.cuda.synchronize()
    for _ in range(reps):
        run()
    torch.cuda.synchronize()
    status = nv.device_status(ws)
    if status:
        raise SystemExit(f"device status {status}")
    print(f"{case}: {reps} reps ok")
    return 0


def run_ours(args):
    world = env_int("WORLD_SIZE", 1)
    rank = env_int("RANK", 0)
    local = env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    step = DiTStep(args.layers, dev)
    stream = torch.cuda.Stream(device=dev)
    # eager warm-up (first calls set kernel attributes), then capture one step
    with torch.cuda.stream(stream):
        step.run()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step.run()
    torch.cuda.synchronize()

    # ---- timed region A: K graph replays, inputs resident in HBM
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    ev0.record(cur)
    for _ in range(args.steps):
        graph.replay()
    ev1.record(cur)
    torch.cuda.synchronize()
    barrier()
    clock_info = clocks.stop()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), dist, dev)
    ms_step = ms_total / args.steps
    flops_step = GEMM_FLOPS_LAYER * args.layers
    value = job_throughput(flops_step, world, ms_step)

    # ---- timed region B: per-kernel CUDA events captured inside a second graph
    names = []
    evs = []

    def mark(name):
        e = torch.cuda.Event(enable_timing=True, external=True)
        e.record(torch.cuda.current_stream())
        evs.append(e)
        names.append(name)

    graph_b = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_b, stream=stream):
        step.run(mark)
    torch.cuda.synchronize()
    per = {}
    n_prof = max(1, min(args.steps, 5))
    for _ in range(n_prof):
        graph_b.replay()
        torch.cuda.synchronize()
        for i in range(len(evs) - 1):
            per.setdefault(names[i], []).append(evs[i].elapsed_time(evs[i + 1]))
    kernel_ms = {k: sum(v) / n_prof for k, v in per.items()}  # per step
    gemm_ms = sum(v for k, v in kernel_ms.items() if k.startswith("gemm"))
    launches = {k: len(v) // n_prof for k, v in per.items()}
    gemm_launches = sum(v for k, v in launches.items() if k.startswith("gemm"))

    # ---- e2e: host input -> device, step, result -> host.  Every step's input
    # comes from pinned host memory and its result goes back to it, inside the
    # timed region; the copies run on a copy stream through two device staging
    # buffers each way, so step i+1's input and step i's result cross PCIe
    # while the neighbouring step computes
    h_in = torch.empty(M, D, dtype=torch.bfloat16, pin_memory=True)
    h_in.copy_(step.x_in.cpu())
    h_out = [torch.empty(M, D, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    x_stage = [torch.empty_like(step.x_in) for _ in range(2)]
    o_stage = [torch.empty_like(step.output()) for _ in range(2)]
    copy_stream = torch.cuda.Stream(device=dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in_ready", "in_free",
                                                             "out_ready", "out_free")}

    def run_e2e(n, eager=False):
        copy_stream.wait_stream(cur)
        with torch.cuda.stream(copy_stream):
            x_stage[0].copy_(h_in, non_blocking=True)
            ev["in_ready"][0].record(copy_stream)
        for i in range(n):
            b = i % 2
            if i + 1 < n:  # the next step's input, behind this step's compute
                nb = (i + 1) % 2
                with torch.cuda.stream(copy_stream):
                    if i >= 1:
                        copy_stream.wait_event(ev["in_free"][nb])
                    x_stage[nb].copy_(h_in, non_blocking=True)
                    ev["in_ready"][nb].record(copy_stream)
            cur.wait_event(ev["in_ready"][b])
            step.x_in.copy_(x_stage[b], non_blocking=True)
            ev["in_free"][b].record(cur)
            if eager:  # the step's C-ABI calls issued one by one through the binding
                step.run()
            else:
                graph.replay()
            if i >= 2:
                cur.wait_event(ev["out_free"][b])
            o_stage[b].copy_(step.output(), non_blocking=True)
            ev["out_ready"][b].record(cur)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(ev["out_ready"][b])
                h_out[b].copy_(o_stage[b], non_blocking=True)
                ev["out_free"][b].record(copy_stream)
        cur.wait_stream(copy_stream)

    run_e2e(2)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    run_e2e(args.steps)
    e1.record(cur)
    torch.cuda.synchronize()
    # the last step's result reached the host intact
    assert torch.equal(h_out[(args.steps - 1) % 2], step.output().cpu())
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    e2e_value = job_throughput(flops_step, world, ms_e2e / args.steps)
    # the same, with the step's launches issued eagerly every step: the host
    # side of every C-ABI call (argument checks, tensor maps) in the timed region
    run_e2e(2, eager=True)
    torch.cuda.synchronize()
    barrier()
    e0.record(cur)
    run_e2e(args.steps, eager=True)
    e1.record(cur)
    torch.cuda.synchronize()
    assert torch.equal(h_out[(args.steps - 1) % 2], step.output().cpu())
    ms_e2e_eager = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    status = nv.device_status(step.ws)
    # the KV chunk under Four Over Six (the adaptive KV scale rule; not on the
    # step's path): one layer's 3 new frames of K and V, graph-replayed
    fos_ms = time_kv_four_over_six(step, dev)
    # attention over the window straight from the NVFP4 pools (the window
    # rebuild's consumer; the step itself keeps a fixed attention output)
    attn_ms = time_window_attention(step, dev)

    peaks, peak_src = measured_peaks()
    # FP4 has no measured peak: 4 x the measured bf16 GEMM (the dense FP4:BF16
    # ratio).  The burst figure applies when the timed region ran at (near) the
    # maximum SM clock with no power cap, the sustained one (taken under the
    # power cap at a lower clock) otherwise.
    burst = 4.0 * peaks["bf16_tflops"]
    sustained = 4.0 * peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    at_max = bool(clock_info and clock_info.get("sm_mhz") and clock_info.get("sm_max_mhz")
                  and clock_info["sm_mhz"] >= 0.95 * clock_info["sm_max_mhz"]
                  and "sw_power_cap" not in clock_info.get("reasons", []))
    if clock_info is None:
        at_max = True
    fp4_peak = burst if at_max else sustained
    gemm_tflops = flops_step / (gemm_ms * 1e-3) / 1e12
    codec = {}
    for k in ("quant_act", "requant_ffn", "kv_quant", "kv_dequant"):
        b = CODEC_BYTES[k] * args.layers
        codec[k] = {"ms_per_step": kernel_ms.get(k), "gb_s": b / (kernel_ms[k] * 1e-3) / 1e9,
                    "frac_hbm": b / (kernel_ms[k] * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    kv_bytes = (CODEC_BYTES["kv_quant"] + CODEC_BYTES["kv_dequant"]) * args.layers
    kv_ms = kernel_ms["kv_quant"] + kernel_ms["kv_dequant"]
    traffic = gemm_traffic_per_launch()

    configs = None if args.no_configs else time_configs(dev, peaks)
    library = None if args.no_configs else library_fp4_gemm(dev)

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            r = CpuSample(rows=args.cpu_rows).run()
            cpu = {"value": r["tflops"], "unit": "TFLOP/s", "cores": r["cores"],
                   "kind": "oracle", "sample": r["sample"], "kv_codec_gbs": r["kv_gbs"]}
            r1 = CpuSample(rows=args.cpu_rows_1core, threads=1).run()
            cpu["one_core"] = {"value": r1["tflops"], "unit": "TFLOP/s", "cores": r1["cores"],
                               "sample": r1["sample"], "kv_codec_gbs": r1["kv_gbs"]}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp4(e2m1)xfp4 -> fp32 acc; codec u8/bf16", "data": "synthetic",
            "config": config_block(args),
            "roofline": {"bound": "tensor", "kernel": "nvfp4_gemm_kernel",
                         "achieved": gemm_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": gemm_tflops / fp4_peak,
                         "peak_source": (f"{peak_src}: 4 x bf16_tflops "
                                         f"({'burst' if at_max else 'sustained'}: "
                                         f"{peaks['bf16_tflops'] if at_max else peaks.get('bf16_tflops_sustained')}"
                                         f"), nominal FP4:BF16 dense ratio 4; chosen from the "
                                         f"clock record (median {clock_info and clock_info.get('sm_mhz')}"
                                         f" MHz of max {clock_info and clock_info.get('sm_max_mhz')})"),
                         "frac_vs_sustained": gemm_tflops / sustained,
                         "frac_vs_nominal_9pf": gemm_tflops / 9000.0,
                         "traffic": traffic,
                         "traffic_note": "ncu dram__bytes_read + dram__bytes_write per launch "
                                         "(writes still in L2 when a launch ends are not "
                                         "counted)"},
            "kv_codec": {"gb_s": kv_bytes / (kv_ms * 1e-3) / 1e9,
                         "frac_hbm": kv_bytes / (kv_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                         "hbm_peak_gbs": peaks["hbm_gbs"]},
            "codec": codec,
            "kv_quant_four_over_six": {
                "us": fos_ms * 1e3,
                "gb_s": CODEC_BYTES["kv_quant"] / (fos_ms * 1e-3) / 1e9,
                "frac_hbm": CODEC_BYTES["kv_quant"] / (fos_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "vs_onto_6_us": kernel_ms["kv_quant"] / args.layers * 1e3},
            "window_attention": {
                "us": attn_ms * 1e3, "tflops": ATTN_FLOPS / (attn_ms * 1e-3) / 1e12,
                "bound": "tensor (bf16 tcgen05.mma, fp32 accumulate in tensor memory)",
                "frac_bf16_peak": ATTN_FLOPS / (attn_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                "shape": f"{M} queries x {WINDOW * TPF} keys x {wl.HEADS} heads x {wl.HEAD_DIM}"},
            "gemm": {"tflops": gemm_tflops, "ms_per_step": gemm_ms,
                     "launches_per_step": gemm_launches,
                     "by_shape_ms": {k: v for k, v in kernel_ms.items() if k.startswith("gemm")}},
            "kernel_ms_per_step": kernel_ms,
            "kernel_ms_note": "CUDA events between every launch of a second graph of the step "
                              "(removes the PDL overlap); quant_act includes the amax passes",
            "configs": configs,
            "library_fp4_gemm_context": library,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": M * D * 2,
                    "d2h_bytes_per_step": M * D * 2, "ms_per_step": ms_e2e / args.steps,
                    "note": "every step's input from pinned host memory and its result back, "
                            "on a copy stream through two staging buffers each way (overlapping "
                            "the neighbouring steps' compute), inside the timed region; the step "
                            "replays the CUDA graph of its C-ABI calls",
                    "eager": {"value": job_throughput(flops_step, world, ms_e2e_eager / args.steps),
                              "ms_per_step": ms_e2e_eager / args.steps,
                              "note": "the same copies, the step's C-ABI calls issued one by one "
                                      "through the Python binding every step (their host-side "
                                      "checks and tensor-map encoding inside the timed region)"}},
            "gpu_launches": step.launches_per_step() * args.steps,
            "clocks": clock_info,
            "device_status": status,
        }
        print(json.dumps(line))
    if dist is not None:
        del graph, graph_b
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=wl.LAYERS)
    ap.add_argument("--ref-rows", type=int, default=16, help="rows per reference-arm step")
    ap.add_argument("--cpu-rows", type=int, default=128, help="rows of the cpu_baseline sample")
    ap.add_argument("--cpu-rows-1core", type=int, default=16,
                    help="rows of the one-core cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the single-call workload timings and the library comparison")
    ap.add_argument("--case", default=None,
                    help="profiling: run one kernel on a step-shaped case --reps times "
                         "(gemm_qkv gemm_out gemm_up gemm_down quant_act quant_ffn quant_amax kv_quant "
                         "kv_quant_fos kv_dequant attention)")
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    if args.case:
        return run_case(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
