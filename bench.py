"""Benchmark of the FP4 hot path on B200.

One step = the linear layers of one Llama-3-8B-shaped transformer block
(QKV 4096->6144, O 4096->4096, gate+up 4096->28672, down 14336->4096) at 8192
tokens, forward and backward:
  fwd    Y  = X W^T     X quantized row-wise NVFP4-global (RNE), block-scaled GEMM
  dgrad  dX = dY W      dY quantized row-wise MXFP4 with stochastic rounding
  wgrad  dW = dY^T X    dY and X quantized column-wise MXFP4 with the
                        fixed-sign 32-point Hadamard (RNE), GEMM with alpha 1/32
X and dY are each read once by the dual-orientation producer: X gives the
forward operand and the saved wgrad operand, dY the dgrad and wgrad
operands.  Weights are quantized once before timing (row-wise NVFP4-global
for fwd, column-wise MXFP4 for dgrad).  Inputs are synthetic (seeded generators in
workloads.py).  Each step reads ~1.1 GB of bf16 inputs, more than the 126 MB
L2, so no timed iteration finds its inputs in L2.

Prints one JSON line (rank 0).  `value` is whole-job tokens/s; the three
metrics of the FP4 path (fused-quantize GB/s, block-scaled GEMM
TFLOP/s, linear tokens/s) are under "metrics".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fa4|reference]
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "fused quantize GB/s; block-scaled FP4 GEMM TFLOPS; 8B-shaped linear tokens/s"
SIGN_MASK = 0x2545F491
T = workloads.LLAMA8B_TOKENS
LAYERS = workloads.LLAMA8B_LINEARS
BYTES_PER_ELEM = {"mx": 2.0 + 0.5 + 1.0 / 32, "nvg": 2.0 + 2.0 + 0.5 + 1.0 / 16,
                  "nvc": 2.0 + 0.5 + 1.0 / 16 + 4.0 / (128 * 128),
                  "mxnc": 2.0 + 0.5 + 1.0 / 32,
                  # dual producers: one read, both operands written (+ the NVFP4-global amax read)
                  "nvg_dual": 2.0 + 2.0 + (0.5 + 1.0 / 16) + (0.5 + 1.0 / 32),
                  "mx_dual": 2.0 + (0.5 + 1.0 / 32) + (0.5 + 1.0 / 32),
                  # SwiGLU producer, per element of h: gate + up read, NVFP4-CTA-local row
                  # (+ its tile scale) and MXFP4 column operands written
                  "swiglu_nvc_dual": 4.0 + (0.5 + 1.0 / 16 + 4.0 / (128 * 128)) + (0.5 + 1.0 / 32)}


# DRAM bytes (read + write) per launch of the dominant kernel, the MXFP4
# 2-SM GEMM (dgrad and wgrad), averaged over its 8 launches in one step of an
# ncu launch-list capture (dram__bytes_read.sum + dram__bytes_write.sum).
# They hold only for the kernel source they were taken on, identified by its
# SHA-256; after any change the traffic is reported as null until re-taken.
GEMM_SOURCE = os.path.join(ROOT, "fp4_quantization_block_b200", "csrc", "gemm_blockscaled.cu")
DOMINANT_TRAFFIC = {"source_sha256": "dbe6ecf0da0897ad844e6a1170350322d00324d711302de726d31ef33a30b3a5",
                    "bytes_per_launch": 240048064}


def dominant_traffic():
    import hashlib
    try:
        with open(GEMM_SOURCE, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    return DOMINANT_TRAFFIC["bytes_per_launch"] if h == DOMINANT_TRAFFIC["source_sha256"] else None


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# --------------------------------------------------------------- clocks ---

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self) -> dict:
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except Exception:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        loaded = [s for s, r in zip(sm, rows) if r[3] and _f(r[3]) > 250.0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(_f(r[3]) for r in rows)}


def _f(s):
    try:
        return float(s)
    except ValueError:
        return 0.0


# ------------------------------------------------------------ fa4 arm ---

def input_seeds(rank: int, layer: int) -> tuple[int, int, int]:
    """Seeds of (X, dY, W) of one layer on one rank (ranks < 1000 and
    layers < 100 never share a seed)."""
    s = rank * 1000 + 10 * layer
    return s, s + 1, s + 2


class Block:
    """Inputs, quantized weights and output buffers of one block's linears."""

    def __init__(self, fa, seed: int, device):
        self.layers = {}
        for i, (name, (cin, cout)) in enumerate(LAYERS.items()):
            sx, sdy, sw = input_seeds(seed, i)
            x = workloads.act(T, cin, seed=sx, device=device)
            dy = workloads.grad(T, cout, seed=sdy, device=device)
            w = workloads.weight(cout, cin, seed=sw, device=device)
            L = dict(cin=cin, cout=cout, x=x, dy=dy, w=w)
            L["xq"] = fa.empty_qtensor(T, cin, fa.NVFP4_GLOBAL, fa.ROWWISE, device)
            L["gq"] = fa.empty_qtensor(T, cout, fa.MXFP4, fa.ROWWISE, device)
            L["gc"] = fa.empty_qtensor(T, cout, fa.MXFP4, fa.COLWISE, device)
            L["xc"] = fa.empty_qtensor(T, cin, fa.MXFP4, fa.COLWISE, device)
            L["y"] = torch.empty(T, cout, dtype=torch.bfloat16, device=device)
            L["dx"] = torch.empty(T, cin, dtype=torch.bfloat16, device=device)
            L["dw"] = torch.empty(cout, cin, dtype=torch.float32, device=device)
            self.layers[name] = L
        self.ws = fa.workspace(1 << 16, device)

    def quantize_weights(self, fa):
        for L in self.layers.values():
            L["wq"] = fa.quantize(L["w"], fa.NVFP4_GLOBAL, fa.RNE, fa.ROWWISE, ws=self.ws)
            L["wc"] = fa.quantize(L["w"], fa.MXFP4, fa.RNE, fa.COLWISE, ws=self.ws)


KINDS = ["quant_fwd_dual", "gemm_fwd", "quant_bwd_dual", "gemm_dgrad", "gemm_wgrad"]


def run_step(fa, blk: Block, step: int, events=None):
    """One fwd+bwd pass over the block's four linears.  With `events`, a CUDA
    event is recorded after each call (list of (kind, layer, event))."""
    stream = torch.cuda.current_stream()
    seed = 1000003 * (step + 1)

    def mark(kind, name):
        if events is not None:
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            events.append((kind, name, e))

    for name, L in blk.layers.items():
        # forward: X -> NVFP4-global operand + saved MXFP4 Hadamard wgrad operand
        fa.quantize_dual(L["x"], fa.NVFP4_GLOBAL, fa.RNE, 0, col_hadamard=True,
                         sign_mask=SIGN_MASK, row_out=L["xq"], col_out=L["xc"], ws=blk.ws)
        mark("quant_fwd_dual", name)
        fa.gemm(L["xq"], L["wq"], 1.0, out=L["y"], ws=blk.ws)
        mark("gemm_fwd", name)
        # backward: dY -> MXFP4 SR dgrad operand + MXFP4 Hadamard wgrad operand
        fa.quantize_dual(L["dy"], fa.MXFP4, fa.SR, seed, col_hadamard=True, sign_mask=SIGN_MASK,
                         row_out=L["gq"], col_out=L["gc"], ws=blk.ws)
        mark("quant_bwd_dual", name)
        fa.gemm(L["gq"], L["wc"], 1.0, out=L["dx"], ws=blk.ws)
        mark("gemm_dgrad", name)
        fa.gemm(L["gc"], L["xc"], 1.0 / 32, out=L["dw"], ws=blk.ws)
        mark("gemm_wgrad", name)


def kernel_work(kind: str, cin: int, cout: int) -> tuple[float, str]:
    """Algorithmic work of one call: bytes (quantizers) or FLOPs (GEMMs)."""
    if kind.startswith("gemm"):
        return 2.0 * T * cin * cout, "flop"
    if kind == "quant_fwd_dual":
        return BYTES_PER_ELEM["nvg_dual"] * T * cin, "byte"
    if kind == "quant_bwd_dual":
        return BYTES_PER_ELEM["mx_dual"] * T * cout, "byte"
    if kind == "swiglu":  # z read (gate + up) + both operands of h[T, cin] written
        return BYTES_PER_ELEM["swiglu_nvc_dual"] * T * cin, "byte"
    if kind == "quant_fwd_nvg":
        return BYTES_PER_ELEM["nvg"] * T * cin, "byte"
    if kind == "quant_dgrad_mx_sr":
        return BYTES_PER_ELEM["mx"] * T * cout, "byte"
    return BYTES_PER_ELEM["mx"] * T * cout, "byte"  # one Hadamard quantization of dY


def launches_per_step() -> int:
    # per layer: amax + dual (X), GEMM, dual (dY), GEMM, GEMM
    return len(LAYERS) * 6


def quantize_sweep(fa, device, reps: int = 20) -> list[dict]:
    """Quantizer sweep shapes (0.5*t_3 with 1% outlier columns x50): every
    format x rounding x orientation, plus the column-wise Hadamard MXFP4
    quantizer, rotating over enough input copies that the working set
    exceeds L2 (>= 256 MB)."""
    hbm = _peaks()[0]
    out = []
    cases = [(fmt, key, rnd, orient, False)
             for orient in (fa.ROWWISE, fa.COLWISE)
             for fmt, key in ((fa.MXFP4, "mx"), (fa.NVFP4_GLOBAL, "nvg"), (fa.NVFP4_CTA, "nvc"),
                              (fa.MXFP4_NOCLIP, "mxnc"))
             for rnd in (fa.RNE, fa.SR)]
    cases += [(fa.MXFP4, "mx", rnd, fa.COLWISE, True) for rnd in (fa.RNE, fa.SR)]
    for rows, cols in workloads.SWEEP_SHAPES:
        nbuf = max(1, (512 << 20) // (rows * cols * 2))
        xs = [workloads.sweep(rows, cols, seed=i, device=device) for i in range(min(nbuf, 8))]
        ws = fa.workspace(1 << 16, device)
        for fmt, key, rnd, orient, had in cases:
            qs = [fa.empty_qtensor(rows, cols, fmt, orient, device) for _ in xs]

            def call(i):
                if had:
                    fa.hadamard32_quantize(xs[i % len(xs)], SIGN_MASK, rnd, 1, out=qs[i % len(xs)],
                                           ws=ws)
                else:
                    fa.quantize(xs[i % len(xs)], fmt, rnd, orient, 1, out=qs[i % len(xs)], ws=ws)

            for i in range(3):
                call(i)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(reps):
                call(i)
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1000.0 / reps
            gbs = BYTES_PER_ELEM[key] * rows * cols / (us * 1e-6) / 1e9
            out.append({"shape": [rows, cols], "fmt": key, "rnd": "sr" if rnd else "rne",
                        "orient": ("col" if orient else "row") + ("+had32" if had else ""),
                        "us": round(us, 2), "GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)})
            del qs
        del xs
        torch.cuda.empty_cache()
    return out


def gemm_sweep(fa, device, reps: int = 10) -> list[dict]:
    """Block-scaled GEMM of each scale domain (MXFP4, NVFP4-global,
    NVFP4-CTA-local) on the 8B forward shapes (M = 8192 tokens), bf16 out."""
    fp4_peak = 4.0 * _peaks()[1]
    out = []
    for name, (cin, cout) in LAYERS.items():
        a = workloads.act(T, cin, seed=5, device=device)
        b = workloads.weight(cout, cin, seed=6, device=device)
        d = torch.empty(T, cout, dtype=torch.bfloat16, device=device)
        ws = fa.workspace(1 << 16, device)
        for fmt, key in ((fa.MXFP4, "mx"), (fa.NVFP4_GLOBAL, "nvg"), (fa.NVFP4_CTA, "nvc")):
            A, B = fa.quantize(a, fmt, ws=ws), fa.quantize(b, fmt, ws=ws)
            for _ in range(3):
                fa.gemm(A, B, 1.0, out=d, ws=ws)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                fa.gemm(A, B, 1.0, out=d, ws=ws)
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1000.0 / reps
            tf = 2.0 * T * cin * cout / (us * 1e-6) / 1e12
            out.append({"layer": name, "M": T, "N": cout, "K": cin, "fmt": key, "us": round(us, 1),
                        "TFLOPS": round(tf, 1), "frac": round(tf / fp4_peak, 3)})
            del A, B
        del a, b, d
    if fa.check_device_status(ws) != 0:
        raise RuntimeError("device status set during the GEMM sweep")
    torch.cuda.empty_cache()
    return out


def ragged_sweep(fa, device, reps: int = 10) -> list[dict]:
    """Ragged shapes beside the aligned shapes they approximate: the same
    quantizers and GEMM with a row count, a block dimension (K) or GEMM M, N
    and K that are not multiples of 128.  Rates use each shape's own
    elements (FLOPs), so a ragged line's ratio to its aligned one is the cost
    of the masked tiles."""
    hbm = _peaks()[0]
    fp4_peak = 4.0 * _peaks()[1]
    ws = fa.workspace(1 << 16, device)
    out = []

    def timed(call):
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            call()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1000.0 / reps

    # quantizers: (label, rows, cols, kind)
    qcases = [("mx row rne", 8192, 14336, "row"), ("mx row rne", 8191, 14336, "row"),
              ("mx row rne", 8192, 14304, "row"),
              ("mx col+had32 rne", 8192, 14336, "had"), ("mx col+had32 rne", 8160, 14336, "had"),
              ("dual mx sr + col had32", 8192, 4096, "dual"),
              ("dual mx sr + col had32", 8160, 4096, "dual")]
    for label, rows, cols, kind in qcases:
        x = workloads.sweep(rows, cols, seed=3, device=device)
        if kind == "row":
            q = fa.empty_qtensor(rows, cols, fa.MXFP4, fa.ROWWISE, device)
            us = timed(lambda: fa.quantize(x, fa.MXFP4, fa.RNE, fa.ROWWISE, 0, out=q, ws=ws))
            bpe = BYTES_PER_ELEM["mx"]
        elif kind == "had":
            q = fa.empty_qtensor(rows, cols, fa.MXFP4, fa.COLWISE, device)
            us = timed(lambda: fa.hadamard32_quantize(x, SIGN_MASK, fa.RNE, 0, out=q, ws=ws))
            bpe = BYTES_PER_ELEM["mx"]
        else:
            r = fa.empty_qtensor(rows, cols, fa.MXFP4, fa.ROWWISE, device)
            c = fa.empty_qtensor(rows, cols, fa.MXFP4, fa.COLWISE, device)
            us = timed(lambda: fa.quantize_dual(x, fa.MXFP4, fa.SR, 1, col_hadamard=True,
                                                sign_mask=SIGN_MASK, row_out=r, col_out=c, ws=ws))
            bpe = BYTES_PER_ELEM["mx_dual"]
        gbs = bpe * rows * cols / (us * 1e-6) / 1e9
        out.append({"op": label, "shape": [rows, cols], "us": round(us, 2), "GBps": round(gbs, 1),
                    "frac_hbm": round(gbs / hbm, 3)})
        del x
    # GEMM (MXFP4, bf16 out): the gate+up forward shape and a ragged neighbour
    for M, N, K in ((8192, 28672, 4096), (8000, 28600, 4064)):
        a = workloads.act(M, K, seed=5, device=device)
        b = workloads.weight(N, K, seed=6, device=device)
        A, B = fa.quantize(a, fa.MXFP4, ws=ws), fa.quantize(b, fa.MXFP4, ws=ws)
        d = fa.gemm(A, B, 1.0, out_dtype=torch.bfloat16, ws=ws)
        us = timed(lambda: fa.gemm(A, B, 1.0, out=d, ws=ws))
        tf = 2.0 * M * N * K / (us * 1e-6) / 1e12
        out.append({"op": "gemm mx", "shape": [M, N, K], "us": round(us, 1), "TFLOPS": round(tf, 1),
                    "frac": round(tf / fp4_peak, 3)})
        del a, b, A, B, d
    if fa.check_device_status(ws) != 0:
        raise RuntimeError("device status set during the ragged sweep")
    torch.cuda.empty_cache()
    return out


def epilogue_quant_run(fa, device, reps: int = 10) -> dict:
    """The gate+up forward GEMM followed by the MXFP4 quantization of its bf16
    output: separate calls against the quantizer fused into the GEMM epilogue
    (with and without storing the bf16 output)."""
    cin, cout = LAYERS["gate_up"]
    x = workloads.act(T, cin, seed=7, device=device)
    w = workloads.weight(cout, cin, seed=8, device=device)
    ws = fa.workspace(1 << 16, device)
    A, B = fa.quantize(x, fa.NVFP4_GLOBAL, ws=ws), fa.quantize(w, fa.NVFP4_GLOBAL, ws=ws)
    d = torch.empty(T, cout, dtype=torch.bfloat16, device=device)
    q = fa.empty_qtensor(T, cout, fa.MXFP4, fa.ROWWISE, device)
    runs = {"separate": lambda: (fa.gemm(A, B, 1.0, out=d, ws=ws),
                                 fa.quantize(d, fa.MXFP4, out=q, ws=ws)),
            "fused": lambda: fa.gemm_mxout(A, B, 1.0, out=d, qout=q, ws=ws),
            "fused_no_bf16": lambda: fa.gemm_mxout(A, B, 1.0, store_d=False, qout=q, ws=ws)}
    res = {"shape": [T, cout, cin]}
    for name, fn in runs.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        res[name + "_us"] = round(e0.elapsed_time(e1) * 1000.0 / reps, 1)
    if fa.check_device_status(ws) != 0:
        raise RuntimeError("device status set during the epilogue-quantization run")
    return res


def swiglu_quant_run(fa, device, reps: int = 10) -> dict:
    """The down projection's input from the gate+up output z[8192, 2 x 14336]:
    the SwiGLU producer fused with its quantizer (row-wise CTA-local NVFP4 and
    column-wise MXFP4 with the Hadamard, h never written) against the
    unfused route (torch's bf16 silu(gate) * up writing h, then the dual
    quantizer reading it).  GB/s over the fused producer's algorithmic bytes:
    z read (4 B per element of h) + both operands written."""
    F = LAYERS["down"][0]
    z = workloads.act(T, 2 * F, seed=9, device=device)
    rq = fa.empty_qtensor(T, F, fa.NVFP4_CTA, fa.ROWWISE, device)
    cq = fa.empty_qtensor(T, F, fa.MXFP4, fa.COLWISE, device)
    h = torch.empty(T, F, dtype=torch.bfloat16, device=device)
    ws = fa.workspace(1 << 16, device)

    def unfused():
        torch.mul(torch.nn.functional.silu(z[:, :F]), z[:, F:], out=h)
        fa.quantize_dual(h, fa.NVFP4_CTA, fa.RNE, 0, True, SIGN_MASK, row_out=rq, col_out=cq, ws=ws)

    runs = {"fused": lambda: fa.swiglu_quantize(z, fa.NVFP4_CTA, fa.RNE, 0, col=True,
                                                sign_mask=SIGN_MASK, row_out=rq, col_out=cq),
            "unfused": unfused}
    res = {"shape": [T, F], "row": "NVFP4-CTA-local RNE", "col": "MXFP4 Hadamard RNE"}
    for name, fn in runs.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        res[name + "_us"] = round(e0.elapsed_time(e1) * 1000.0 / reps, 1)
    nbytes = BYTES_PER_ELEM["swiglu_nvc_dual"] * T * F
    res["fused_GBps"] = round(nbytes / (res["fused_us"] * 1e-6) / 1e9, 1)
    return res


STACK_LAYERS = 32
STACK_BF16_LAYERS = 4          # the last four blocks keep bf16 linears
STACK_TOKENS = 2 * T           # sequence 8192 x batch 2


def stack_run(fa, device, steps: int = 3, warmup: int = 3) -> dict:
    """The linears of a 32-layer Llama-3-8B-shaped stack, forward then
    backward, at 16384 tokens: layers 0-27 on the FP4 path (the block step's
    calls), layers 28-31 as bf16 cuBLAS matmuls through torch.  Every layer
    has its own seeded weights (FP4 layers keep only their quantized copies);
    activations and gradients are one buffer per linear shape, shared by the
    layers (each is larger than L2 or read beside others that are, so no
    layer finds its inputs in L2).  No attention, normalisation or optimizer:
    the stack's linears only."""
    Ts = STACK_TOKENS
    n_fp4 = STACK_LAYERS - STACK_BF16_LAYERS
    ws = fa.workspace(1 << 16, device)
    act = {}
    for i, (name, (cin, cout)) in enumerate(LAYERS.items()):
        a = dict(cin=cin, cout=cout,
                 x=workloads.act(Ts, cin, seed=70000 + i, device=device),
                 dy=workloads.grad(Ts, cout, seed=70010 + i, device=device))
        a["xq"] = fa.empty_qtensor(Ts, cin, fa.NVFP4_GLOBAL, fa.ROWWISE, device)
        a["xc"] = fa.empty_qtensor(Ts, cin, fa.MXFP4, fa.COLWISE, device)
        a["gq"] = fa.empty_qtensor(Ts, cout, fa.MXFP4, fa.ROWWISE, device)
        a["gc"] = fa.empty_qtensor(Ts, cout, fa.MXFP4, fa.COLWISE, device)
        a["y"] = torch.empty(Ts, cout, dtype=torch.bfloat16, device=device)
        a["dx"] = torch.empty(Ts, cin, dtype=torch.bfloat16, device=device)
        a["dw"] = torch.empty(cout, cin, dtype=torch.float32, device=device)
        a["dw16"] = torch.empty(cout, cin, dtype=torch.bfloat16, device=device)
        act[name] = a
    weights = []
    t_wq = time.perf_counter()
    for layer in range(STACK_LAYERS):
        lw = {}
        for i, (name, (cin, cout)) in enumerate(LAYERS.items()):
            w = workloads.weight(cout, cin, seed=80000 + 10 * layer + i, device=device)
            if layer < n_fp4:
                lw[name] = (fa.quantize(w, fa.NVFP4_GLOBAL, fa.RNE, fa.ROWWISE, ws=ws),
                            fa.quantize(w, fa.MXFP4, fa.RNE, fa.COLWISE, ws=ws))
                del w
            else:
                lw[name] = w
        weights.append(lw)
    torch.cuda.synchronize()
    t_wq = time.perf_counter() - t_wq

    def fwd(layer):
        for name, a in act.items():
            if layer < n_fp4:
                wq, _ = weights[layer][name]
                fa.quantize_dual(a["x"], fa.NVFP4_GLOBAL, fa.RNE, 0, col_hadamard=True,
                                 sign_mask=SIGN_MASK, row_out=a["xq"], col_out=a["xc"], ws=ws)
                fa.gemm(a["xq"], wq, 1.0, out=a["y"], ws=ws)
            else:
                torch.matmul(a["x"], weights[layer][name].t(), out=a["y"])

    def bwd(layer, seed):
        for name, a in act.items():
            if layer < n_fp4:
                _, wc = weights[layer][name]
                fa.quantize_dual(a["dy"], fa.MXFP4, fa.SR, seed, col_hadamard=True,
                                 sign_mask=SIGN_MASK, row_out=a["gq"], col_out=a["gc"], ws=ws)
                fa.gemm(a["gq"], wc, 1.0, out=a["dx"], ws=ws)
                fa.gemm(a["gc"], a["xc"], 1.0 / 32, out=a["dw"], ws=ws)
            else:
                w = weights[layer][name]
                torch.matmul(a["dy"], w, out=a["dx"])
                torch.matmul(a["dy"].t(), a["x"], out=a["dw16"])

    stream = torch.cuda.current_stream(device)
    marks = []

    def step(s, timed):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)] if timed else None
        if timed:
            ev[0].record(stream)
        for layer in range(STACK_LAYERS):
            fwd(layer)
            if timed and layer == n_fp4 - 1:
                ev[1].record(stream)
        if timed:
            ev[2].record(stream)
        for layer in reversed(range(STACK_LAYERS)):
            bwd(layer, 1000003 * (s + 1) + layer)
            if timed and layer == n_fp4:
                ev[3].record(stream)
        if timed:
            ev[4].record(stream)
            marks.append(ev)

    for s in range(warmup):
        step(s, False)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        start.record(stream)
        for s in range(steps):
            step(warmup + s, True)
        end.record(stream)
        torch.cuda.synchronize()
    if fa.check_device_status(ws) != 0:
        raise RuntimeError("device status set during the stack run")
    ms = start.elapsed_time(end) / steps
    fp4_ms = sum(e[0].elapsed_time(e[1]) + e[3].elapsed_time(e[4]) for e in marks) / steps
    bf16_ms = sum(e[1].elapsed_time(e[2]) + e[2].elapsed_time(e[3]) for e in marks) / steps
    flop_layer = 3 * 2.0 * Ts * sum(cin * cout for cin, cout in LAYERS.values())
    return {"workload": "llama3-8b-32-layer-linear-stack-fwd-bwd", "tokens": Ts,
            "layers": STACK_LAYERS, "bf16_layers": f"{n_fp4}-{STACK_LAYERS - 1}",
            "steps": steps, "warmup": warmup, "ms_per_step": round(ms, 3),
            "tokens_per_s": round(Ts / (ms * 1e-3), 1),
            "fp4_layers_ms": round(fp4_ms, 3),
            "fp4_layers_TFLOPS": round(n_fp4 * flop_layer / (fp4_ms * 1e-3) / 1e12, 1),
            "bf16_layers_ms": round(bf16_ms, 3),
            "bf16_layers_TFLOPS": round(STACK_BF16_LAYERS * flop_layer / (bf16_ms * 1e-3) / 1e12, 1),
            "weight_quantize_s": round(t_wq, 3), "clocks": clk.summary(),
            "scope": "linears only (no attention, norms or optimizer); activations shared by layers"}


def e2e_run(fa, blk: Block, steps: int, device) -> dict:
    """Same step through the public training-form linear calls
    (linear_fwd_save, linear_bwd) with host (pinned) inputs and outputs: the
    H2D copy of X and dY and the D2H copy of Y, dX and dW of every layer are
    inside the timed region.  Copies run on their own streams, layer by
    layer, so the H2D of one layer, the kernels of another and the D2H of a
    third overlap (PCIe is full duplex); events order each buffer's reuse."""
    host = {}
    h2d = d2h = 0
    for name, L in blk.layers.items():
        host[name] = dict(x=L["x"].cpu().pin_memory(), dy=L["dy"].cpu().pin_memory(),
                          y=torch.empty_like(L["y"], device="cpu").pin_memory(),
                          dx=torch.empty_like(L["dx"], device="cpu").pin_memory(),
                          dw=torch.empty_like(L["dw"], device="cpu").pin_memory())
        h2d += L["x"].numel() * 2 + L["dy"].numel() * 2
        d2h += L["y"].numel() * 2 + L["dx"].numel() * 2 + L["dw"].numel() * 4
    wsz = max(fa.linear_ws_bytes(k, T, cin, cout, fa.NVFP4_GLOBAL if k == 3 else fa.MXFP4)
              for k in (3, 4) for cin, cout in LAYERS.values())
    ws = fa.workspace(wsz, device)
    comp = torch.cuda.current_stream(device)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {name: {"loaded": torch.cuda.Event(), "computed": torch.cuda.Event(),
                 "stored": torch.cuda.Event(), "used": False} for name in blk.layers}

    def one(step):
        for name, L in blk.layers.items():
            H, E = host[name], ev[name]
            with torch.cuda.stream(s_in):
                if E["used"]:
                    s_in.wait_event(E["computed"])  # the last step's kernels have read x, dy
                L["x"].copy_(H["x"], non_blocking=True)
                L["dy"].copy_(H["dy"], non_blocking=True)
                E["loaded"].record(s_in)
            comp.wait_event(E["loaded"])
            if E["used"]:
                comp.wait_event(E["stored"])  # the last step's outputs have left the device
            fa.linear_fwd_save(L["x"], L["wq"], fa.NVFP4_GLOBAL, SIGN_MASK, out=L["y"],
                               xcol=L["xc"], ws=ws)
            fa.linear_bwd(L["dy"], L["wc"], L["xc"], fa.MXFP4, fa.SR, seed=step,
                          sign_mask=SIGN_MASK, dx=L["dx"], dw=L["dw"], ws=ws)
            E["computed"].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(E["computed"])
                H["y"].copy_(L["y"], non_blocking=True)
                H["dx"].copy_(L["dx"], non_blocking=True)
                H["dw"].copy_(L["dw"], non_blocking=True)
                E["stored"].record(s_out)
            E["used"] = True

    one(0)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for s in range(steps):
        one(s + 1)
    comp.wait_stream(s_out)
    e1.record(comp)
    torch.cuda.synchronize()
    if fa.check_device_status(ws) != 0:
        raise RuntimeError("device status set during the e2e run")
    ms = e0.elapsed_time(e1) / steps
    return {"ms_per_step": ms, "tokens_per_s": T / (ms * 1e-3), "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h}


_ORACLE_WEIGHTS = None


def _oracle_weights():
    """Weights quantized by the oracle and expanded to binary64 block values,
    once (the GPU arm also quantizes weights before timing)."""
    global _ORACLE_WEIGHTS
    if _ORACLE_WEIGHTS is None:
        import oracle as O
        _ORACLE_WEIGHTS = {}
        for i, (name, (cin, cout)) in enumerate(LAYERS.items()):
            w = workloads.weight(cout, cin, seed=10 * i + 2)
            wq = O.quantize(w, O.NVFP4_GLOBAL)
            wc = O.quantize(w, O.MXFP4, orient=O.COLWISE)
            _ORACLE_WEIGHTS[name] = (wq, O.dequantize_blocks(wq), O.dequantize_blocks(wc))
    return _ORACLE_WEIGHTS


def cpu_baseline(sample_tokens: int = 128) -> dict:
    """The oracle as it stands on a bounded sample of the same step:
    `sample_tokens` tokens through the four linears, fwd + dgrad + wgrad.
    Quantization by the C oracle; each GEMM is the oracle's binary64 block
    values summed by a numpy binary64 matmul (its large-shape path), with the
    weight operands prepared once outside the timed part."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count() or 1
    S = sample_tokens
    prepared = _oracle_weights()
    inputs = {name: (workloads.act(S, cin, seed=10 * i), workloads.grad(S, cout, seed=10 * i + 1))
              for i, (name, (cin, cout)) in enumerate(LAYERS.items())}
    t0 = time.perf_counter()
    for name in LAYERS:
        x, dy = inputs[name]
        wq, wq_blocks, wc_blocks = prepared[name]
        xq = O.quantize(x, O.NVFP4_GLOBAL)                                       # fwd
        _ = (O.dequantize_blocks(xq) @ wq_blocks.T) * (float(xq.ts[0]) * float(wq.ts[0]))
        gq = O.quantize(dy, O.MXFP4, O.SR, seed=1)                               # dgrad
        _ = O.dequantize_blocks(gq) @ wc_blocks.T
        gc = O.quantize(dy, O.MXFP4, O.RNE, O.COLWISE, hadamard_mask=SIGN_MASK)  # wgrad
        xc = O.quantize(x, O.MXFP4, O.RNE, O.COLWISE, hadamard_mask=SIGN_MASK)
        _ = O.gemm_sampled(gc, xc, 1.0 / 32)
    dt = time.perf_counter() - t0
    return {"value": round(S / dt, 3), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{S} tokens through the block's 4 linears fwd+dgrad+wgrad, {dt:.2f} s "
                      f"(weights prepared by the oracle before timing)"}


def max_over_ranks(x: float, device) -> float:
    """Max of x over the ranks of the default process group (x itself when
    there is no group or one rank).  Every rank must call it."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def bench_config(world: int) -> dict:
    return {"workload": "llama3-8b-block-linears-fwd-bwd", "tokens": T,
            "layers": {k: list(v) for k, v in LAYERS.items()},
            "fwd": "NVFP4-global RNE", "dgrad": "MXFP4 row-wise SR",
            "wgrad": "MXFP4 column-wise fixed-sign Hadamard-32 RNE, alpha 1/32",
            "producers": "dual-orientation: one read each of X and dY",
            "parallelism": f"replicas x{world}", "l2": "inputs > L2 (1.1 GB bf16 read per step)"}


def whole_job_tokens_per_s(world: int, ms_step: float) -> float:
    """Weak scaling: every rank runs its own replica of the step on T tokens,
    so the job processes world * T tokens in the slowest rank's step time."""
    return world * T / (ms_step * 1e-3)


def init_ranks(world: int, device, backend: str = "nccl"):
    """One process per GPU; a short timeout so ranks that wait on a dead peer
    end with an error instead of hanging."""
    if world <= 1:
        return
    import datetime
    kw = {"device_id": device} if backend == "nccl" else {}
    torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)


def fa4_arm(args, rank, world, device) -> dict | None:
    import fp4_quantization_block_b200 as fa
    fa.lib()
    hbm, bf16, bf16s, peak_src = _peaks()
    blk = Block(fa, seed=rank, device=device)
    t_wq = time.perf_counter()
    blk.quantize_weights(fa)
    torch.cuda.synchronize()
    t_wq = time.perf_counter() - t_wq

    for s in range(args.warmup):
        run_step(fa, blk, s)
    torch.cuda.synchronize()
    if fa.check_device_status(blk.ws) != 0:
        raise RuntimeError("device status set during warm-up")

    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # the timed region: the steps alone (an event between calls would cost
    # the GPU a few microseconds at each of the step's 24 kernel boundaries)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        start.record(stream)
        for s in range(args.steps):
            run_step(fa, blk, args.warmup + s)
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    if fa.check_device_status(blk.ws) != 0:
        raise RuntimeError("device status set during the timed region")
    ms_total = max_over_ranks(start.elapsed_time(end), device)
    ms_step = ms_total / args.steps

    # the per-call breakdown: the same steps again, an event after each call
    events = []
    t0 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for s in range(args.steps):
        events.append(("step_begin", None, None))
        run_step(fa, blk, args.warmup + args.steps + s, events)
    torch.cuda.synchronize()
    if fa.check_device_status(blk.ws) != 0:
        raise RuntimeError("device status set during the instrumented steps")

    # per-kind durations from consecutive events (previous event = start of call)
    per_kind = {k: [0.0, 0.0] for k in KINDS}  # ms, work
    prev = t0
    for kind, name, ev in events:
        if kind == "step_begin":
            continue
        dt = prev.elapsed_time(ev)
        cin, cout = LAYERS[name]
        work, _ = kernel_work(kind, cin, cout)
        per_kind[kind][0] += dt
        per_kind[kind][1] += work
        prev = ev
    gemm_ms = sum(per_kind[k][0] for k in KINDS if k.startswith("gemm"))
    gemm_flop = sum(per_kind[k][1] for k in KINDS if k.startswith("gemm"))
    q_ms = sum(per_kind[k][0] for k in KINDS if k.startswith("quant"))
    q_bytes = sum(per_kind[k][1] for k in KINDS if k.startswith("quant"))
    gemm_tflops = gemm_flop / (gemm_ms * 1e-3) / 1e12
    # dominant kernel: the MXFP4 2-SM GEMM (dgrad + wgrad launches)
    dom_ms = per_kind["gemm_dgrad"][0] + per_kind["gemm_wgrad"][0]
    dom_flop = per_kind["gemm_dgrad"][1] + per_kind["gemm_wgrad"][1]
    dom_tflops = dom_flop / (dom_ms * 1e-3) / 1e12
    q_gbs = q_bytes / (q_ms * 1e-3) / 1e9
    fp4_peak = 4.0 * bf16  # dense FP4 = 4 x dense bf16 (nominal ratio 9 / 2.25 PFLOP/s)
    breakdown = {k: {"ms_per_step": round(v[0] / args.steps, 4),
                     ("TFLOPS" if k.startswith("gemm") else "GBps"):
                         round(v[1] / (v[0] * 1e-3) / (1e12 if k.startswith("gemm") else 1e9), 1)}
                 for k, v in per_kind.items()}
    clocks = clk.summary()

    # end to end on every rank (each GPU has its own host link): whole-job
    # tokens/s from the slowest rank, like the device-timed value
    e2e = e2e_run(fa, blk, max(2, min(args.steps, 5)), device)
    e2e_ms = max_over_ranks(e2e["ms_per_step"], device)
    e2e["ms_per_step"] = e2e_ms
    e2e["tokens_per_s"] = whole_job_tokens_per_s(world, e2e_ms)
    e2e["h2d_bytes_per_step"] *= world  # all ranks' copies, like the whole-job tokens
    e2e["d2h_bytes_per_step"] *= world
    result = None
    if rank == 0:
        # single-GPU microbenchmarks and the oracle baseline: one GPU only
        solo = world == 1 and not args.quick
        sweep = quantize_sweep(fa, device) if solo else []
        gsweep = gemm_sweep(fa, device) if solo else []
        epiq = epilogue_quant_run(fa, device) if solo else {}
        swq = swiglu_quant_run(fa, device) if solo else {}
        ragged = []
        if solo:
            try:
                ragged = ragged_sweep(fa, device)
            except (RuntimeError, torch.cuda.OutOfMemoryError) as e:
                ragged = [{"error": f"{type(e).__name__}: {e}"}]
        stack = {}
        if solo or args.stack:
            try:
                stack = stack_run(fa, device)
            except (RuntimeError, torch.cuda.OutOfMemoryError) as e:
                stack = {"error": f"{type(e).__name__}: {e}"}
        cpu = cpu_baseline() if (world == 1 and not args.no_cpu_baseline) else None
        tok_s = whole_job_tokens_per_s(world, ms_step)
        result = {
            "metric": METRIC,
            "value": round(tok_s, 1),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "e2m1",
            "data": "synthetic (seeded generators: act N(0,1)+0.5% channels x20, W N(0,0.02), "
                    "dY N(0,1e-3) x lognormal rows)",
            "config": bench_config(world),
            "metrics": {"linear_tokens_per_s": round(tok_s, 1),
                        "fp4_gemm_TFLOPS": round(gemm_tflops, 1),
                        "fused_quantize_GBps": round(q_gbs, 1),
                        "breakdown": breakdown,
                        "weight_quantize_s": round(t_wq, 4),
                        "quantize_sweep": sweep,
                        "gemm_sweep": gsweep,
                        "gemm_epilogue_mxfp4": epiq,
                        "swiglu_quantize": swq,
                        "ragged_sweep": ragged,
                        "linear_stack": stack},
            "roofline": {"bound": "tensor", "achieved": round(dom_tflops, 1),
                         "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                         "frac": round(dom_tflops / fp4_peak, 4), "traffic": dominant_traffic(),
                         "kernel": "gemm_st_kernel<MXFP4, 256, 2-SM> (dgrad + wgrad, 8 launches "
                                   "per step; achieved = their FLOPs / their event time in the "
                                   "instrumented pass of the same steps)",
                         "peak_src": f"{peak_src} bf16 burst {bf16} x 4 (nominal dense FP4/bf16 "
                                     f"ratio 9/2.25), of {peak_src}"},
            "roofline_all_gemms": {"achieved": round(gemm_tflops, 1), "unit": "TFLOP/s",
                                   "frac": round(gemm_tflops / fp4_peak, 4)},
            "roofline_quantize": {"bound": "hbm", "achieved": round(q_gbs, 1), "peak": hbm,
                                  "unit": "GB/s", "frac": round(q_gbs / hbm, 4),
                                  "peak_src": f"{peak_src} HBM copy"},
            "e2e": {"value": round(e2e["tokens_per_s"], 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                    "d2h_bytes_per_step": e2e["d2h_bytes_per_step"],
                    "ms_per_step": round(e2e["ms_per_step"], 3)},
            "gpu_launches": launches_per_step() * args.steps,  # in the timed region
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        del bf16s
    return result


def profile_arm(args, device) -> dict:
    """Run one call kind on one layer only (warm-up + steps launches), for a
    profiler capture of a single kernel: --profile KIND:LAYER, KIND one of
    gemm_fwd, gemm_fwd_nvc, gemm_dgrad, gemm_wgrad, quant_fwd_nvg, quant_dgrad_mx_sr,
    quant_wgrad_had, quant_fwd_dual, quant_bwd_dual, swiglu (LAYER = down: the
    SwiGLU producer of the down projection's input, NVFP4-CTA-local row +
    MXFP4 Hadamard column)."""
    import fp4_quantization_block_b200 as fa
    kind, layer = args.profile.split(":")
    cin, cout = LAYERS[layer]
    x = workloads.act(T, cin, seed=1, device=device)
    dy = workloads.grad(T, cout, seed=2, device=device)
    w = workloads.weight(cout, cin, seed=3, device=device)
    ws = fa.workspace(1 << 16, device)
    if kind == "gemm_fwd":
        a, b = fa.quantize(x, fa.NVFP4_GLOBAL, ws=ws), fa.quantize(w, fa.NVFP4_GLOBAL, ws=ws)
        out = torch.empty(T, cout, dtype=torch.bfloat16, device=device)
        call = lambda: fa.gemm(a, b, 1.0, out=out, ws=ws)
    elif kind == "gemm_fwd_nvc":
        a, b = fa.quantize(x, fa.NVFP4_CTA, ws=ws), fa.quantize(w, fa.NVFP4_CTA, ws=ws)
        out = torch.empty(T, cout, dtype=torch.bfloat16, device=device)
        call = lambda: fa.gemm(a, b, 1.0, out=out, ws=ws)
    elif kind == "gemm_dgrad":
        a = fa.quantize(dy, fa.MXFP4, fa.SR, seed=1, ws=ws)
        b = fa.quantize(w, fa.MXFP4, orient=fa.COLWISE, ws=ws)
        out = torch.empty(T, cin, dtype=torch.bfloat16, device=device)
        call = lambda: fa.gemm(a, b, 1.0, out=out, ws=ws)
    elif kind == "gemm_wgrad":
        a = fa.hadamard32_quantize(dy, SIGN_MASK, ws=ws)
        b = fa.hadamard32_quantize(x, SIGN_MASK, ws=ws)
        out = torch.empty(cout, cin, dtype=torch.float32, device=device)
        call = lambda: fa.gemm(a, b, 1.0 / 32, out=out, ws=ws)
    elif kind == "quant_fwd_nvg":
        q = fa.empty_qtensor(T, cin, fa.NVFP4_GLOBAL, fa.ROWWISE, device)
        call = lambda: fa.quantize(x, fa.NVFP4_GLOBAL, out=q, ws=ws)
    elif kind == "quant_dgrad_mx_sr":
        q = fa.empty_qtensor(T, cout, fa.MXFP4, fa.ROWWISE, device)
        call = lambda: fa.quantize(dy, fa.MXFP4, fa.SR, seed=1, out=q, ws=ws)
    elif kind == "quant_wgrad_had":
        q = fa.empty_qtensor(T, cout, fa.MXFP4, fa.COLWISE, device)
        call = lambda: fa.hadamard32_quantize(dy, SIGN_MASK, out=q, ws=ws)
    elif kind == "quant_fwd_dual":
        qr = fa.empty_qtensor(T, cin, fa.NVFP4_GLOBAL, fa.ROWWISE, device)
        qc = fa.empty_qtensor(T, cin, fa.MXFP4, fa.COLWISE, device)
        call = lambda: fa.quantize_dual(x, fa.NVFP4_GLOBAL, fa.RNE, 0, True, SIGN_MASK,
                                        row_out=qr, col_out=qc, ws=ws)
    elif kind == "quant_bwd_dual":
        qr = fa.empty_qtensor(T, cout, fa.MXFP4, fa.ROWWISE, device)
        qc = fa.empty_qtensor(T, cout, fa.MXFP4, fa.COLWISE, device)
        call = lambda: fa.quantize_dual(dy, fa.MXFP4, fa.SR, 1, True, SIGN_MASK,
                                        row_out=qr, col_out=qc, ws=ws)
    elif kind == "swiglu":
        z = workloads.act(T, 2 * cin, seed=9, device=device)
        qr = fa.empty_qtensor(T, cin, fa.NVFP4_CTA, fa.ROWWISE, device)
        qc = fa.empty_qtensor(T, cin, fa.MXFP4, fa.COLWISE, device)
        call = lambda: fa.swiglu_quantize(z, fa.NVFP4_CTA, fa.RNE, 0, col=True, sign_mask=SIGN_MASK,
                                          row_out=qr, col_out=qc)
    else:
        raise SystemExit(f"unknown kind {kind}")
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    if fa.check_device_status(ws) != 0:
        raise RuntimeError("device status set")
    us = e0.elapsed_time(e1) * 1000 / args.steps
    work, unit = kernel_work(kind, cin, cout)
    rate = work / (us * 1e-6) / (1e12 if unit == "flop" else 1e9)
    return {"profile": args.profile, "us_per_call": round(us, 2),
            ("TFLOPS" if unit == "flop" else "GBps"): round(rate, 1)}


# ------------------------------------------------------ reference arm ---

def reference_arm(args) -> dict:
    """The oracle as it stands, on the host cores: each step is a bounded
    sample of the same workload (64 tokens through the block's linears)."""
    _oracle_weights()
    for _ in range(args.warmup):
        cpu_baseline(sample_tokens=32)  # the smallest sample the 32-token MXFP4 blocks allow
    t0 = time.perf_counter()
    res = None
    for _ in range(args.steps):
        res = cpu_baseline(sample_tokens=64)
    dt = (time.perf_counter() - t0) / args.steps
    value = 64 / dt
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": res["cores"],
                             "kind": "oracle", "sample": "64 tokens per step through the block's 4 linears"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="fa4", choices=["fa4", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true",
                    help="skip the single-GPU sweeps and the 32-layer stack")
    ap.add_argument("--stack", action="store_true",
                    help="run the 32-layer linear stack even with --quick")
    ap.add_argument("--profile", default=None,
                    help="KIND:LAYER -- run only that call (for a single-kernel profiler capture)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)), flush=True)
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_ranks(world, device)
    if args.profile:
        print(json.dumps(profile_arm(args, device)), flush=True)
        return
    try:
        res = fa4_arm(args, rank, world, device)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
