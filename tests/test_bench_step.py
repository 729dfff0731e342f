"""Host bookkeeping of the benchmark's one-block step, on the CPU: the calls
one step makes (and so the kernel launches it claims), their operands and
the algorithmic work each call kind is credited with.  The FP4 calls are
replaced by a fake that records them; no device is involved."""
import os
import sys
import types

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_fa(calls):
    fa = types.SimpleNamespace(NVFP4_GLOBAL=1, MXFP4=0, RNE=0, SR=1, ROWWISE=0, COLWISE=1)

    def quantize_dual(x, fmt, rnd, seed, col_hadamard, sign_mask, row_out, col_out, ws):
        calls.append(("dual", tuple(x.shape), fmt, rnd, col_hadamard, sign_mask, row_out, col_out))

    def gemm(a, b, alpha, out=None, ws=None):
        calls.append(("gemm", a, b, alpha, out))

    fa.quantize_dual, fa.gemm = quantize_dual, gemm
    return fa


def _block(layers, T):
    blk = types.SimpleNamespace(ws=None, layers={})
    for name, (cin, cout) in layers.items():
        blk.layers[name] = dict(cin=cin, cout=cout, x=torch.zeros(T, cin), dy=torch.zeros(T, cout),
                                xq=("xq", name), xc=("xc", name), gq=("gq", name), gc=("gc", name),
                                wq=("wq", name), wc=("wc", name), y=("y", name), dx=("dx", name),
                                dw=("dw", name))
    return blk


def test_step_calls_and_launch_count(monkeypatch):
    layers = {"qkv": (64, 96), "o": (64, 64), "gate_up": (64, 128), "down": (128, 64)}
    T = 32
    calls = []
    fa = _fake_fa(calls)
    blk = _block(layers, T)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: None)
    bench.run_step(fa, blk, 0)
    assert len(calls) == 5 * len(layers)
    launches = 0
    for i, name in enumerate(layers):
        fx, g1, fdy, g2, g3 = calls[5 * i:5 * i + 5]
        # forward: X -> NVFP4-global RNE row-wise + saved MXFP4 Hadamard column-wise
        assert fx[0] == "dual" and fx[2:6] == (fa.NVFP4_GLOBAL, fa.RNE, True, bench.SIGN_MASK)
        assert fx[6:] == (("xq", name), ("xc", name))
        assert g1[1:] == (("xq", name), ("wq", name), 1.0, ("y", name))
        # backward: dY -> MXFP4 SR row-wise + MXFP4 Hadamard column-wise
        assert fdy[0] == "dual" and fdy[2:6] == (fa.MXFP4, fa.SR, True, bench.SIGN_MASK)
        assert g2[1:] == (("gq", name), ("wc", name), 1.0, ("dx", name))
        # wgrad: the two Hadamard operands, alpha 1/32 (H H^T = 32 I)
        assert g3[1:] == (("gc", name), ("xc", name), 1.0 / 32, ("dw", name))
        # the NVFP4-global dual producer is two kernels (tensor amax, then the producer)
        launches += 2 + 1 + 1 + 1 + 1
    assert launches == bench.launches_per_step() // len(bench.LAYERS) * len(layers)
    assert bench.launches_per_step() == 6 * len(bench.LAYERS)


def test_algorithmic_work_per_call():
    T = bench.T
    cin, cout = 4096, 28672
    for kind in ("gemm_fwd", "gemm_dgrad", "gemm_wgrad"):
        assert bench.kernel_work(kind, cin, cout) == (2.0 * T * cin * cout, "flop")
    # bf16 read (2 B) + payload (0.5 B) + scale bytes (1/32 MX, 1/16 NV) per element;
    # NVFP4-global reads x twice (tensor amax first)
    assert bench.BYTES_PER_ELEM["mx"] == 2.53125
    assert bench.BYTES_PER_ELEM["nvg"] == 4.5625
    assert bench.BYTES_PER_ELEM["mx_dual"] == 2.0 + 2 * 0.53125
    assert bench.BYTES_PER_ELEM["nvg_dual"] == 2.0 + 2.0 + 0.5625 + 0.53125
    assert bench.kernel_work("quant_fwd_dual", cin, cout) == (bench.BYTES_PER_ELEM["nvg_dual"] * T * cin, "byte")
    assert bench.kernel_work("quant_bwd_dual", cin, cout) == (bench.BYTES_PER_ELEM["mx_dual"] * T * cout, "byte")


def test_whole_block_flops_match_the_layer_shapes():
    per_token = sum(2.0 * ci * co for ci, co in bench.LAYERS.values())
    assert per_token == pytest.approx(0.436e9, rel=0.01)  # 8B-shaped linears, forward
    flops = sum(bench.kernel_work(k, ci, co)[0] for k in ("gemm_fwd", "gemm_dgrad", "gemm_wgrad")
                for ci, co in bench.LAYERS.values())
    assert flops == 3 * per_token * bench.T
