"""Host bookkeeping of the benchmark's 32-layer linear stack, on the CPU.

The FP4 calls and the CUDA events are replaced by fakes that advance a fake
device clock by a fixed cost per call, so the test can check what the stack
runner launches (which layers take the FP4 path, in which order, with which
operands) and that its per-part times and FLOP rates come out of the right
events.  Shapes are shrunk; the arithmetic of the FP4 path is not involved."""
import os
import sys
import types

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

COST = {"quantize_dual": 0.5, "gemm": 1.0, "matmul": 2.0}


class FakeClock:
    def __init__(self):
        self.now = 0.0


class FakeEvent:
    clock = None

    def __init__(self, enable_timing=False):
        self.t = None

    def record(self, stream=None):
        self.t = FakeEvent.clock.now

    def elapsed_time(self, other):
        return other.t - self.t


def _fake_fa(clock, calls):
    fa = types.SimpleNamespace(NVFP4_GLOBAL=1, MXFP4=0, RNE=0, SR=1, ROWWISE=0, COLWISE=1)

    def tagged(tag):
        return types.SimpleNamespace(tag=tag)

    fa.workspace = lambda n, device: torch.zeros(n, dtype=torch.uint8)
    fa.empty_qtensor = lambda r, c, fmt, orient, device: tagged(("q", r, c, fmt, orient))
    fa.quantize = lambda w, fmt, rnd, orient, ws=None: tagged(("w", tuple(w.shape), fmt, orient))
    fa.check_device_status = lambda ws: 0

    def quantize_dual(x, fmt, rnd, seed, col_hadamard, sign_mask, row_out, col_out, ws):
        calls.append(("dual", tuple(x.shape), fmt, rnd, seed, col_hadamard))
        clock.now += COST["quantize_dual"]

    def gemm(a, b, alpha, out=None, ws=None):
        calls.append(("gemm", a.tag, b.tag, alpha, tuple(out.shape), out.dtype))
        clock.now += COST["gemm"]

    fa.quantize_dual = quantize_dual
    fa.gemm = gemm
    return fa


@pytest.fixture
def small_stack(monkeypatch):
    clock = FakeClock()
    FakeEvent.clock = clock
    calls = []
    layers = {"qkv": (64, 96), "o": (64, 64), "gate_up": (64, 128), "down": (128, 64)}
    monkeypatch.setattr(bench, "LAYERS", layers)
    monkeypatch.setattr(bench, "STACK_TOKENS", 32)
    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: None)
    real_matmul = torch.matmul

    def matmul(a, b, out=None):
        calls.append(("matmul", tuple(a.shape), tuple(b.shape)))
        clock.now += COST["matmul"]
        return real_matmul(a, b, out=out)

    monkeypatch.setattr(torch, "matmul", matmul)
    return _fake_fa(clock, calls), calls, layers


def test_stack_launches_and_accounting(small_stack):
    fa, calls, layers = small_stack
    steps, warmup = 2, 3
    res = bench.stack_run(fa, torch.device("cpu"), steps=steps, warmup=warmup)
    n_fp4 = bench.STACK_LAYERS - bench.STACK_BF16_LAYERS
    nl = len(layers)

    # per step: FP4 layers 2 calls fwd + 3 bwd per linear, bf16 layers 1 + 2 matmuls
    per_step = n_fp4 * nl * 5 + bench.STACK_BF16_LAYERS * nl * 3
    assert len(calls) == per_step * (steps + warmup)

    # one step's order: forward over layers 0..31, then backward over 31..0
    step = calls[:per_step]
    fwd_fp4 = step[:n_fp4 * nl * 2]
    assert all(c[0] in ("dual", "gemm") for c in fwd_fp4)
    fwd_bf16 = step[n_fp4 * nl * 2:n_fp4 * nl * 2 + bench.STACK_BF16_LAYERS * nl]
    assert all(c[0] == "matmul" for c in fwd_bf16)
    bwd_bf16 = step[len(fwd_fp4) + len(fwd_bf16):][:bench.STACK_BF16_LAYERS * nl * 2]
    assert all(c[0] == "matmul" for c in bwd_bf16)
    bwd_fp4 = step[len(fwd_fp4) + len(fwd_bf16) + len(bwd_bf16):]
    assert len(bwd_fp4) == n_fp4 * nl * 3 and all(c[0] in ("dual", "gemm") for c in bwd_fp4)

    # forward: X NVFP4-global RNE; backward: dY MXFP4 SR, seeds distinct per layer
    assert {(c[2], c[3]) for c in fwd_fp4 if c[0] == "dual"} == {(fa.NVFP4_GLOBAL, fa.RNE)}
    bwd_duals = [c for c in bwd_fp4 if c[0] == "dual"]
    assert {(c[2], c[3]) for c in bwd_duals} == {(fa.MXFP4, fa.SR)}
    assert len({c[4] for c in bwd_duals}) == n_fp4
    # wgrad GEMMs: alpha 1/32 and fp32 dW [Cout, Cin]; the others alpha 1, bf16
    gemms = [c for c in bwd_fp4 if c[0] == "gemm"]
    wgrad = [c for c in gemms if c[3] == 1.0 / 32]
    assert len(wgrad) == n_fp4 * nl
    assert all(c[5] == torch.float32 for c in wgrad)
    assert {c[4] for c in wgrad} == {(cout, cin) for cin, cout in layers.values()}
    assert all(c[5] == torch.bfloat16 for c in gemms + [c for c in fwd_fp4 if c[0] == "gemm"]
               if c[3] == 1.0)

    # times from the fake clock
    fp4_ms = n_fp4 * nl * (2 * COST["quantize_dual"] + 3 * COST["gemm"])
    bf16_ms = bench.STACK_BF16_LAYERS * nl * 3 * COST["matmul"]
    assert res["fp4_layers_ms"] == pytest.approx(fp4_ms)
    assert res["bf16_layers_ms"] == pytest.approx(bf16_ms)
    assert res["ms_per_step"] == pytest.approx(fp4_ms + bf16_ms)
    Ts = bench.STACK_TOKENS
    assert res["tokens_per_s"] == pytest.approx(Ts / ((fp4_ms + bf16_ms) * 1e-3), abs=0.05)
    flop_layer = 3 * 2.0 * Ts * sum(ci * co for ci, co in layers.values())
    assert res["fp4_layers_TFLOPS"] == pytest.approx(
        n_fp4 * flop_layer / (fp4_ms * 1e-3) / 1e12, abs=0.05)
    assert res["tokens"] == Ts and res["layers"] == bench.STACK_LAYERS
