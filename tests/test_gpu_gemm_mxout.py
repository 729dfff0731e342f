"""GEMM with the MXFP4 quantizer fused into its epilogue: the quantized
operand of the bf16 output must equal the quantization of that output, byte
for byte (against the separate GPU quantizer and the oracle)."""
import numpy as np
import pytest
import torch

import fp4_quantization_block_b200 as fa
import oracle as O
import workloads
from gpu_util import assert_qt_equal, need_gpu, to_cpu_qt, to_gpu_qt

pytestmark = pytest.mark.gpu

SHAPES = [(256, 256, 512), (384, 640, 256), (384, 512, 256), (256, 512, 768), (512, 384, 1024)]


@pytest.mark.parametrize("fmt", [fa.MXFP4, fa.NVFP4_GLOBAL], ids=["mx", "nvg"])
@pytest.mark.parametrize("M,N,K", SHAPES, ids=[f"{m}x{n}x{k}" for m, n, k in SHAPES])
def test_epilogue_operand_equals_quantized_output(fmt, M, N, K):
    """Pair (M, N multiples of 256), 1-SM 256-wide and 128-wide tiles."""
    need_gpu()
    a = workloads.act(M, K, seed=71)
    b = workloads.weight(N, K, seed=72)
    A, B = to_gpu_qt(O.quantize(a, fmt)), to_gpu_qt(O.quantize(b, fmt))
    d, dq = fa.gemm_mxout(A, B, 0.75)
    torch.cuda.synchronize()
    assert torch.equal(d, fa.gemm(A, B, 0.75, out_dtype=torch.bfloat16))
    sep = fa.quantize(d, fa.MXFP4, fa.RNE, fa.ROWWISE)
    assert torch.equal(dq.payload, sep.payload) and torch.equal(dq.scales, sep.scales)
    assert_qt_equal(to_cpu_qt(dq), O.quantize(d.cpu(), O.MXFP4, O.RNE, O.ROWWISE))


def test_quantized_output_only():
    """With D not stored, the quantized operand is the same."""
    need_gpu()
    a = workloads.act(512, 1024, seed=73, device="cuda")
    b = workloads.weight(768, 1024, seed=74, device="cuda")
    A, B = fa.quantize(a, fa.MXFP4), fa.quantize(b, fa.MXFP4)
    d, _ = fa.gemm_mxout(A, B)
    none, dq = fa.gemm_mxout(A, B, store_d=False)
    assert none is None
    sep = fa.quantize(d, fa.MXFP4)
    assert torch.equal(dq.payload, sep.payload) and torch.equal(dq.scales, sep.scales)


def test_llama8b_forward_gate_up_sampled():
    """Full 8B forward gate+up shape: sampled 128-row blocks of the fused
    operand against the oracle's quantization of the GPU's bf16 output."""
    need_gpu()
    T = workloads.LLAMA8B_TOKENS
    cin, cout = workloads.LLAMA8B_LINEARS["gate_up"]
    x = workloads.act(T, cin, seed=75, device="cuda")
    w = workloads.weight(cout, cin, seed=76, device="cuda")
    A, B = fa.quantize(x, fa.NVFP4_GLOBAL), fa.quantize(w, fa.NVFP4_GLOBAL)
    d, dq = fa.gemm_mxout(A, B)
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    gq = to_cpu_qt(dq)
    for _ in range(2):
        r0 = 128 * int(rng.integers(T // 128))
        rows = d[r0:r0 + 128].cpu()
        o = O.quantize(rows, O.MXFP4, O.RNE, O.ROWWISE)
        assert np.array_equal(gq.payload[r0:r0 + 128], o.payload)
        kb4 = cout // 32 // 4
        sl = slice((r0 // 128) * kb4 * 512, (r0 // 128 + 1) * kb4 * 512)
        assert np.array_equal(gq.scales[sl], o.scales)
