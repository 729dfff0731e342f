"""The 32-layer 8B-shaped stack's FP4 linears: sequence 8192 x batch 2 =
16384 tokens through the QKV, O, gate+up and down shapes, forward (NVFP4-
global), dgrad (MXFP4, stochastic rounding) and wgrad (MXFP4, fixed-sign
Hadamard-32).  Each layer's FP4 work in the stack is one of these four
shapes at this token count, so the stack's parity is theirs.  Quantized bytes
are compared bit-exactly on sampled 128-row blocks; GEMM outputs on sampled
rows within the tolerance."""
import numpy as np
import pytest
import torch

import fp4_quantization_block_b200 as fa
import oracle as O
import workloads
from gpu_util import accumulation_bound, assert_gemm_close, assert_qt_equal, need_gpu, to_cpu_qt, to_gpu_qt

pytestmark = pytest.mark.gpu

SIGN_MASK = 0x2545F491
TOKENS = 2 * workloads.LLAMA8B_TOKENS


@pytest.mark.parametrize("layer", list(workloads.LLAMA8B_LINEARS), ids=str)
def test_stack_linear_16384_tokens_sampled(layer):
    need_gpu()
    cin, cout = workloads.LLAMA8B_LINEARS[layer]
    T = TOKENS
    rng = np.random.default_rng(100 + list(workloads.LLAMA8B_LINEARS).index(layer))
    x = workloads.act(T, cin, seed=21)
    dy = workloads.grad(T, cout, seed=22)
    w = workloads.weight(cout, cin, seed=23)
    xg, dyg = x.cuda(), dy.cuda()

    # forward: X row-wise NVFP4-global, bytes of one sampled row block
    r0 = 128 * int(rng.integers(T // 128))
    Xq = O.quantize(x, O.NVFP4_GLOBAL, row_range=(r0, r0 + 128))
    assert_qt_equal(to_cpu_qt(fa.quantize(xg, fa.NVFP4_GLOBAL)), Xq, (r0, r0 + 128))
    Wq = O.quantize(w, O.NVFP4_GLOBAL)
    y = fa.linear_fwd(xg, to_gpu_qt(Wq), fa.NVFP4_GLOBAL)
    rows = r0 + np.sort(rng.choice(128, 16, replace=False))
    assert_gemm_close(y.float().cpu().numpy()[rows], O.gemm_sampled(Xq, Wq, 1.0, rows, None),
                      O.gemm_tolerance(Xq, Wq), bf16=True,
                      tight=accumulation_bound(Xq, Wq, 1.0, rows, None))

    # dgrad: dY row-wise MXFP4 with stochastic rounding (seed 1)
    Wc = O.quantize(w, O.MXFP4, orient=O.COLWISE)
    g0 = 128 * int(rng.integers(T // 128))
    Gq = O.quantize(dy, O.MXFP4, O.SR, O.ROWWISE, seed=1, row_range=(g0, g0 + 128))
    assert_qt_equal(to_cpu_qt(fa.quantize(dyg, fa.MXFP4, fa.SR, fa.ROWWISE, seed=1)), Gq,
                    (g0, g0 + 128))
    dx = fa.linear_dgrad(dyg, to_gpu_qt(Wc), fa.MXFP4, fa.SR, seed=1)
    rows = g0 + np.sort(rng.choice(128, 16, replace=False))
    assert_gemm_close(dx.float().cpu().numpy()[rows], O.gemm_sampled(Gq, Wc, 1.0, rows, None),
                      O.gemm_tolerance(Gq, Wc), bf16=True,
                      tight=accumulation_bound(Gq, Wc, 1.0, rows, None))

    # wgrad: dY^T and X^T column-wise MXFP4 with the Hadamard, alpha 1/32, fp32 dW
    c0 = 128 * int(rng.integers(cout // 128))
    Gc = O.quantize(dy, O.MXFP4, O.RNE, O.COLWISE, hadamard_mask=SIGN_MASK,
                    row_range=(c0, c0 + 128))
    assert_qt_equal(to_cpu_qt(fa.hadamard32_quantize(dyg, SIGN_MASK)), Gc, (c0, c0 + 128))
    Xc = O.quantize(x, O.MXFP4, O.RNE, O.COLWISE, hadamard_mask=SIGN_MASK)
    dw = fa.linear_wgrad(dyg, xg, SIGN_MASK, fa.RNE, seed=3)
    wrows = c0 + np.sort(rng.choice(128, 16, replace=False))
    assert_gemm_close(dw.cpu().numpy()[wrows], O.gemm_sampled(Gc, Xc, 1.0 / 32, wrows, None),
                      O.gemm_tolerance(Gc, Xc, 1.0 / 32),
                      tight=accumulation_bound(Gc, Xc, 1.0 / 32, wrows, None))
