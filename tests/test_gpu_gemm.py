"""Block-scaled FP4 GEMM on the tcgen05 tensor cores against the oracle's
binary64 dequantize-then-accumulate GEMM.  Operands are quantized by the
oracle and uploaded, so these tests isolate the GEMM.

Tolerance: max |D_gpu - D_oracle| <= 1e-3 * max|A_hat| * max|B_hat| * sqrt(K)
(dequantized operands with second-level scales and alpha), plus half a bf16
ulp of the exact value for bf16 output."""
import numpy as np
import pytest
import torch

import fp4_quantization_block_b200 as fa
import oracle as O
import workloads
from gpu_util import FMT_IDS, FMTS, accumulation_bound, assert_gemm_close, need_gpu, to_gpu_qt

pytestmark = pytest.mark.gpu


def _run(xa, xb, fmt, alpha=1.0, out=torch.float32, rows=None, cols=None):
    need_gpu()
    A = O.quantize(xa, fmt)
    B = O.quantize(xb, fmt)
    d = fa.gemm(to_gpu_qt(A), to_gpu_qt(B), alpha, out_dtype=out)
    torch.cuda.synchronize()
    dg = d.float().cpu().numpy().astype(np.float64)
    if rows is not None or cols is not None:
        want = O.gemm_sampled(A, B, alpha, rows, cols)
        r = np.arange(A.R) if rows is None else np.asarray(rows)
        c = np.arange(B.R) if cols is None else np.asarray(cols)
        dg = dg[np.ix_(r, c)]
    else:
        want = O.gemm_sampled(A, B, alpha) if A.R * B.R * A.K > (1 << 24) else O.gemm(A, B, alpha)
    tol = O.gemm_tolerance(A, B, alpha)
    tight = accumulation_bound(A, B, alpha, rows, cols)
    return assert_gemm_close(dg, want, tol, bf16=(out == torch.bfloat16), tight=tight), tol


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
def test_tiny_config(fmt, out):
    """A = X[0:128, 0:256], B = X[128:256, 256:512] of the tiny workload."""
    x = workloads.tiny(0)
    _run(x[0:128, 0:256].contiguous(), x[128:256, 256:512].contiguous(), fmt, out=out)


def test_single_nonzero_element_locates_nibbles_and_scales():
    """One nonzero element per operand: checks element order inside a byte,
    row/column placement and the scale byte the MMA applies."""
    need_gpu()
    for fmt in FMTS:
        for (m, k, n) in [(0, 0, 0), (5, 1, 7), (127, 255, 100), (64, 130, 33)]:
            xa = torch.zeros(128, 256, dtype=torch.bfloat16)
            xb = torch.zeros(128, 256, dtype=torch.bfloat16)
            xa[m, k] = 3.0
            xb[n, k] = -0.5
            _run(xa, xb, fmt)


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
@pytest.mark.parametrize("mnk", [(384, 640, 768), (256, 512, 512), (640, 256, 1280)],
                         ids=lambda t: "x".join(map(str, t)))
def test_multi_tile(fmt, mnk):
    M, N, K = mnk
    xa = workloads.sweep(M, K, seed=31)
    xb = workloads.weight(N, K, seed=32)
    _run(xa, xb, fmt, alpha=0.5)


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
def test_scale_spread(fmt):
    """Rows and K ranges with very different magnitudes (different block and
    tile scales), including all-zero blocks."""
    xa = workloads.act(512, 1024, seed=41)
    xa[:, :256] *= 1e-4
    xa[128:256] *= 300.0
    xa[:, 512:544] = 0
    xb = workloads.grad(256, 1024, seed=42)
    _run(xa, xb, fmt)


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
def test_persistent_many_tiles(fmt):
    """More output tiles than SMs, so every CTA loops over tiles and the
    accumulator and pipeline phases wrap."""
    xa = workloads.act(2048, 1024, seed=51)
    xb = workloads.weight(3072, 1024, seed=52)
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(2048, 96, replace=False))
    _run(xa, xb, fmt, rows=rows)


@pytest.mark.parametrize("fmt", [fa.NVFP4_GLOBAL, fa.NVFP4_CTA, fa.MXFP4], ids=["nvg", "nvc", "mx"])
@pytest.mark.parametrize("layer", list(workloads.LLAMA8B_LINEARS), ids=str)
def test_llama8b_forward_shapes_sampled(layer, fmt):
    """The 8B-shaped forward GEMMs at full size (M = 8192 tokens) in each scale
    domain: sampled 64 rows and 64 columns of D against the oracle."""
    need_gpu()
    cin, cout = workloads.LLAMA8B_LINEARS[layer]
    x = workloads.act(workloads.LLAMA8B_TOKENS, cin, seed=1)
    w = workloads.weight(cout, cin, seed=2)
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(x.shape[0], 64, replace=False))
    cols = np.sort(rng.choice(cout, 64, replace=False))
    A = O.quantize(x, fmt)
    B = O.quantize(w, fmt)
    d = fa.gemm(to_gpu_qt(A), to_gpu_qt(B), 1.0, out_dtype=torch.float32)
    torch.cuda.synchronize()
    dg = d.cpu().numpy().astype(np.float64)
    tol = O.gemm_tolerance(A, B)
    assert_gemm_close(dg[rows, :], O.gemm_sampled(A, B, 1.0, rows, None), tol,
                      tight=accumulation_bound(A, B, 1.0, rows, None))
    assert_gemm_close(dg[:, cols], O.gemm_sampled(A, B, 1.0, None, cols), tol,
                      tight=accumulation_bound(A, B, 1.0, None, cols))
