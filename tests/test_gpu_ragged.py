"""Ragged shapes on the GPU: operands whose row count is not a multiple of
128 and whose block dimension K is a multiple of 32 but not of 128, and
GEMMs with any M and N.  Quantized bytes (payload, every scale byte of the
padded atoms, FP32 second-level scales) must equal the oracle's; GEMM
outputs must be within the GEMM tolerance.

The shapes are chosen to reach every launch path: only R ragged (unmasked
interior tiles plus an EDGE row of tiles), only K ragged (every tile EDGE),
both, a single partial tile, a 2-SM pair whose second CTA's rows are
partly outside A, 256-wide B tiles cut by N, and a last k-tile holding one
scale atom (or, CTA-local, one whole 128-wide K chunk past K)."""
import numpy as np
import pytest
import torch

import fp4_quantization_block_b200 as fa
import oracle as O
import workloads
from gpu_util import (FMT_IDS, FMTS, accumulation_bound, assert_gemm_close, assert_qt_equal, need_gpu, to_cpu_qt,
                      to_gpu_qt)

pytestmark = pytest.mark.gpu

MASK = 0x2545F491

# x[rows, cols] -> row-wise Q[rows, cols]: rows any, cols a multiple of 32
ROW_SHAPES = [(200, 352), (300, 640), (384, 416), (1, 32), (129, 160), (96, 96)]
# x[rows, cols] -> column-wise Q[cols, rows]: rows a multiple of 32, cols a multiple of 8
COL_SHAPES = [(352, 200), (640, 300 - 300 % 8), (416, 384), (32, 8), (160, 136)]


def _x(rows, cols, seed):
    return workloads.sweep(max(rows, 2), cols, seed=seed)[:rows].contiguous()


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
@pytest.mark.parametrize("rnd", [fa.RNE, fa.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("shape", ROW_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
def test_rowwise(fmt, rnd, shape):
    need_gpu()
    x = _x(*shape, seed=shape[0] + 3 * shape[1])
    g = fa.quantize(x.cuda(), fmt, rnd, fa.ROWWISE, seed=11)
    assert_qt_equal(to_cpu_qt(g), O.quantize(x, fmt, rnd, O.ROWWISE, seed=11))


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
@pytest.mark.parametrize("rnd", [fa.RNE, fa.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("shape", COL_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
def test_colwise(fmt, rnd, shape):
    need_gpu()
    x = _x(*shape, seed=7 * shape[0] + shape[1])
    g = fa.quantize(x.cuda(), fmt, rnd, fa.COLWISE, seed=13)
    assert_qt_equal(to_cpu_qt(g), O.quantize(x, fmt, rnd, O.COLWISE, seed=13))


@pytest.mark.parametrize("shape", COL_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
def test_hadamard(shape):
    need_gpu()
    x = _x(*shape, seed=5 + shape[1])
    g = fa.hadamard32_quantize(x.cuda(), MASK, fa.SR, 17)
    assert_qt_equal(to_cpu_qt(g), O.quantize(x, O.MXFP4, O.SR, O.COLWISE, 17, hadamard_mask=MASK))


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
@pytest.mark.parametrize("shape", [(352, 224), (96, 160), (256, 96), (32, 32)],
                         ids=lambda s: f"{s[0]}x{s[1]}")
def test_dual(fmt, shape):
    need_gpu()
    x = _x(*shape, seed=19 + shape[0])
    gr, gc = fa.quantize_dual(x.cuda(), fmt, fa.SR, 3, col_hadamard=True, sign_mask=MASK,
                              col_rnd=fa.RNE, col_seed=0)
    assert_qt_equal(to_cpu_qt(gr), O.quantize(x, fmt, O.SR, O.ROWWISE, 3))
    assert_qt_equal(to_cpu_qt(gc), O.quantize(x, O.MXFP4, O.RNE, O.COLWISE, hadamard_mask=MASK))


def test_unmasked_and_edge_tiles_agree_with_the_aligned_call():
    """Rows 0..255 of a 300-row operand come from the unmasked kernel: they
    equal the quantization of those 256 rows alone, byte for byte."""
    need_gpu()
    x = workloads.sweep(300, 512, seed=23).cuda()
    for fmt in (fa.MXFP4, fa.NVFP4_CTA):
        a = fa.quantize(x, fmt, fa.SR, fa.ROWWISE, seed=5)
        b = fa.quantize(x[:256].contiguous(), fmt, fa.SR, fa.ROWWISE, seed=5)
        assert torch.equal(a.payload[:256], b.payload)
        assert torch.equal(a.scales[:b.scales.numel()], b.scales)


# M, N, K: pair path with M cut inside the second CTA's rows (400 -> 512),
# 256-wide tiles cut by N, 128-wide tiles, K with a last k-tile of 96
# (one 32-block atom for MX, a CTA-local chunk wholly past K) or 160
GEMM_SHAPES = [(200, 72, 352), (400, 400, 352), (72, 200, 160), (130, 136, 544), (1, 8, 32),
               (384, 257 - 257 % 8, 256)]


@pytest.mark.parametrize("fmt", [fa.MXFP4, fa.NVFP4_GLOBAL, fa.NVFP4_CTA],
                         ids=["mx", "nvg", "nvc"])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
@pytest.mark.parametrize("mnk", GEMM_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_gemm(fmt, out, mnk):
    need_gpu()
    M, N, K = mnk
    rng = np.random.default_rng(M + N + K)
    xa = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    xb = torch.from_numpy((rng.standard_normal((N, K)) * 0.05).astype(np.float32)).to(torch.bfloat16)
    xb[:, K // 2:] *= 30.0  # K chunks with different CTA-local scales
    A, B = O.quantize(xa, fmt), O.quantize(xb, fmt)
    d = fa.gemm(to_gpu_qt(A), to_gpu_qt(B), 0.5, out_dtype=out)
    torch.cuda.synchronize()
    assert d.shape == (M, N)
    assert_gemm_close(d.float().cpu().numpy(), O.gemm(A, B, 0.5), O.gemm_tolerance(A, B, 0.5),
                      bf16=(out == torch.bfloat16), tight=accumulation_bound(A, B, 0.5))


def test_gemm_writes_nothing_outside_d():
    """D is a view into a larger buffer filled with a sentinel: the GEMM of a
    ragged shape leaves every element outside [M, N] untouched."""
    need_gpu()
    M, N, K = 200, 72, 352
    rng = np.random.default_rng(2)
    xa = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    xb = torch.from_numpy(rng.standard_normal((N, K)).astype(np.float32)).to(torch.bfloat16)
    A, B = fa.quantize(xa.cuda(), fa.MXFP4), fa.quantize(xb.cuda(), fa.MXFP4)
    big = torch.full((M + 64, 128), 7.0, dtype=torch.float32, device="cuda")
    fa.gemm(A, B, 1.0, out=big[:M, :N])
    torch.cuda.synchronize()
    assert torch.all(big[M:] == 7.0) and torch.all(big[:M, N:] == 7.0)


@pytest.mark.parametrize("fmt", [fa.MXFP4, fa.NVFP4_GLOBAL], ids=["mx", "nvg"])
@pytest.mark.parametrize("mnk", [(200, 96, 352), (400, 416, 160)], ids=lambda s: "x".join(map(str, s)))
def test_gemm_mxout(fmt, mnk):
    """The epilogue's MXFP4 operand of a ragged D equals the row-wise
    quantization of that bf16 D (padding scale bytes zero)."""
    need_gpu()
    M, N, K = mnk
    rng = np.random.default_rng(K)
    xa = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16).cuda()
    xb = torch.from_numpy(rng.standard_normal((N, K)).astype(np.float32)).to(torch.bfloat16).cuda()
    A, B = fa.quantize(xa, fmt), fa.quantize(xb, fmt)
    d, dq = fa.gemm_mxout(A, B, 0.25)
    torch.cuda.synchronize()
    assert torch.equal(d, fa.gemm(A, B, 0.25, out_dtype=torch.bfloat16))
    assert_qt_equal(to_cpu_qt(dq), O.quantize(d.cpu(), O.MXFP4))


def test_training_linear_ragged_tokens():
    """T = 224 tokens (a multiple of 32, not of 128) through the training-form
    linear calls: equal to the separate calls, and the quantized operands
    equal to the oracle's."""
    need_gpu()
    T, Cin, Cout = 224, 160, 96
    x = workloads.act(T, Cin, seed=71, device="cuda")
    dy = workloads.grad(T, Cout, seed=72, device="cuda")
    w = workloads.weight(Cout, Cin, seed=73, device="cuda")
    for fmt in (fa.MXFP4, fa.NVFP4_GLOBAL):
        wq = fa.quantize(w, fmt)
        wc = fa.quantize(w, fmt, orient=fa.COLWISE)
        y, xcol = fa.linear_fwd_save(x, wq, fmt, MASK)
        assert torch.equal(y, fa.linear_fwd(x, wq, fmt))
        assert_qt_equal(to_cpu_qt(xcol),
                        O.quantize(x.cpu(), O.MXFP4, O.RNE, O.COLWISE, hadamard_mask=MASK))
        dx, dw = fa.linear_bwd(dy, wc, xcol, fmt, fa.SR, 3, MASK)
        assert torch.equal(dx, fa.linear_dgrad(dy, wc, fmt, fa.SR, 3))
        assert torch.equal(dw, fa.linear_wgrad(dy, x, MASK, fa.RNE, 0))
