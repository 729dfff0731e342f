"""Dual-orientation producer on the GPU: one read of x gives the row-wise
operand (any format) and the column-wise MXFP4 operand (with or without the
fixed-sign Hadamard).  Both must equal the oracle's single-orientation
quantizations byte for byte."""
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
COMBOS = [(f, rr, cr, h) for f in FMTS for rr in (fa.RNE, fa.SR) for cr in (fa.RNE, fa.SR)
          for h in (False, True)]
CID = [f"{FMT_IDS[f]}-{'sr' if rr else 'rne'}-col{'sr' if cr else 'rne'}{'-had' if h else ''}"
       for f, rr, cr, h in COMBOS]


def _check(x_cpu, fmt, rr, cr, had, x_gpu=None, rows=None, cols=None, seeds=(7, 9)):
    need_gpu()
    xg = x_cpu.cuda() if x_gpu is None else x_gpu
    gr, gc = fa.quantize_dual(xg, fmt, rr, seeds[0], col_hadamard=had, sign_mask=MASK,
                              col_rnd=cr, col_seed=seeds[1])
    orow = O.quantize(x_cpu, fmt, rr, O.ROWWISE, seeds[0], row_range=rows)
    ocol = O.quantize(x_cpu, O.MXFP4, cr, O.COLWISE, seeds[1],
                      hadamard_mask=MASK if had else None, row_range=cols)
    assert_qt_equal(to_cpu_qt(gr), orow, rows)
    assert_qt_equal(to_cpu_qt(gc), ocol, cols)


@pytest.mark.parametrize("fmt,rr,cr,had", COMBOS, ids=CID)
def test_tiny(fmt, rr, cr, had):
    _check(workloads.tiny(2), fmt, rr, cr, had)


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
def test_edge_values(fmt):
    _check(workloads.with_specials(workloads.tiny(5)), fmt, fa.SR, fa.RNE, True)


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
def test_multi_tile_strided(fmt):
    """Odd tile counts both ways and a leading dimension wider than the row."""
    wide = workloads.sweep(384, 896, seed=21)
    x_cpu = wide[:, 128:768].contiguous()
    x_gpu = wide.cuda()[:, 128:768]
    _check(x_cpu, fmt, fa.SR, fa.RNE, True, x_gpu=x_gpu)
    _check(x_cpu, fmt, fa.RNE, fa.SR, False, x_gpu=x_gpu)


def test_equals_single_orientation_kernels():
    """GPU against GPU: the dual producer and the two single-orientation
    calls agree byte for byte on a medium tensor."""
    need_gpu()
    x = workloads.grad(1024, 2048, seed=4, device="cuda")
    gr, gc = fa.quantize_dual(x, fa.MXFP4, fa.SR, 5, col_hadamard=True, sign_mask=MASK)
    sr = fa.quantize(x, fa.MXFP4, fa.SR, fa.ROWWISE, 5)
    sc = fa.hadamard32_quantize(x, MASK)
    for a, b in ((gr, sr), (gc, sc)):
        assert torch.equal(a.payload, b.payload)
        assert torch.equal(a.scales, b.scales)


@pytest.mark.parametrize("layer", ["gate_up", "down"], ids=str)
def test_llama8b_full_size_sampled(layer):
    """Full 8B shapes at 8192 tokens: dY (MXFP4 SR row-wise + Hadamard
    column-wise) and X (NVFP4-global row-wise + Hadamard column-wise), bytes of
    sampled 128-row blocks of each operand."""
    need_gpu()
    cin, cout = workloads.LLAMA8B_LINEARS[layer]
    T = workloads.LLAMA8B_TOKENS
    rng = np.random.default_rng(31)
    dy = workloads.grad(T, cout, seed=41)
    r0 = 128 * int(rng.integers(T // 128))
    c0 = 128 * int(rng.integers(cout // 128))
    _check(dy, fa.MXFP4, fa.SR, fa.RNE, True, rows=(r0, r0 + 128), cols=(c0, c0 + 128))
    x = workloads.act(T, cin, seed=42)
    r0 = 128 * int(rng.integers(T // 128))
    c0 = 128 * int(rng.integers(cin // 128))
    _check(x, fa.NVFP4_GLOBAL, fa.RNE, fa.RNE, True, rows=(r0, r0 + 128), cols=(c0, c0 + 128))


def test_sr_counters_of_a_2_32_element_tensor():
    """A tensor of 2^32 elements takes the quantizers' 64-bit Philox counter
    path (smaller ones take the 32-bit one): MXFP4 stochastic rounding
    row-wise and column-wise from one read, bytes of the last 128-row block
    of each operand (the largest counters) against the oracle."""
    need_gpu()
    T, C = 32768, 131072
    gen = torch.Generator(device="cuda").manual_seed(61)
    xg = torch.randn(T, C, device="cuda", dtype=torch.bfloat16, generator=gen)
    try:
        _check(xg.cpu(), fa.MXFP4, fa.SR, fa.SR, False, x_gpu=xg, rows=(T - 128, T),
               cols=(C - 128, C), seeds=(71, 73))
    finally:
        del xg
        torch.cuda.empty_cache()


@pytest.mark.parametrize("fmt", [fa.MXFP4, fa.NVFP4_GLOBAL], ids=["mx", "nvg"])
def test_training_linear_equals_the_separate_calls(fmt):
    """linear_fwd_save + linear_bwd (dual producers) give exactly the bytes of
    linear_fwd, hadamard32_quantize, linear_dgrad and linear_wgrad."""
    need_gpu()
    T, Cin, Cout = 512, 512, 768  # GEMM K (Cin, Cout, T) multiples of 256
    x = workloads.act(T, Cin, seed=51, device="cuda")
    dy = workloads.grad(T, Cout, seed=52, device="cuda")
    w = workloads.weight(Cout, Cin, seed=53, device="cuda")
    wq = fa.quantize(w, fmt)
    wc = fa.quantize(w, fmt, orient=fa.COLWISE)
    y, xcol = fa.linear_fwd_save(x, wq, fmt, MASK)
    assert torch.equal(y, fa.linear_fwd(x, wq, fmt))
    xc_ref = fa.hadamard32_quantize(x, MASK)
    assert torch.equal(xcol.payload, xc_ref.payload) and torch.equal(xcol.scales, xc_ref.scales)
    dx, dw = fa.linear_bwd(dy, wc, xcol, fmt, fa.SR, 3, MASK)
    assert torch.equal(dx, fa.linear_dgrad(dy, wc, fmt, fa.SR, 3))
    assert torch.equal(dw, fa.linear_wgrad(dy, x, MASK, fa.RNE, 0))


def test_training_linear_against_the_oracle():
    """The training-form outputs against oracle compositions (quantize, then
    the binary64 GEMM) within the GEMM tolerance."""
    need_gpu()
    T, Cin, Cout = 256, 256, 512
    x = workloads.act(T, Cin, seed=61)
    dy = workloads.grad(T, Cout, seed=62)
    w = workloads.weight(Cout, Cin, seed=63)
    Wq = O.quantize(w, O.NVFP4_GLOBAL)
    Wc = O.quantize(w, O.NVFP4_GLOBAL, orient=O.COLWISE)
    y, xcol = fa.linear_fwd_save(x.cuda(), to_gpu_qt(Wq), fa.NVFP4_GLOBAL, MASK)
    dx, dw = fa.linear_bwd(dy.cuda(), to_gpu_qt(Wc), xcol, fa.NVFP4_GLOBAL, fa.SR, 5, MASK)
    Xq = O.quantize(x, O.NVFP4_GLOBAL)
    assert_gemm_close(y.float().cpu().numpy(), O.gemm(Xq, Wq), O.gemm_tolerance(Xq, Wq), bf16=True,
                      tight=accumulation_bound(Xq, Wq))
    Gq = O.quantize(dy, O.NVFP4_GLOBAL, O.SR, O.ROWWISE, 5)
    assert_gemm_close(dx.float().cpu().numpy(), O.gemm(Gq, Wc), O.gemm_tolerance(Gq, Wc), bf16=True,
                      tight=accumulation_bound(Gq, Wc))
    Gc = O.quantize(dy, O.MXFP4, O.RNE, O.COLWISE, hadamard_mask=MASK)
    Xc = O.quantize(x, O.MXFP4, O.RNE, O.COLWISE, hadamard_mask=MASK)
    assert_qt_equal(to_cpu_qt(xcol), Xc)
    assert_gemm_close(dw.cpu().numpy(), O.gemm(Gc, Xc, 1.0 / 32), O.gemm_tolerance(Gc, Xc, 1.0 / 32),
                      tight=accumulation_bound(Gc, Xc, 1.0 / 32))
