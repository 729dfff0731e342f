"""Fused quantizers on the GPU against the oracle, bit-exact: payload bytes,
scale bytes and FP32 second-level scales."""
import numpy as np
import pytest
import torch

import fp4_quantization_block_b200 as fa
import oracle as O
import workloads
from gpu_util import FMT_IDS, FMTS, assert_qt_equal, need_gpu, to_cpu_qt

pytestmark = pytest.mark.gpu

COMBOS = [(f, r, o) for f in FMTS for r in (fa.RNE, fa.SR) for o in (fa.ROWWISE, fa.COLWISE)]
CID = [f"{FMT_IDS[f]}-{'sr' if r else 'rne'}-{'col' if o else 'row'}" for f, r, o in COMBOS]


def _check(x_cpu, fmt, rnd, orient, seed=1, x_gpu=None, row_range=None, hadamard=None):
    need_gpu()
    xg = x_cpu.cuda() if x_gpu is None else x_gpu
    if hadamard is None:
        g = fa.quantize(xg, fmt, rnd, orient, seed)
    else:
        g = fa.hadamard32_quantize(xg, hadamard, rnd, seed)
    o = O.quantize(x_cpu, fmt, rnd, orient, seed, hadamard_mask=hadamard, row_range=row_range)
    assert_qt_equal(to_cpu_qt(g), o, row_range)


@pytest.mark.parametrize("fmt,rnd,orient", COMBOS, ids=CID)
def test_tiny(fmt, rnd, orient):
    _check(workloads.tiny(0), fmt, rnd, orient)


@pytest.mark.parametrize("fmt,rnd,orient", COMBOS, ids=CID)
def test_edge_values(fmt, rnd, orient):
    """Zero blocks, signed zeros, bf16 extremes and subnormals, grid points
    and midpoints after scaling."""
    _check(workloads.with_specials(workloads.tiny(3)), fmt, rnd, orient)


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
def test_all_zero_tensor(fmt):
    x = torch.zeros(256, 384, dtype=torch.bfloat16)
    for orient in (fa.ROWWISE, fa.COLWISE):
        _check(x, fmt, fa.RNE, orient)


@pytest.mark.parametrize("fmt,rnd,orient", COMBOS, ids=CID)
def test_multi_tile_strided(fmt, rnd, orient):
    """Several tiles in both directions, odd tile counts, and a leading
    dimension larger than the row (a column slice of a wider tensor)."""
    wide = workloads.sweep(384, 896, seed=11)
    x_cpu = wide[:, 64:704].contiguous()           # oracle sees the logical tensor
    x_gpu = wide.cuda()[:, 64:704]                 # GPU reads it in place, ld = 896
    assert x_gpu.stride(0) == 896
    _check(x_cpu, fmt, rnd, orient, seed=12345, x_gpu=x_gpu)


@pytest.mark.parametrize("rnd", [fa.RNE, fa.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("mask", [0x0, 0xFFFFFFFF, 0x2545F491])
def test_hadamard_colwise(rnd, mask):
    _check(workloads.grad(512, 384, seed=4), fa.MXFP4, rnd, fa.COLWISE, seed=77, hadamard=mask)
    _check(workloads.with_specials(workloads.tiny(5)), fa.MXFP4, rnd, fa.COLWISE, seed=78,
           hadamard=mask)


@pytest.mark.parametrize("fmt,rnd,orient", COMBOS, ids=CID)
def test_sweep_recipe_medium(fmt, rnd, orient):
    _check(workloads.sweep(1024, 1536, seed=2), fmt, rnd, orient, seed=3)


@pytest.fixture(scope="module")
def sweep_full():
    need_gpu()
    return {shape: workloads.sweep(*shape, seed=0) for shape in workloads.SWEEP_SHAPES}


@pytest.mark.parametrize("shape", workloads.SWEEP_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
@pytest.mark.parametrize("fmt,rnd,orient", COMBOS, ids=CID)
def test_sweep_full_size_sampled(sweep_full, shape, fmt, rnd, orient):
    """Full quantizer-sweep sizes: the GPU quantizes the whole tensor in the
    benchmark's launch configuration; the oracle recomputes three sampled
    128-row blocks of the quantized operand (the first, one in the middle and
    the last), with second-level scales over the whole tensor."""
    x = sweep_full[shape]
    xg = x.cuda()
    g = to_cpu_qt(fa.quantize(xg, fmt, rnd, orient, 1))
    R = g.R
    for r0 in (0, (R // 256) * 128, R - 128):
        o = O.quantize(x, fmt, rnd, orient, 1, row_range=(r0, r0 + 128))
        assert_qt_equal(g, o, (r0, r0 + 128))


def test_repeat_calls_are_deterministic():
    need_gpu()
    x = workloads.sweep(512, 512, seed=9).cuda()
    for fmt in FMTS:
        a = to_cpu_qt(fa.quantize(x, fmt, fa.SR, fa.ROWWISE, 5))
        b = to_cpu_qt(fa.quantize(x, fmt, fa.SR, fa.ROWWISE, 5))
        assert np.array_equal(a.payload, b.payload) and np.array_equal(a.scales, b.scales)
        c = to_cpu_qt(fa.quantize(x, fmt, fa.SR, fa.ROWWISE, 6))
        assert not np.array_equal(a.payload, c.payload)
