"""The SwiGLU producer fused with its quantizer (fa4_swiglu_quantize) against
the oracle: h = bf16(silu(gate) * up) from the oracle's step-by-step binary32
definition, then the oracle's quantization of h.  Payload and scale bytes
(and CTA-local second-level scales) must be identical, row-wise and
column-wise, on tiles cut by the tensor's edge, on values that reach the
exp clamp, and at the 8B down projection's input size."""
import numpy as np
import pytest
import torch

import fp4_quantization_block_b200 as fa
import oracle as O
from gpu_util import FMT_IDS, assert_qt_equal, need_gpu, to_cpu_qt

pytestmark = pytest.mark.gpu

MASK = 0x2545F491
ROW_FMTS = [fa.MXFP4, fa.MXFP4_NOCLIP, fa.NVFP4_CTA]
COLS = {"nocol": None, "had-rne": (fa.RNE, True), "had-sr": (fa.SR, True), "plain-rne": (fa.RNE, False)}


def _z(T, F, seed, scale=2.0):
    g = torch.Generator().manual_seed(seed)
    gate = torch.randn(T, F, generator=g) * scale
    up = torch.randn(T, F, generator=g)
    up[:, ::37] *= 20.0  # outlier channels
    return torch.cat([gate, up], 1).to(torch.bfloat16)


def _check(z, fmt, rnd, col, row_range=None, col_range=None):
    h = O.swiglu_bf16(z)
    col_rnd, had = col if col else (fa.RNE, True)
    rq, cq = fa.swiglu_quantize(z.cuda(), fmt, rnd, 5, col=col is not None, col_hadamard=had,
                                sign_mask=MASK, col_rnd=col_rnd, col_seed=7)
    torch.cuda.synchronize()
    assert_qt_equal(to_cpu_qt(rq), O.quantize(h, fmt, rnd, O.ROWWISE, seed=5, row_range=row_range),
                    row_range)
    if col:
        want = O.quantize(h, O.MXFP4, col_rnd, O.COLWISE, seed=7,
                          hadamard_mask=MASK if had else None, row_range=col_range)
        assert_qt_equal(to_cpu_qt(cq), want, col_range)


@pytest.mark.parametrize("fmt", ROW_FMTS, ids=[FMT_IDS[f] for f in ROW_FMTS])
@pytest.mark.parametrize("rnd", [fa.RNE, fa.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("col", list(COLS.values()), ids=list(COLS))
def test_swiglu_quantize_matches_oracle(fmt, rnd, col):
    need_gpu()
    _check(_z(256, 384, seed=3), fmt, rnd, col)


@pytest.mark.parametrize("T,F,col", [(200, 160, False), (224, 96, True), (33 * 32, 32, True)],
                         ids=["200x160", "224x96-col", "1056x32-col"])
def test_swiglu_ragged(T, F, col):
    need_gpu()
    _check(_z(T, F, seed=T + F), fa.NVFP4_CTA, fa.RNE, (fa.RNE, True) if col else None)


def test_swiglu_clamp_and_special_values():
    """Gate values past the exp clamp (|g| > 87), zeros of both signs, bf16
    subnormals and large up values."""
    need_gpu()
    T, F = 128, 128
    gen = torch.Generator().manual_seed(11)
    gate = torch.randn(T, F, generator=gen) * 40.0
    gate[0, :8] = torch.tensor([0.0, -0.0, 100.0, -100.0, 87.25, -87.25, 1e-39, -1e-39])
    up = torch.randn(T, F, generator=gen)
    up[1, :] = 0.0
    up[2, :] = 3.0e30
    z = torch.cat([gate, up], 1).to(torch.bfloat16)
    for fmt in ROW_FMTS:
        _check(z, fmt, fa.RNE, (fa.SR, True))


def test_swiglu_8b_down_input_sampled():
    """The down projection's input at 8192 tokens x 14336 channels (z is the
    8192 x 28672 gate+up output): bytes of a sampled 128-row block of the
    row-wise operand and a sampled 128-channel block of the column-wise one."""
    need_gpu()
    T, F = 8192, 14336
    z = _z(T, F, seed=21, scale=1.5)
    rng = np.random.default_rng(3)
    r0 = 128 * int(rng.integers(T // 128))
    c0 = 128 * int(rng.integers(F // 128))
    _check(z, fa.NVFP4_CTA, fa.RNE, (fa.RNE, True), row_range=(r0, r0 + 128),
           col_range=(c0, c0 + 128))


def test_silu_every_finite_bf16_gate():
    """silu in binary32 as the producer computes it (packed exp steps, the
    quotient through a reciprocal estimate and Markstein's correction)
    against the oracle's IEEE steps, for every finite bf16 gate value."""
    need_gpu()
    bits = np.arange(1 << 16, dtype=np.uint32)
    finite = ((bits >> 7) & 0xFF) != 0xFF
    g16 = bits[finite].astype(np.uint16)
    g = torch.from_numpy(g16.view(np.int16).copy()).view(torch.bfloat16)
    got = fa.debug_silu(g.cuda()).cpu().numpy()
    want = np.array([O.silu_f32(v) for v in g.float().numpy()], dtype=np.float32)
    bad = np.nonzero(got.view(np.uint32) != want.view(np.uint32))[0]
    assert bad.size == 0, (int(bad.size), float(g.float()[bad[0]]), float(got[bad[0]]), float(want[bad[0]]))
