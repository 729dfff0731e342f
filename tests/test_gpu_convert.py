"""Device element conversions (E2M1 RNE/SR, E4M3, Philox bits) against the
oracle on dense sweeps that cover every rounding boundary."""
import numpy as np
import pytest
import torch

import fp4_quantization_block_b200 as fa
import oracle as O
from gpu_util import need_gpu
from oracle_pins import _e2m1_sweep

pytestmark = pytest.mark.gpu


def _boundary_sweep():
    grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    pts = grid + [(a + b) / 2 for a, b in zip(grid, grid[1:])]
    out = []
    for p in pts:
        base = np.float32(p).view(np.int32)
        out.append((base + np.arange(-4096, 4097, dtype=np.int32)).view(np.float32))
    out = np.concatenate(out)
    out = out[np.isfinite(out) & (out >= 0)]
    # a strided walk over every binade from 2^-149 to 2^8
    walk = np.arange(1, 0x43800000, 97, dtype=np.int64).astype(np.int32).view(np.float32)
    allv = np.concatenate([out, walk, _e2m1_sweep(), np.array([0.0, 1e30, 3e38], np.float32)])
    return np.concatenate([allv, -allv]).astype(np.float32)


def test_e2m1_rne_matches_oracle():
    need_gpu()
    ys = _boundary_sweep()
    rne, _, _ = fa.debug_convert(torch.from_numpy(ys).cuda())
    got = rne.cpu().numpy()
    want = O.e2m1_rne(ys)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. y={ys[bad[:4]]} gpu={got[bad[:4]]} oracle={want[bad[:4]]}"


def test_e2m1_sr_matches_oracle():
    need_gpu()
    rng = np.random.default_rng(17)
    ys = np.concatenate([_boundary_sweep()[::3], rng.uniform(-7, 7, 1 << 20).astype(np.float32)])
    u = rng.integers(0, 1 << 16, ys.size, dtype=np.uint32)
    # the u values at both sides of the threshold of some inputs
    u[:4096] = 0
    u[4096:8192] = 65535
    _, sr, _ = fa.debug_convert(torch.from_numpy(ys).cuda(), torch.from_numpy(u.view(np.int32)).cuda())
    got = sr.cpu().numpy()
    want = O.e2m1_sr(ys, u)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. y={ys[bad[:4]]} u={u[bad[:4]]}"


def test_e4m3_block_scale_matches_oracle():
    need_gpu()
    rng = np.random.default_rng(19)
    codes = np.arange(1, 127)
    vals = np.array([O.e4m3_decode(int(c)) for c in codes], np.float32)
    mids = ((vals[:-1].astype(np.float64) + vals[1:]) / 2).astype(np.float32)
    near = np.concatenate([(m.view(np.int32) + np.arange(-64, 65, dtype=np.int32)).view(np.float32)
                           for m in mids])
    ys = np.concatenate([vals, mids, near, np.exp2(rng.uniform(-12, 10, 1 << 20)).astype(np.float32),
                         np.array([0.0, 1e-30, 448.0, 449.0, 1e9], np.float32)])
    _, _, e4 = fa.debug_convert(torch.from_numpy(ys).cuda(), e4m3=True)
    got = e4.cpu().numpy()
    clamped = np.minimum(np.maximum(ys, np.float32(2.0 ** -9)), np.float32(448.0))
    want = O.e4m3_rne(clamped)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. {ys[bad[:4]]}"


def test_sr_bits_match_oracle():
    need_gpu()
    rng = np.random.default_rng(23)
    idx = np.concatenate([np.arange(4096, dtype=np.uint64),
                          rng.integers(0, 1 << 62, 1 << 16, dtype=np.uint64),
                          np.array([(1 << 35) - 1, 1 << 35, (1 << 64) - 1], dtype=np.uint64)])
    for seed in (0, 1, 0xDEADBEEF12345678):
        got = fa.debug_sr_bits(seed, torch.from_numpy(idx.view(np.int64)).cuda()).cpu().numpy()
        want = O.sr_bits(seed, idx)
        assert np.array_equal(got.view(np.uint32), want)


def test_nv_block_scale_all_bf16_amax():
    """The quantizers' NVFP4 block-scale step (exactly rounded amax / 6, clamp
    to [2^-9, 448], E4M3 code, element multiplier s_enc / decode(code) from a
    table) against the oracle's one-IEEE-operation-at-a-time rule, for every
    non-negative finite bf16 block amax (subnormals and zero included) under
    encode scales from tensor amaxes across the range."""
    need_gpu()
    bits = np.arange(0x7F80, dtype=np.uint32)  # +0 .. largest finite bf16
    amax = (bits << 16).view(np.float32)
    ag = torch.from_numpy(amax.copy()).cuda()
    for amax_t in (1.0, 6.0, 2688.0, 3.5e-3, 1e-30, 3.0e38, float(amax[1])):
        s_enc = O.nv_encode_scale(amax_t)
        codes, mults = fa.debug_nv_block_scale(ag, s_enc)
        codes, mults = codes.cpu().numpy(), mults.cpu().numpy()
        want = [O.nv_block_scale(float(a), s_enc) for a in amax]
        wc = np.array([c for c, _ in want], dtype=np.uint8)
        wm = np.array([m for _, m in want], dtype=np.float32)
        bad = np.nonzero((codes != wc) | (mults.view(np.uint32) != wm.view(np.uint32)))[0]
        assert bad.size == 0, (amax_t, int(bad.size), float(amax[bad[0]]), int(codes[bad[0]]), int(wc[bad[0]]))
