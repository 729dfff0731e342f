"""Pins for the CPU oracle: checks against facts fixed by the pages and by
mathematics, never against the oracle itself.

Each ``pin_*`` raises AssertionError on failure.  ``test_oracle_pins.py`` runs
them on the real oracle; ``test_oracle_planted.py`` runs them on builds with a
planted mistake and expects a failure.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import torch

import oracle as O
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _golden(name):
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, *v = line.split()
                out[k] = v
    return out


def _grid():
    return [float(v) for v in _golden("e2m1_format.txt")["magnitudes"]]


# ------------------------------------------------------------------- E2M1 ---

def pin_e2m1_decode():
    g = _golden("e2m1_format.txt")
    vals = [O.e2m1_decode(c) for c in range(16)]
    assert int(g["codes"][0]) == 16
    assert max(abs(v) for v in vals) == float(g["max_magnitude"][0])
    assert sorted({abs(v) for v in vals}) == _grid()
    # sign bit is the top bit of the 4-bit code: codes 8..15 negate codes 0..7
    for c in range(8):
        assert vals[c] >= 0 and vals[c + 8] == -vals[c]
        assert math.copysign(1.0, vals[c + 8]) == -1.0
    # monotone in the magnitude code (exponent above mantissa)
    assert all(vals[c] < vals[c + 1] for c in range(7))


def _nearest_code_bruteforce(y: float) -> int:
    """Nearest grid value by exhaustive search; ties go to the even code;
    magnitudes beyond 6 give 6; the sign is kept."""
    grid = _grid()
    a = abs(y)
    s = 8 if math.copysign(1.0, y) < 0 else 0
    if a >= grid[-1]:
        return s | 7
    best, bestd = None, None
    for c, v in enumerate(grid):
        d = abs(Fraction(a) - Fraction(v))
        if bestd is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    return s | best


def _e2m1_sweep() -> np.ndarray:
    grid = _grid()
    pts = []
    for v in grid + [(a + b) / 2 for a, b in zip(grid, grid[1:])]:
        for direction in (np.float32(np.inf), np.float32(-np.inf)):
            f = np.float32(v)
            for _ in range(40):
                pts.append(f)
                f = np.nextafter(f, direction, dtype=np.float32)
    # every bf16 value in [-8, 8]
    b = np.arange(0, 1 << 16, dtype=np.uint32)
    f = (b << 16).view(np.float32)
    f = f[np.isfinite(f) & (np.abs(f) <= 8.0)]
    rng = np.random.default_rng(1234)
    r = rng.uniform(-7, 7, 20000).astype(np.float32)
    big = np.array([6.0, 6.5, 7.999, 8.0, 1e6, 3.0e38, 0.0, 1e-30, 1e-45], dtype=np.float32)
    allv = np.concatenate([np.array(pts, dtype=np.float32), f, r, big])
    return np.concatenate([allv, -allv])


def pin_e2m1_rne():
    ys = _e2m1_sweep()
    got = O.e2m1_rne(ys)
    # brute force over a subset (exact rational arithmetic is slow), plus the
    # vectorised nearest search over everything
    grid = np.array(_grid())
    a = np.abs(ys.astype(np.float64))
    d = np.abs(a[:, None] - grid[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = (d == dmin)
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    code = np.where(even.any(axis=1), np.argmax(even, axis=1), np.argmax(cand, axis=1))
    code = np.where(a >= 6.0, 7, code)
    sign = np.signbit(ys).astype(np.int64) * 8
    want = (code + sign).astype(np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"E2M1 RNE mismatch at {ys[bad[:5]]}: got {got[bad[:5]]}, want {want[bad[:5]]}"
    for y in ys[:: max(1, ys.size // 400)]:
        assert int(O.e2m1_rne([y])[0]) == _nearest_code_bruteforce(float(y))
    # the printed tie cases of the round-half-to-even rule
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for y, c in ties.items():
        assert int(O.e2m1_rne([y])[0]) == c, y
        assert int(O.e2m1_rne([-y])[0]) == c | 8, -y
    assert int(O.e2m1_rne([-0.1])[0]) == 8  # sign kept on zero
    assert int(O.e2m1_rne([0.0])[0]) == 0


def pin_e2m1_sr():
    grid = _grid()
    u = np.arange(65536, dtype=np.uint32)
    # on-grid values never move, for every possible 16-bit draw
    for v in grid:
        for s in (1.0, -1.0):
            codes = O.e2m1_sr(np.full(65536, s * v, dtype=np.float32), u)
            want = grid.index(v) | (8 if s < 0 else 0)
            assert np.all(codes == want), (v, s)
    # beyond 6 saturates
    assert np.all(O.e2m1_sr(np.full(65536, 7.5, np.float32), u) == 7)
    # exact expectation: averaging over all 2^16 draws gives
    # lo + g * floor(65536 f) / 65536, within g/65536 of y (unbiased to 2^-16 g)
    rng = np.random.default_rng(7)
    for y in list(rng.uniform(-6, 6, 24).astype(np.float32)) + [np.float32(0.3), np.float32(5.9)]:
        codes = O.e2m1_sr(np.full(65536, y, dtype=np.float32), u)
        counts = np.bincount(codes, minlength=16)
        mean = sum(counts[c] * O.e2m1_decode(c) for c in range(16)) / 65536.0
        a = abs(float(y))
        lo = max(v for v in grid if v <= a)
        hi = min(v for v in grid if v > a)
        g = hi - lo
        assert abs(mean - float(y)) <= g / 65536.0 + 1e-12, (y, mean)
        # only the two neighbours ever appear
        vals = {abs(O.e2m1_decode(c)) for c in range(16) if counts[c]}
        assert vals <= {lo, hi}
    # the number of the 2^16 draws that round up is the integer part of
    # 65536 f (f the fraction between the neighbours), computed here from the
    # grid by exact rational arithmetic, including fractions with bits below
    # 2^-16 (where the integer part and a plain comparison u < 65536 f differ)
    from fractions import Fraction
    for y in (1.0 + 0.5 * 12345.75 / 65536, 0.25 + 2.0 ** -20, 4.0 + 2.0 * 3.5 / 65536,
              2.0 ** -17 * 1.5, 0.6 + 2.0 ** -19, 5.0 + 2.0 ** -21):
        y32 = np.float32(y)
        a = Fraction(float(y32))
        lo = max(Fraction(v) for v in grid if Fraction(v) <= a)
        hi = min(Fraction(v) for v in grid if Fraction(v) > a)
        ups = int(np.sum(np.abs([O.e2m1_decode(c) for c in
                                 O.e2m1_sr(np.full(65536, y32, np.float32), u)]) == float(hi)))
        assert ups == int((a - lo) / (hi - lo) * 65536), (y, ups)
    # with the Philox stream: 10^5 draws, mean within 3 sigma
    for y in (np.float32(0.3), np.float32(-2.7), np.float32(4.9)):
        n = 100000
        bits = O.sr_bits(99, np.arange(n, dtype=np.uint64))
        codes = O.e2m1_sr(np.full(n, y, dtype=np.float32), bits)
        vals = np.array([O.e2m1_decode(c) for c in range(16)])[codes]
        a = abs(float(y))
        lo = max(v for v in grid if v <= a)
        hi = min(v for v in grid if v > a)
        p = (a - lo) / (hi - lo)
        sigma = (hi - lo) * math.sqrt(p * (1 - p) / n)
        assert abs(vals.mean() - float(y)) <= 3 * sigma + (hi - lo) / 65536.0, (y, vals.mean())


# ------------------------------------------------------------------- E4M3 ---

def _e4m3_value(code: int) -> float:
    """E4M3 by its definition: bias 7, 3 mantissa bits, subnormals at e=0."""
    e, m = (code >> 3) & 15, code & 7
    if e == 0:
        return m * 2.0 ** -9
    return (8 + m) * 2.0 ** (e - 10)


def pin_e4m3():
    g = _golden("nvfp4_contract.txt")
    vals = [O.e4m3_decode(c) for c in range(127)]
    assert vals == [_e4m3_value(c) for c in range(127)]
    assert max(vals) == float(g["e4m3_max"][0]) == vals[0x7E]
    assert vals[1] == float(g["e4m3_min_subnormal"][0])
    assert vals[8] == float(g["e4m3_min_normal"][0])
    assert math.isnan(O.e4m3_decode(int(g["e4m3_nan_code"][0])))
    # RNE encode against brute-force nearest (ties to even code), saturating at 448
    rng = np.random.default_rng(11)
    xs = np.concatenate([
        np.exp2(rng.uniform(-10, 9.5, 30000)).astype(np.float32),
        np.array(vals[1:], np.float32),
        np.array([(a + b) / 2 for a, b in zip(vals[1:], vals[2:])], np.float32),
        np.array([448.0, 460.0, 479.0, 1e6, 2.0 ** -9, 2.0 ** -10, 2.0 ** -10 * 1.5], np.float32),
    ])
    got = O.e4m3_rne(xs)
    table = np.array(vals)
    d = np.abs(xs.astype(np.float64)[:, None] - table[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    even = cand & (np.arange(127)[None, :] % 2 == 0)
    want = np.where(even.any(axis=1), np.argmax(even, axis=1), np.argmax(cand, axis=1))
    want = np.where(xs >= 448.0, 0x7E, want)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (xs[bad[:5]], got[bad[:5]], want[bad[:5]])


# ----------------------------------------------------------------- scales ---

def pin_mx_exponent():
    # every positive finite bf16 value: 4 <= amax * 2^-e < 8 unless clamped
    b = np.arange(1, 0x7F80, dtype=np.uint32)
    amax = (b << 16).view(np.float32)
    for a in amax[:: 7]:
        e = O.mx_exponent(float(a))
        assert -127 <= e <= 127
        v = float(a) * 2.0 ** (-e)
        if e > -127:
            assert 4.0 <= v < 8.0, (a, e)
        else:
            assert v < 8.0
    assert O.mx_exponent(0.0) == -127
    assert O.mx_exponent(3.3895313892515355e38) == 125
    assert O.mx_exponent(9.183549615799121e-41) == -127
    assert O.mx_exponent(6.0) == 0 and O.mx_exponent(4.0) == 0 and O.mx_exponent(8.0) == 1
    assert O.mx_exponent(3.99) == -1



def pin_mx_exponent_noclip():
    """The no-clip MXFP4 exponent is the smallest e with amax <= 6 * 2^e
    (clamped to [-127, 127]): checked by its definition on every positive
    finite bf16 value, and no element of a no-clip block saturates."""
    bits = np.arange(1, 0x7F80, dtype=np.uint32) << 16          # positive finite bf16
    vals = bits.view(np.float32)
    for a in vals[:: 7]:
        a = float(a)
        e = O.mx_exponent_noclip(a)
        if e > -127:
            assert a <= 6.0 * 2.0 ** e and a > 6.0 * 2.0 ** (e - 1), (a, e)
        else:
            assert a <= 6.0 * 2.0 ** -127 or a <= 6.0 * 2.0 ** e, (a, e)
    assert O.mx_exponent_noclip(0.0) == -127
    assert O.mx_exponent_noclip(6.0) == 0 and O.mx_exponent_noclip(6.0000005) == 1
    assert O.mx_exponent_noclip(1.5) == -2 and O.mx_exponent_noclip(1.5000001) == -1
    # a block quantized with it never saturates: the block max lands on a
    # grid value within half a grid step, never clipped to 6 from above
    rng = np.random.default_rng(3)
    x = torch.from_numpy((rng.standard_normal((128, 256)) * 3).astype(np.float32)).to(torch.bfloat16)
    q = O.quantize(x, O.MXFP4_NOCLIP)
    d = O.dequantize(q)
    xf = x.float().numpy().astype(np.float64)
    for r in range(0, 128, 17):
        for kb in range(0, 256, 32):
            blk = xf[r, kb:kb + 32]
            e = O.mx_exponent_noclip(float(np.abs(blk).max()))
            assert np.all(np.abs(blk) * 2.0 ** -e <= 6.0)
            step = 2.0 ** (e + 1)                                  # largest grid step (4 -> 6)
            assert np.all(np.abs(d[r, kb:kb + 32] - blk) <= step / 2 + 1e-30)


def pin_nv_scales():
    g = _golden("nvfp4_contract.txt")
    emax = float(g["e4m3_max"][0])
    rng = np.random.default_rng(5)
    for amax_t in list(np.exp2(rng.uniform(-40, 40, 200)).astype(np.float32)) + [np.float32(1.0)]:
        s_enc = O.nv_encode_scale(float(amax_t))
        ts = O.nv_decode_scale(s_enc)
        # the decode scale maps the tensor amax onto 6 * E4M3-max (two roundings)
        assert abs(ts * 6.0 * emax - float(amax_t)) <= 3 * np.spacing(np.float32(amax_t)), amax_t
        for frac in (1.0, 0.5, 0.1, 1e-3):
            amax_b = np.float32(amax_t * frac)
            code, mult = O.nv_block_scale(float(amax_b), s_enc)
            sv = _e4m3_value(code)
            # block scale * decode scale ~ amax_b / 6 within E4M3's 2^-4 relative rounding
            assert abs(sv * ts - amax_b / 6.0) <= 2.0 ** -4 * amax_b / 6.0 * 1.001, (amax_t, frac)
            # the element multiplier takes the block max to about 6
            assert 6.0 * (1 - 2 ** -3) <= amax_b * mult <= 6.0 * (1 + 2 ** -3)
    assert O.nv_encode_scale(0.0) == 1.0
    assert O.nv_decode_scale(O.nv_encode_scale(0.0)) == 1.0
    # zero block: clamped to the smallest E4M3 value
    code, mult = O.nv_block_scale(0.0, O.nv_encode_scale(10.0))
    assert code == 1
    # a block 10^6 below the tensor amax clamps up; 10^5 below does not
    s = O.nv_encode_scale(1.0)
    assert O.nv_block_scale(1e-6, s)[0] == 1
    assert O.nv_block_scale(1e-5, s)[0] > 1
    # a block at the tensor amax takes the largest scale
    assert O.nv_block_scale(1.0, s)[0] == 0x7E


# -------------------------------------------------------------- Hadamard ---

def pin_hadamard():
    H = np.stack([O.hadamard32(np.eye(32, dtype=np.float32)[j], 0) for j in range(32)], axis=1)
    # Sylvester closed form
    want = np.array([[(-1) ** bin(i & j).count("1") for j in range(32)] for i in range(32)], float)
    assert np.array_equal(H, want)
    assert np.array_equal(H @ H.T, 32 * np.eye(32))
    # fixed signs act on the input: H diag(s)
    mask = 0x9E3779B9
    s = np.array([-1.0 if (mask >> j) & 1 else 1.0 for j in range(32)])
    rng = np.random.default_rng(3)
    for _ in range(20):
        x = rng.integers(-20, 21, 32).astype(np.float32)
        assert np.array_equal(O.hadamard32(x, mask), (want @ (s * x)).astype(np.float32))
    # weight-gradient identity (R dY)^T (R X) = 32 dY^T X, R = H diag(s), exact on integers
    dy = rng.integers(-4, 5, (32, 6)).astype(np.float32)
    xx = rng.integers(-4, 5, (32, 5)).astype(np.float32)
    rdy = np.stack([O.hadamard32(dy[:, c], mask) for c in range(6)], axis=1).astype(np.float64)
    rx = np.stack([O.hadamard32(xx[:, c], mask) for c in range(5)], axis=1).astype(np.float64)
    assert np.array_equal(rdy.T @ rx, 32.0 * (dy.T.astype(np.float64) @ xx.astype(np.float64)))


# --------------------------------------------------------------- swizzle ---

def pin_swizzle():
    # bijection onto [0, padded bytes) for several shapes
    for rows, kbt in ((128, 4), (256, 8), (384, 12), (128, 32)):
        offs = {O.sf_offset(r, kb, kbt) for r in range(rows) for kb in range(kbt)}
        assert len(offs) == rows * kbt
        assert min(offs) == 0 and max(offs) == O.sf_bytes(rows, kbt) - 1
    # one atom is 512 contiguous bytes holding 128 rows x 4 blocks, and four
    # consecutive blocks of one row share one 32-bit word
    for r in range(128):
        base = O.sf_offset(r, 0, 4)
        assert base % 4 == 0
        assert [O.sf_offset(r, kb, 4) - base for kb in range(4)] == [0, 1, 2, 3]
    # rows r, r+32, r+64, r+96 share one 16-byte line
    for r in range(32):
        line = {O.sf_offset(r + 32 * j, 0, 4) // 16 for j in range(4)}
        assert len(line) == 1
        assert [O.sf_offset(r + 32 * j, 0, 4) % 16 for j in range(4)] == [0, 4, 8, 12]
    # K-direction atoms are adjacent in memory before the next 128 rows
    assert O.sf_offset(0, 4, 8) == 512 and O.sf_offset(128, 0, 8) == 1024


# ---------------------------------------------------------- quantization ---

def _bf16_np(x: torch.Tensor) -> np.ndarray:
    return x.float().numpy().astype(np.float64)


def _check_quant_bounds(x: torch.Tensor, q: O.QTensor, fmt: int, orient: int,
                        hadamard_mask=None, sr=False):
    """Element-wise closed-form error bound and the per-block scale invariants,
    computed from the input with numpy (independent of the oracle's code)."""
    xv = _bf16_np(x)
    Q = xv if orient == O.ROWWISE else xv.T
    R, K = Q.shape
    bs = O.BLOCK[fmt]
    if hadamard_mask is not None:
        s = np.array([-1.0 if (hadamard_mask >> j) & 1 else 1.0 for j in range(32)])
        Hs = np.array([[(-1) ** bin(i & j).count("1") for j in range(32)] for i in range(32)]) * s[None, :]
        Q = (Q.reshape(R, K // 32, 32) @ Hs.T).reshape(R, K)
    deq = O.dequantize(q)
    blocks = Q.reshape(R, K // bs, bs)
    amax_b = np.abs(blocks).max(axis=2)
    # block scale bytes through the layout
    kb = np.arange(K // bs)
    offs = np.array([[O.sf_offset(r, k, K // bs) for k in kb] for r in range(R)])
    sbytes = q.scales[offs].astype(np.int64)
    if fmt == O.MXFP4:
        scale = np.exp2(sbytes - 127.0)
        ratio = amax_b / scale
        live = sbytes > 0
        assert np.all((ratio[live] >= 4.0) & (ratio[live] < 8.0)), "MX scale invariant"
        assert np.all(amax_b[~live] < 8.0 * 2.0 ** -127)
        eff = np.repeat(scale, bs, axis=1)
    else:
        sv = np.vectorize(_e4m3_value)(sbytes)
        if fmt == O.NVFP4_GLOBAL:
            amax_t = np.abs(Q).max()
            ts = np.full((R, K // bs), float(q.ts[0]))
            assert abs(float(q.ts[0]) * 2688.0 - amax_t) <= 3 * np.spacing(np.float32(amax_t)) or amax_t == 0
        else:
            # 128x128 tiles; those at a ragged edge hold fewer values (zero
            # padding leaves a tile's amax unchanged)
            nr, nk = -(-R // 128), -(-K // 128)
            t = q.ts.reshape(nr, nk).astype(np.float64)
            Qa = np.zeros((nr * 128, nk * 128))
            Qa[:R, :K] = np.abs(Q)
            tile_amax = Qa.reshape(nr, 128, nk, 128).max(axis=(1, 3))
            nz = tile_amax > 0
            assert np.all(np.abs(t[nz] * 2688.0 - tile_amax[nz]) <= 3 * np.spacing(tile_amax[nz].astype(np.float32)))
            ts = np.repeat(np.repeat(t, 128, axis=0), 128 // bs, axis=1)[:R, :K // bs]
        eff_b = sv * ts
        live = amax_b > 2 ** -9 * 448 * 6 * ts * 1.01 / 448  # not clamped at the bottom
        rel = np.abs(eff_b[live] - amax_b[live] / 6.0) / (amax_b[live] / 6.0)
        assert np.all(rel <= 2.0 ** -4 * 1.001), "NV block scale ~ amax_b/6"
        eff = np.repeat(eff_b, bs, axis=1)
    # scaled-domain error bound: |Q/eff - code| <= half the grid spacing there,
    # or the saturation distance above 6
    y = Q / eff
    c = deq / eff
    a = np.abs(y)
    gap = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    err = np.abs(y - c)
    sat = a > 6.0
    if sr:  # one of the two neighbouring grid values
        ok = np.where(sat, np.abs(c) == 6.0, err < gap + 1e-6 * a)
    else:
        ok = np.where(sat, np.abs(c) == 6.0, err <= gap / 2 + 1e-6 * a)
    assert np.all(ok), f"quantization error bound violated at {np.argwhere(~ok)[:3].tolist()}"
    # signs agree wherever the value is nonzero
    nzc = c != 0
    assert np.all(np.sign(c[nzc]) == np.sign(y[nzc]))


def pin_quantize_rne():
    x = workloads.with_specials(workloads.tiny(0))
    for fmt in (O.MXFP4, O.NVFP4_GLOBAL, O.NVFP4_CTA):
        for orient in (O.ROWWISE, O.COLWISE):
            q = O.quantize(x, fmt, O.RNE, orient)
            _check_quant_bounds(x, q, fmt, orient)
    # outlier-heavy sweep recipe at a small size
    xs = workloads.sweep(256, 384, seed=3)
    for fmt in (O.MXFP4, O.NVFP4_GLOBAL, O.NVFP4_CTA):
        _check_quant_bounds(xs, O.quantize(xs, fmt, O.RNE, O.ROWWISE), fmt, O.ROWWISE)


def pin_quantize_sr():
    x = workloads.with_specials(workloads.tiny(0))[:128, :256].contiguous()
    for fmt in (O.MXFP4, O.NVFP4_GLOBAL, O.NVFP4_CTA):
        q = O.quantize(x, fmt, O.SR, O.ROWWISE, seed=1)
        r = O.quantize(x, fmt, O.RNE, O.ROWWISE)
        # the rounding mode changes elements only, never the scales
        assert np.array_equal(q.scales, r.scales) and np.array_equal(q.ts, r.ts)
        _check_quant_bounds(x, q, fmt, O.ROWWISE, sr=True)
        # and it does change some elements
        assert not np.array_equal(q.payload, r.payload)
    # unbiased on average over seeds
    xb = torch.full((128, 256), 0.7, dtype=torch.bfloat16)
    xb[:, ::32] = 5.0  # sets the MX block max so that 0.7 is off-grid after scaling
    acc = np.zeros((128, 256))
    n = 64
    for sd in range(n):
        acc += O.dequantize(O.quantize(xb, O.MXFP4, O.SR, O.ROWWISE, seed=sd))
    m = acc[:, 1:32].mean() / n
    assert abs(m - float(torch.tensor(0.7, dtype=torch.bfloat16))) < 0.01, m


def pin_quantize_orientation():
    x = workloads.sweep(256, 384, seed=5)
    for fmt in (O.MXFP4, O.NVFP4_GLOBAL, O.NVFP4_CTA):
        for rnd in (O.RNE, O.SR):
            a = O.quantize(x, fmt, rnd, O.COLWISE, seed=9)
            b = O.quantize(x.t().contiguous(), fmt, rnd, O.ROWWISE, seed=9)
            assert np.array_equal(a.payload, b.payload) and np.array_equal(a.scales, b.scales)
            assert np.array_equal(a.ts, b.ts)


def pin_quantize_hadamard():
    rng = np.random.default_rng(8)
    xi = rng.integers(-3, 4, (256, 128)).astype(np.float32)  # [T, C]
    x = torch.from_numpy(xi).to(torch.bfloat16)
    mask = 0x2545F491
    s = np.array([-1.0 if (mask >> j) & 1 else 1.0 for j in range(32)])
    Hs = np.array([[(-1) ** bin(i & j).count("1") for j in range(32)] for i in range(32)]) * s[None, :]
    # transform along T (columns of the [C, T] view) by a plain matmul; small
    # integers keep every sum exact and representable in bf16
    xt = xi.T.reshape(128, 256 // 32, 32) @ Hs.T
    pre = torch.from_numpy(np.ascontiguousarray(xt.reshape(128, 256).T.astype(np.float32))).to(torch.bfloat16)
    assert np.array_equal(pre.float().numpy(), xt.reshape(128, 256).T)
    a = O.quantize(x, O.MXFP4, O.RNE, O.COLWISE, hadamard_mask=mask)
    b = O.quantize(pre, O.MXFP4, O.RNE, O.COLWISE)
    assert np.array_equal(a.payload, b.payload) and np.array_equal(a.scales, b.scales)
    _check_quant_bounds(x, a, O.MXFP4, O.COLWISE, hadamard_mask=mask)


def pin_packing():
    # a row whose quantized codes are known by construction: MX block max 6
    vals = np.array([6, 0, 0.5, 1, 1.5, 2, 3, 4] * 4, dtype=np.float32)
    x = torch.zeros(128, 128, dtype=torch.bfloat16)
    x[0, :32] = torch.from_numpy(vals).to(torch.bfloat16)
    x[0, 32:64] = torch.from_numpy(-vals).to(torch.bfloat16)
    q = O.quantize(x, O.MXFP4, O.RNE, O.ROWWISE)
    grid = _grid()
    codes = [grid.index(abs(v)) for v in vals]
    want = bytes((codes[2 * j] | (codes[2 * j + 1] << 4)) for j in range(16))
    assert bytes(q.payload[0, :16]) == want
    wneg = bytes(((codes[2 * j] | 8) | ((codes[2 * j + 1] | 8) << 4)) for j in range(16))
    assert bytes(q.payload[0, 16:32]) == wneg
    assert q.scales[O.sf_offset(0, 0, 4)] == 127  # 6 -> exponent 0


def _valid_scale_offsets(R: int, kb_total: int) -> np.ndarray:
    return np.array([O.sf_offset(r, k, kb_total) for r in range(R) for k in range(kb_total)])


def pin_quantize_ragged():
    """Row counts that are not a multiple of 128 and K that is not a multiple
    of 128 (MX/NV blocks still whole): the closed-form bounds hold, and the
    result equals the valid part of the same tensor zero-padded to whole
    128x128 tiles -- zero rows and columns change no block, tensor or tile
    amax.  Scale bytes outside the valid rows and blocks are zero."""
    for (R, K) in ((200, 352), (1, 96), (129, 160)):
        x = workloads.sweep(max(R, 2), K, seed=R + K)[:R].contiguous()
        Rp, Kp = -(-R // 128) * 128, -(-K // 128) * 128
        xp = torch.zeros(Rp, Kp, dtype=torch.bfloat16)
        xp[:R, :K] = x
        xr = torch.zeros(Rp, K, dtype=torch.bfloat16)  # rows padded only: same SR indices
        xr[:R] = x
        for fmt in (O.MXFP4, O.MXFP4_NOCLIP, O.NVFP4_GLOBAL, O.NVFP4_CTA):
            bs = O.BLOCK[fmt]
            q = O.quantize(x, fmt, O.RNE, O.ROWWISE)
            if fmt != O.MXFP4_NOCLIP:
                _check_quant_bounds(x, q, fmt, O.ROWWISE)
            assert q.payload.shape == (R, K // 2)
            assert q.scales.size == Rp * (-(-(K // bs) // 4) * 4)
            assert q.ts.size == (0 if O.BLOCK[fmt] == 32 else O.ts_count(R, K, fmt))
            valid = _valid_scale_offsets(R, K // bs)
            pad = np.setdiff1d(np.arange(q.scales.size), valid)
            assert np.all(q.scales[pad] == 0)
            for xpad, rnd in ((xp, O.RNE), (xr, O.SR)):
                p = O.quantize(xpad, fmt, rnd, O.ROWWISE, seed=5)
                g = q if rnd == O.RNE else O.quantize(x, fmt, O.SR, O.ROWWISE, seed=5)
                assert np.array_equal(g.payload, p.payload[:R, :K // 2]), (R, K, fmt, rnd)
                Kbp = xpad.shape[1] // bs
                vp = np.array([O.sf_offset(r, k, Kbp) for r in range(R) for k in range(K // bs)])
                assert np.array_equal(g.scales[valid], p.scales[vp]), (R, K, fmt, rnd)
                assert np.array_equal(g.ts, p.ts), (R, K, fmt, rnd)
        # column-wise: the token dimension K of the quantized operand is ragged
        xc = workloads.sweep(K, max(R, 2), seed=7)[:, :R].contiguous()
        for fmt in (O.MXFP4, O.NVFP4_CTA):
            a = O.quantize(xc, fmt, O.RNE, O.COLWISE)
            b = O.quantize(xc.t().contiguous(), fmt, O.RNE, O.ROWWISE)
            assert np.array_equal(a.payload, b.payload) and np.array_equal(a.scales, b.scales)
            assert np.array_equal(a.ts, b.ts)


# ------------------------------------------------------------------ GEMM ---

def pin_gemm_bruteforce():
    rng = np.random.default_rng(21)
    for fmt in (O.MXFP4, O.NVFP4_GLOBAL, O.NVFP4_CTA):
        for K in (128, 256, 512):
            xa = torch.from_numpy(rng.standard_normal((128, K)).astype(np.float32)).to(torch.bfloat16)
            xb = torch.from_numpy((rng.standard_normal((256, K)) * 3).astype(np.float32)).to(torch.bfloat16)
            xb[:, :K // 2] *= 0.01  # different tiles get different second-level scales
            xb[128:] *= 40.0
            A = O.quantize(xa, fmt)
            B = O.quantize(xb, fmt)
            alpha = 0.75
            mi = rng.choice(128, 6, replace=False)
            ni = np.concatenate([rng.choice(128, 3, replace=False), 128 + rng.choice(128, 3, replace=False)])
            got = O.gemm(A, B, alpha, mi, ni)
            # exact rational brute force from the fully dequantized values
            da = O.dequantize(A, mi)
            db = O.dequantize(B, ni)
            for i in range(6):
                for j in range(6):
                    s = sum(Fraction(float(da[i, k])) * Fraction(float(db[j, k])) for k in range(K))
                    want = float(Fraction(alpha) * s)
                    assert abs(got[i, j] - want) <= 1e-12 * max(1.0, abs(want)), (fmt, K, i, j)
            # and the large-shape helper agrees
            assert np.allclose(O.gemm_sampled(A, B, alpha, mi, ni), got, rtol=1e-13, atol=0)


def pin_gemm_ragged():
    """M, N and K that are not multiples of 128: the GEMM equals the valid
    block of the GEMM of the zero-padded operands (binary64 sums are exact,
    so equality is exact), and exact rational brute force on sampled entries."""
    rng = np.random.default_rng(23)
    for fmt in (O.MXFP4, O.NVFP4_GLOBAL, O.NVFP4_CTA):
        M, N, K = 200, 72, 352
        xa = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
        xb = torch.from_numpy((rng.standard_normal((N, K)) * 3).astype(np.float32)).to(torch.bfloat16)
        xb[:, 300:] *= 50.0  # the ragged last K chunk gets its own tile scale
        pa = torch.zeros(256, 384, dtype=torch.bfloat16)
        pb = torch.zeros(128, 384, dtype=torch.bfloat16)
        pa[:M, :K], pb[:N, :K] = xa, xb
        A, B = O.quantize(xa, fmt), O.quantize(xb, fmt)
        d = O.gemm(A, B, 0.5)
        dp = O.gemm(O.quantize(pa, fmt), O.quantize(pb, fmt), 0.5)
        assert np.array_equal(d, dp[:M, :N]), fmt
        assert np.array_equal(O.gemm_sampled(A, B, 0.5), d), fmt
        da, db = O.dequantize(A, [0, 199]), O.dequantize(B, [3, 71])
        for i, m in enumerate((0, 199)):
            for j, n in enumerate((3, 71)):
                s = sum(Fraction(float(da[i, k])) * Fraction(float(db[j, k])) for k in range(K))
                assert abs(d[m, n] - float(Fraction(1, 2) * s)) <= 1e-12 * max(1.0, abs(d[m, n]))


def pin_gemm_approximates_matmul():
    """Quantize-then-GEMM approximates the exact bf16 matmul: catches a
    transposed operand or a dropped scale (relative error of FP4 ~ 0.1)."""
    rng = np.random.default_rng(4)
    xa = torch.from_numpy(rng.standard_normal((256, 512)).astype(np.float32)).to(torch.bfloat16)
    xb = torch.from_numpy((rng.standard_normal((128, 512)) * 0.02).astype(np.float32)).to(torch.bfloat16)
    ref = _bf16_np(xa) @ _bf16_np(xb).T
    for fmt in (O.MXFP4, O.NVFP4_GLOBAL, O.NVFP4_CTA):
        d = O.gemm(O.quantize(xa, fmt), O.quantize(xb, fmt))
        rel = np.linalg.norm(d - ref) / np.linalg.norm(ref)
        assert rel < (0.2 if fmt == O.MXFP4 else 0.16), (fmt, rel)


# --------------------------------------------------------------- Philox ---

def pin_philox_structure():
    k = _golden("philox_constants.txt")
    m0, m1 = int(k["M0"][0], 16), int(k["M1"][0], 16)
    # two rounds from zero: the first round maps 0 -> key, the second exposes
    # the key-schedule increments (golden ratio and sqrt(3)-1, 32-bit fixed point)
    w0 = int(math.floor(((1 + math.sqrt(5)) / 2 - 1) * 2 ** 32))
    w1 = int(math.floor((math.sqrt(3) - 1) * 2 ** 32))
    assert list(O.philox4x32([0, 0, 0, 0], [0, 0], 2)) == [w0, 0, w1, 0]
    # one round exposes the multipliers through the low words
    assert int(O.philox4x32([1, 0, 0, 0], [0, 0], 1)[3]) == m0
    assert int(O.philox4x32([0, 0, 1, 0], [0, 0], 1)[1]) == m1
    # high words of the products land XORed with the key and the other words
    out = O.philox4x32([3, 5, 7, 11], [13, 17], 1)
    assert int(out[0]) == (((m1 * 7) >> 32) ^ 5 ^ 13)
    assert int(out[2]) == (((m0 * 3) >> 32) ^ 11 ^ 17)
    # statistics of the 16-bit stream: uniform bytes, balanced bits, seeds differ
    bits = O.sr_bits(12345, np.arange(1 << 18, dtype=np.uint64))
    assert bits.max() <= 0xFFFF
    hist = np.bincount((bits >> 8).astype(np.int64), minlength=256)
    exp = bits.size / 256
    chi2 = float(((hist - exp) ** 2 / exp).sum())
    assert chi2 < 400, chi2  # 255 dof; p ~ 1e-8 at 400
    ones = np.unpackbits(bits.astype(">u2").view(np.uint8)).mean()
    assert abs(ones - 0.5) < 0.005
    other = O.sr_bits(12346, np.arange(1 << 12, dtype=np.uint64))
    assert np.mean(other == bits[: 1 << 12]) < 0.01
    # eight elements per Philox block of sr_rounds() (= 7) rounds: indices
    # 8j..8j+7 use the four words
    assert O.sr_rounds() == 7
    b = O.sr_bits(1, np.arange(16, dtype=np.uint64))
    w = O.philox4x32([0, 0, 0, 0], [1, 0], O.sr_rounds())
    assert [int(v) for v in b[:8]] == [int(w[i // 2] >> (16 * (i % 2))) & 0xFFFF for i in range(8)]
    # 64-bit counter: the high word comes from index bits 35..
    hi = O.sr_bits(1, np.array([1 << 35], dtype=np.uint64))
    w2 = O.philox4x32([0, 1, 0, 0], [1, 0], O.sr_rounds())
    assert int(hi[0]) == int(w2[0]) & 0xFFFF


# ------------------------------------------------------------ SwiGLU ---

def pin_exp_f32():
    """The producer's binary32 exp against binary64 exp: within 3 units in the
    last place over the whole clamped range, exact at 0, monotone, and the
    clamp ends."""
    x = np.linspace(-87.0, 88.0, 400001).astype(np.float32)
    e = O.exp_f32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    rel = np.abs(e - ref) / ref
    assert rel.max() <= 3 * 2.0 ** -23, rel.max()
    assert float(O.exp_f32([0.0])[0]) == 1.0
    assert np.all(np.diff(e) >= 0)
    assert O.exp_f32([-100.0])[0] == O.exp_f32([-87.0])[0]
    assert O.exp_f32([100.0])[0] == O.exp_f32([88.0])[0]


def pin_swiglu():
    """silu(g) = g / (1 + e^-g) against binary64; h = silu(gate) * up rounded
    to bf16 against the binary64 product (the nearest bf16, or a neighbour only
    where the exact value lies within a few binary32 units of a bf16
    rounding boundary); gate and up taken from the two halves of z."""
    assert O.silu_f32(0.0) == 0.0
    for g in (20.0, 30.0, 87.5):
        assert O.silu_f32(g) == g
    gs = np.linspace(-80.0, 80.0, 20001).astype(np.float32)
    got = np.array([O.silu_f32(float(g)) for g in gs])
    g64 = gs.astype(np.float64)
    ref = g64 / (1.0 + np.exp(-g64))
    nz = np.abs(ref) > 1e-30
    assert np.max(np.abs(got[nz] - ref[nz]) / np.abs(ref[nz])) <= 6 * 2.0 ** -24
    gen = torch.Generator().manual_seed(7)
    T, F = 64, 96
    gate = torch.randn(T, F, generator=gen) * 3.0
    up = torch.randn(T, F, generator=gen) * 0.25 + 0.1
    z = torch.cat([gate, up], dim=1).to(torch.bfloat16)
    h = O.swiglu_bf16(z).astype(np.uint32) << 16
    hv = h.view(np.float32).astype(np.float64)
    g64 = z[:, :F].float().double().numpy()
    u64 = z[:, F:].float().double().numpy()
    exact = g64 / (1.0 + np.exp(-g64)) * u64
    want = torch.from_numpy(exact).to(torch.bfloat16).float().double().numpy()  # RNE to bf16
    ulp_bf16 = np.exp2(np.floor(np.log2(np.maximum(np.abs(exact), 1e-38))) - 7)
    frac = np.abs(exact) / ulp_bf16 - np.floor(np.abs(exact) / ulp_bf16)
    near_tie = np.abs(frac - 0.5) < 2.0 ** -12  # within a few binary32 units of a midpoint
    same = hv == want
    assert np.all(same | (near_tie & (np.abs(hv - want) <= ulp_bf16 * 1.0001))), \
        int((~same & ~near_tie).sum())
    assert same.mean() > 0.999


ALL_PINS = [pin_e2m1_decode, pin_e2m1_rne, pin_e2m1_sr, pin_e4m3, pin_mx_exponent,
            pin_mx_exponent_noclip, pin_nv_scales,
            pin_hadamard, pin_swizzle, pin_quantize_rne, pin_quantize_sr, pin_quantize_orientation,
            pin_quantize_hadamard, pin_packing, pin_quantize_ragged, pin_gemm_bruteforce,
            pin_gemm_ragged, pin_gemm_approximates_matmul,
            pin_philox_structure, pin_exp_f32, pin_swiglu]
