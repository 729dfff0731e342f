"""Helpers shared by the GPU parity tests (comparison against the oracle)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import fp4_quantization_block_b200 as fa
import oracle as O

FMTS = [fa.MXFP4, fa.NVFP4_GLOBAL, fa.NVFP4_CTA, fa.MXFP4_NOCLIP]
FMT_IDS = {fa.MXFP4: "mx", fa.NVFP4_GLOBAL: "nvg", fa.NVFP4_CTA: "nvc", fa.MXFP4_NOCLIP: "mxnc"}


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def to_cpu_qt(q: fa.QTensor) -> O.QTensor:
    ts = q.ts.cpu().numpy() if q.ts is not None else np.zeros(0, np.float32)
    return O.QTensor(q.payload.cpu().numpy(), q.scales.cpu().numpy(), ts, q.R, q.K, q.fmt)


def to_gpu_qt(q: O.QTensor, device="cuda") -> fa.QTensor:
    ts = torch.from_numpy(q.ts.copy()).to(device) if q.ts.size else None
    return fa.QTensor(torch.from_numpy(q.payload.copy()).to(device),
                      torch.from_numpy(q.scales.copy()).to(device), ts, q.R, q.K, q.fmt)


def scale_byte_range(q: O.QTensor, r0: int, r1: int) -> slice:
    """Scale bytes of the 128-row atom rows that hold rows r0 .. r1-1 (with
    the padding of a ragged last atom row)."""
    kb4 = -(-(q.K // O.BLOCK[q.fmt]) // 4)
    return slice((r0 // 128) * kb4 * 512, -(-r1 // 128) * kb4 * 512)


def assert_qt_equal(g: O.QTensor, o: O.QTensor, row_range=None):
    """Bit-exact comparison of payload, scale bytes and FP32 second-level scales."""
    assert (g.R, g.K, g.fmt) == (o.R, o.K, o.fmt)
    r0, r1 = row_range if row_range else (0, g.R)
    gp, op = g.payload[r0:r1], o.payload[r0:r1]
    if not np.array_equal(gp, op):
        bad = np.argwhere(gp != op)
        r, c = bad[0]
        raise AssertionError(f"payload differs at {len(bad)} bytes; first row {r0 + r} byte {c}: "
                             f"gpu {gp[r, c]:#04x} oracle {op[r, c]:#04x}")
    sl = scale_byte_range(g, r0, r1)
    gs, os_ = g.scales[sl], o.scales[sl]
    if not np.array_equal(gs, os_):
        bad = np.nonzero(gs != os_)[0]
        raise AssertionError(f"scale bytes differ at {len(bad)} offsets; first {sl.start + bad[0]}: "
                             f"gpu {gs[bad[0]]} oracle {os_[bad[0]]}")
    if g.fmt == O.NVFP4_GLOBAL:
        assert g.ts.view(np.uint32)[0] == o.ts.view(np.uint32)[0], (g.ts, o.ts)
    elif g.fmt == O.NVFP4_CTA:
        nk = -(-g.K // 128)
        gt = g.ts.reshape(-1, nk)[r0 // 128:-(-r1 // 128)]
        ot = o.ts.reshape(-1, nk)[r0 // 128:-(-r1 // 128)]
        assert np.array_equal(gt.view(np.uint32), ot.view(np.uint32))


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


U32 = 2.0 ** -24  # unit roundoff of binary32


def accumulation_bound(A: O.QTensor, B: O.QTensor, alpha: float = 1.0, m_idx=None, n_idx=None):
    """Per-output bound on |D_gpu - D_exact| from binary32 accumulation:
    (gamma_K + 8u) * |alpha| * sum_k |a_k| |b_k|, with gamma_K = K u / (1 - K u)
    the recursive-summation bound and a_k, b_k the dequantized operands
    (second-level scales included; u = 2^-24).  The 8u covers the few
    roundings outside the sum: alpha and the tensor-scale product, the
    CTA-local chunk factor and its fused fold.  Far tighter than the
    configuration's tolerance: a wrong scale on one block row or tile fails
    it."""
    a = np.abs(O.dequantize(A, m_idx))
    b = np.abs(O.dequantize(B, n_idx))
    K = A.K
    gamma = K * U32 / (1.0 - K * U32)
    return (gamma + 8 * U32) * abs(alpha) * (a @ b.T)


def assert_gemm_close(d_gpu: np.ndarray, d_orc: np.ndarray, tol: float, bf16: bool = False,
                      tight=None):
    """max |D_gpu - D_oracle| <= tol (plus half a bf16 ulp of the exact value
    for bf16 output) and, when `tight` (accumulation_bound) is given, every
    element within its accumulation bound too.  Prints the observed worst
    ratios to both bounds."""
    d_gpu = d_gpu.astype(np.float64)
    err = np.abs(d_gpu - d_orc)
    half = bf16_half_ulp(d_orc) if bf16 else 0.0
    allow = tol + half
    worst = float((err - allow).max())
    assert np.all(err <= allow), f"max|err| {err.max():.3e} exceeds the bound by {worst:.3e} (tol {tol:.3e})"
    msg = f"{'bf16' if bf16 else 'fp32'} out: max|err| {err.max():.3e} = {err.max() / tol:.2e} of tol"
    if tight is not None:
        t_allow = tight + half
        ratio = float((err / np.where(t_allow > 0, t_allow, np.inf)).max())
        msg += f", {ratio:.3f} of the accumulation bound"
        bad = err > t_allow
        if np.any(bad):
            i = np.argwhere(bad)[0]
            raise AssertionError(f"{int(bad.sum())} outputs exceed the accumulation bound; first "
                                 f"{tuple(int(v) for v in i)}: err {err[tuple(i)]:.3e} > "
                                 f"{t_allow[tuple(i)]:.3e}")
    print(msg)
    return float(err.max())
