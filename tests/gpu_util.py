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


def assert_gemm_close(d_gpu: np.ndarray, d_orc: np.ndarray, tol: float, bf16: bool = False):
    d_gpu = d_gpu.astype(np.float64)
    err = np.abs(d_gpu - d_orc)
    allow = tol + (bf16_half_ulp(d_orc) if bf16 else 0.0)
    worst = float((err - allow).max())
    assert np.all(err <= allow), f"max|err| {err.max():.3e} exceeds the bound by {worst:.3e} (tol {tol:.3e})"
    return float(err.max())
