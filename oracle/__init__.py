"""CPU oracle for FP4 block quantization and the block-scaled FP4 GEMM.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``fp4_quantization_block_b200``) never imports it
and never falls back to it.

The arithmetic lives in ``fa4_oracle.c`` (plain C, one element at a time,
binary32 steps in the order the pages give, binary64 GEMM accumulation); this
module only marshals numpy arrays through ctypes.  ``gemm_sampled`` uses a
numpy binary64 matmul as a library step over the oracle's own dequantized
blocks.

Parity status per function (pins in ``tests/test_oracle_*.py``):
  e2m1_decode, e2m1_rne, e2m1_sr, e4m3_rne/decode, mx_exponent, nv scales,
  hadamard32, sf_offset, quantize, gemm: pinned.
  sr_bits (Philox4x32-7 stream, sr_rounds()): pinned by structure (one-round closed form,
  key-schedule and counter properties) and statistics only; the published
  known-answer vectors are not available, so the exact bit stream is
  "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

MXFP4, NVFP4_GLOBAL, NVFP4_CTA, MXFP4_NOCLIP = 0, 1, 2, 3
RNE, SR = 0, 1
ROWWISE, COLWISE = 0, 1
BLOCK = {MXFP4: 32, NVFP4_GLOBAL: 16, NVFP4_CTA: 16, MXFP4_NOCLIP: 32}

_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    global _lib
    if path is not None:
        return _setup(ctypes.CDLL(path))
    if _lib is None:
        _lib = _setup(ctypes.CDLL(_build.build()))
    return _lib


class using:
    """Context manager: route every function of this module through another
    build of the oracle (the planted-mistake tests use it)."""

    def __init__(self, path: str):
        self._new = _setup(ctypes.CDLL(path))

    def __enter__(self):
        global _lib
        load()
        self._old, _lib = _lib, self._new
        return self._new

    def __exit__(self, *exc):
        global _lib
        _lib = self._old
        return False


def _setup(lib: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    i64, u64, u32, f32, f64, ci = (ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32,
                                   ctypes.c_float, ctypes.c_double, ctypes.c_int)
    sig = {
        "orc_e2m1_decode": (f64, [ci]),
        "orc_e2m1_rne": (ci, [f32]),
        "orc_e2m1_sr": (ci, [f32, u32]),
        "orc_e4m3_decode": (f64, [ci]),
        "orc_e4m3_rne": (ci, [f32]),
        "orc_mx_exponent": (ci, [f32]),
        "orc_mx_exponent_noclip": (ci, [f32]),
        "orc_nv_encode_scale": (f32, [f32]),
        "orc_nv_decode_scale": (f32, [f32]),
        "orc_nv_block_scale": (ci, [f32, f32, P]),
        "orc_philox4x32": (None, [P, P, ci, P]),
        "orc_sr_bits": (u32, [u64, u64]),
        "orc_sr_rounds": (ci, []),
        "orc_sf_offset": (i64, [i64, i64, i64]),
        "orc_sf_bytes": (i64, [i64, i64]),
        "orc_hadamard32": (None, [P, u32, P]),
        "orc_quantize": (ci, [P, i64, i64, i64, ci, ci, ci, u64, ci, u32, P, P, P, i64, i64]),
        "orc_dequantize_blocks": (ci, [P, P, i64, i64, ci, P, i64, P]),
        "orc_gemm": (ci, [P, P, P, P, P, P, i64, i64, i64, ci, f64, P, i64, P, i64, P]),
        "orc_e2m1_rne_batch": (None, [P, i64, P]),
        "orc_e2m1_sr_batch": (None, [P, P, i64, P]),
        "orc_e4m3_rne_batch": (None, [P, i64, P]),
        "orc_sr_bits_batch": (None, [u64, P, i64, P]),
        "orc_exp_f32": (f32, [f32]),
        "orc_silu_f32": (f32, [f32]),
        "orc_exp_f32_batch": (None, [P, i64, P]),
        "orc_swiglu_bf16": (None, [P, i64, i64, i64, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- scalars ---

def e2m1_decode(code: int) -> float:
    return load().orc_e2m1_decode(int(code))


def e2m1_rne(y) -> np.ndarray:
    y = np.ascontiguousarray(np.asarray(y, dtype=np.float32).ravel())
    out = np.empty(y.size, dtype=np.uint8)
    load().orc_e2m1_rne_batch(_ptr(y), y.size, _ptr(out))
    return out


def e2m1_sr(y, u16) -> np.ndarray:
    y = np.ascontiguousarray(np.asarray(y, dtype=np.float32).ravel())
    u = np.ascontiguousarray(np.broadcast_to(np.asarray(u16, dtype=np.uint32), y.shape))
    out = np.empty(y.size, dtype=np.uint8)
    load().orc_e2m1_sr_batch(_ptr(y), _ptr(u), y.size, _ptr(out))
    return out


def e4m3_decode(code: int) -> float:
    return load().orc_e4m3_decode(int(code))


def e4m3_rne(v) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32).ravel())
    out = np.empty(v.size, dtype=np.uint8)
    load().orc_e4m3_rne_batch(_ptr(v), v.size, _ptr(out))
    return out


def mx_exponent(amax: float) -> int:
    return load().orc_mx_exponent(float(amax))


def mx_exponent_noclip(amax: float) -> int:
    return load().orc_mx_exponent_noclip(float(amax))


def nv_encode_scale(amax_t: float) -> float:
    return load().orc_nv_encode_scale(float(amax_t))


def nv_decode_scale(s_enc: float) -> float:
    return load().orc_nv_decode_scale(float(s_enc))


def nv_block_scale(amax_b: float, s_enc: float) -> tuple[int, float]:
    mult = ctypes.c_float(0.0)
    code = load().orc_nv_block_scale(float(amax_b), float(s_enc), ctypes.byref(mult))
    return code, mult.value


def philox4x32(ctr, key, rounds: int = 10) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.empty(4, dtype=np.uint32)
    load().orc_philox4x32(_ptr(c), _ptr(k), int(rounds), _ptr(out))
    return out


def sr_rounds() -> int:
    """Rounds of the Philox block behind the stochastic-rounding bits."""
    return int(load().orc_sr_rounds())


def sr_bits(seed: int, idx) -> np.ndarray:
    i = np.ascontiguousarray(np.asarray(idx, dtype=np.uint64).ravel())
    out = np.empty(i.size, dtype=np.uint32)
    load().orc_sr_bits_batch(int(seed), _ptr(i), i.size, _ptr(out))
    return out


def exp_f32(x) -> np.ndarray:
    """The oracle's binary32 exp (the SwiGLU producer's step-by-step definition)."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32).ravel())
    out = np.empty_like(a)
    load().orc_exp_f32_batch(_ptr(a), a.size, _ptr(out))
    return out


def silu_f32(g: float) -> float:
    return float(load().orc_silu_f32(float(g)))


def swiglu_bf16(z) -> np.ndarray:
    """h[T, F] = bf16(silu(gate) * up) as bf16 bits (uint16), from z[T, 2F]
    (torch bf16 or uint16 bf16 bits): gate = z[:, :F], up = z[:, F:]."""
    bits = _bf16_bits(z)
    T, F2 = bits.shape
    assert F2 % 2 == 0
    h = np.empty((T, F2 // 2), dtype=np.uint16)
    load().orc_swiglu_bf16(_ptr(bits), T, F2 // 2, F2, _ptr(h))
    return h


def sf_offset(r: int, kb: int, kb_total: int) -> int:
    return load().orc_sf_offset(int(r), int(kb), int(kb_total))


def sf_bytes(rows: int, kb_total: int) -> int:
    return load().orc_sf_bytes(int(rows), int(kb_total))


def hadamard32(x, sign_mask: int) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32).ravel())
    assert x.size == 32
    y = np.empty(32, dtype=np.float32)
    load().orc_hadamard32(_ptr(x), int(sign_mask) & 0xFFFFFFFF, _ptr(y))
    return y


# ------------------------------------------------------------ quantization ---

@dataclass
class QTensor:
    """A quantized operand Q[R, K]: payload [R, K/2] (K-major, low nibble =
    even element), swizzled block scales, FP32 second-level decode scales."""
    payload: np.ndarray
    scales: np.ndarray
    ts: np.ndarray
    R: int
    K: int
    fmt: int


def _bf16_bits(x) -> np.ndarray:
    """Accept a torch bf16 tensor or a numpy uint16 array of bf16 bits."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16
            return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(x)
    assert a.dtype == np.uint16
    return np.ascontiguousarray(a)


def ts_count(R: int, K: int, fmt: int) -> int:
    if fmt == NVFP4_GLOBAL:
        return 1
    if fmt == NVFP4_CTA:
        return -(-R // 128) * -(-K // 128)
    return 0


def quantize(x, fmt: int, rnd: int = RNE, orient: int = ROWWISE, seed: int = 0,
             hadamard_mask: int | None = None, row_range: tuple[int, int] | None = None) -> QTensor:
    """Quantize bf16 x.  ``row_range=(r0, r1)`` produces only rows r0..r1-1 of the
    quantized operand (the rest stay zero); second-level scales always cover
    the whole operand."""
    bits = _bf16_bits(x)
    rows, cols = bits.shape
    R, K = (rows, cols) if orient == ROWWISE else (cols, rows)
    bs = BLOCK[fmt]
    payload = np.zeros((R, K // 2), dtype=np.uint8)
    scales = np.zeros(sf_bytes(R, K // bs), dtype=np.uint8)
    ts = np.zeros(max(1, ts_count(R, K, fmt)), dtype=np.float32)
    rc = load().orc_quantize(_ptr(bits), rows, cols, cols, fmt, rnd, orient, int(seed),
                             0 if hadamard_mask is None else 1,
                             0 if hadamard_mask is None else int(hadamard_mask) & 0xFFFFFFFF,
                             _ptr(payload), _ptr(scales), _ptr(ts),
                             0 if row_range is None else int(row_range[0]),
                             0 if row_range is None else int(row_range[1]))
    if rc != 0:
        raise ValueError(f"oracle quantize rejected the arguments (rc={rc})")
    if fmt in (MXFP4, MXFP4_NOCLIP):
        ts = np.zeros(0, dtype=np.float32)
    return QTensor(payload, scales, ts, R, K, fmt)


def dequantize_blocks(q: QTensor, rows=None) -> np.ndarray:
    """e2m1 * block scale in binary64, without the second-level scale."""
    idx = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = q.R if idx is None else idx.size
    out = np.empty((n, q.K), dtype=np.float64)
    rc = load().orc_dequantize_blocks(_ptr(q.payload), _ptr(q.scales), q.R, q.K, q.fmt,
                                      _ptr(idx), n, _ptr(out))
    if rc != 0:
        raise ValueError("bad row index")
    return out


def dequantize(q: QTensor, rows=None) -> np.ndarray:
    """Full dequantized values (block scale and second-level scale) in binary64."""
    d = dequantize_blocks(q, rows)
    r = np.arange(q.R) if rows is None else np.asarray(rows, dtype=np.int64)
    if q.fmt == NVFP4_GLOBAL:
        d *= float(q.ts[0])
    elif q.fmt == NVFP4_CTA:
        nk = -(-q.K // 128)
        t = q.ts.reshape(-(-q.R // 128), nk).astype(np.float64)
        d *= np.repeat(t[r // 128], 128, axis=1)[:, :q.K]
    return d


def gemm(A: QTensor, B: QTensor, alpha: float = 1.0, m_idx=None, n_idx=None) -> np.ndarray:
    """D = alpha * A B^T through the C oracle (plain loops; small sizes)."""
    assert A.K == B.K and A.fmt == B.fmt
    mi = None if m_idx is None else np.ascontiguousarray(np.asarray(m_idx, dtype=np.int64))
    ni = None if n_idx is None else np.ascontiguousarray(np.asarray(n_idx, dtype=np.int64))
    nm = A.R if mi is None else mi.size
    nn = B.R if ni is None else ni.size
    out = np.empty((nm, nn), dtype=np.float64)
    tsa = A.ts if A.ts.size else np.ones(1, np.float32)
    tsb = B.ts if B.ts.size else np.ones(1, np.float32)
    rc = load().orc_gemm(_ptr(A.payload), _ptr(A.scales), _ptr(tsa), _ptr(B.payload),
                         _ptr(B.scales), _ptr(tsb), A.R, B.R, A.K, A.fmt, float(alpha),
                         _ptr(mi), nm, _ptr(ni), nn, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle gemm failed (rc={rc})")
    return out


def gemm_sampled(A: QTensor, B: QTensor, alpha: float = 1.0, m_idx=None, n_idx=None) -> np.ndarray:
    """Same result as ``gemm`` for large shapes: the oracle's binary64 block
    values, summed by a numpy binary64 matmul (the block products have at most
    12 significant bits, so every partial sum is exact whatever the order).
    Second-level scales multiply the exact per-128-K-chunk sums."""
    assert A.K == B.K and A.fmt == B.fmt
    a = dequantize_blocks(A, m_idx)
    b = dequantize_blocks(B, n_idx)
    mi = np.arange(A.R) if m_idx is None else np.asarray(m_idx, dtype=np.int64)
    ni = np.arange(B.R) if n_idx is None else np.asarray(n_idx, dtype=np.int64)
    if A.fmt == NVFP4_CTA:
        nk = -(-A.K // 128)  # the last chunk ends at K
        ta = A.ts.reshape(-(-A.R // 128), nk).astype(np.float64)[mi // 128]  # [nm, nk]
        tb = B.ts.reshape(-(-B.R // 128), nk).astype(np.float64)[ni // 128]  # [nn, nk]
        d = np.zeros((a.shape[0], b.shape[0]), dtype=np.float64)
        for kc in range(nk):
            s = a[:, kc * 128:(kc + 1) * 128] @ b[:, kc * 128:(kc + 1) * 128].T
            d += (ta[:, kc:kc + 1] * tb[:, kc][None, :]) * s
    else:
        d = a @ b.T
        if A.fmt == NVFP4_GLOBAL:
            d = d * (float(A.ts[0]) * float(B.ts[0]))
    return float(alpha) * d


def gemm_tolerance(A: QTensor, B: QTensor, alpha: float = 1.0) -> float:
    """Allowed max |D_gpu - D_oracle| for fp32 output:
    1e-3 * max|A_hat| * max|B_hat| * sqrt(K) with the dequantized operands
    including second-level scales and alpha."""
    amax = float(np.abs(dequantize(A)).max()) if A.R * A.K <= (1 << 26) else _sampled_absmax(A)
    bmax = float(np.abs(dequantize(B)).max()) if B.R * B.K <= (1 << 26) else _sampled_absmax(B)
    return 1e-3 * abs(alpha) * amax * bmax * float(np.sqrt(A.K))


def _sampled_absmax(q: QTensor) -> float:
    m = 0.0
    for r0 in range(0, q.R, 1024):
        rows = np.arange(r0, min(q.R, r0 + 1024))
        m = max(m, float(np.abs(dequantize(q, rows)).max()))
    return m
