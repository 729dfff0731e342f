"""FP4 quantization producers + block-scaled FP4 GEMM for B200 (sm_100a).

A thin ctypes binding of ``libfa4.so`` (C ABI in ``include/fa4.h``).  This
module only allocates tensors with PyTorch, picks the current CUDA stream and
marshals arguments; every step of the computation runs in the library's CUDA
kernels.  There is no CPU or PyTorch fallback: if the library is missing or a
call fails, an exception is raised.

Names follow the pages on format-aware fusion for FP4: the scale domains
MXFP4 (native mxfp), NVFP4_GLOBAL (global nvfp) and NVFP4_CTA (CTA-local nvfp)
of "Format-Aware Fusion: The Engineering Practice That Doubles FP4
Pretraining Throughput", section "The Design Philosophy of Format-Aware
Fusion"; row-gradient stochastic rounding and the fixed-sign 32-value
Hadamard of its section "Two Key Numerical Techniques".
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = [
    "MXFP4", "NVFP4_GLOBAL", "NVFP4_CTA", "MXFP4_NOCLIP", "RNE", "SR", "ROWWISE", "COLWISE",
    "QTensor", "FA4Error", "lib", "library_path", "quant_sizes", "empty_qtensor", "quantize",
    "swiglu_quantize",
    "hadamard32_quantize", "quantize_dual", "gemm", "gemm_mxout", "linear_ws_bytes", "linear_fwd", "linear_dgrad",
    "linear_wgrad", "linear_fwd_save", "linear_bwd", "workspace", "check_device_status",
]

MXFP4, NVFP4_GLOBAL, NVFP4_CTA, MXFP4_NOCLIP = 0, 1, 2, 3
RNE, SR = 0, 1
ROWWISE, COLWISE = 0, 1
OUT_BF16, OUT_FP32 = 0, 1
WS_HEADER_BYTES = 256
BLOCK = {MXFP4: 32, NVFP4_GLOBAL: 16, NVFP4_CTA: 16, MXFP4_NOCLIP: 32}

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libfa4.so")

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "misaligned pointer",
          4: "unsupported combination", 5: "workspace too small", 6: "CUDA error",
          7: "bounded device wait timed out"}


class FA4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} (status {status})")
        self.status = status


class _QT(ctypes.Structure):
    _fields_ = [("payload", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libfa4.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise ImportError(f"{library_path} is missing: build it with "
                              "`python -m fp4_quantization_block_b200.build`")
        _lib = _declare(ctypes.CDLL(library_path))
    return _lib


def _declare(L: ctypes.CDLL) -> ctypes.CDLL:
    P, i64, u64, u32, sz, ci, f32 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                     ctypes.c_uint32, ctypes.c_size_t, ctypes.c_int,
                                     ctypes.c_float)
    PSZ = ctypes.POINTER(ctypes.c_size_t)
    sig = {
        "fa4_quant_sizes": [i64, i64, ci, ci, PSZ, PSZ, PSZ, PSZ],
        "fa4_quantize": [P, i64, i64, i64, ci, ci, ci, u64, _QT, P, sz, P],
        "fa4_hadamard32_quantize": [P, i64, i64, i64, u32, ci, u64, _QT, P, sz, P],
        "fa4_quantize_dual": [P, i64, i64, i64, ci, ci, u64, _QT, ci, u32, ci, u64, _QT, P, sz, P],
        "fa4_gemm_blockscaled": [_QT, _QT, i64, i64, i64, ci, f32, P, i64, ci, P, sz, P],
        "fa4_gemm_blockscaled_mxout": [_QT, _QT, i64, i64, i64, ci, f32, P, i64, _QT, P, sz, P],
        "fa4_linear_ws_bytes": [ci, i64, i64, i64, ci, PSZ],
        "fa4_linear_fwd": [P, _QT, i64, i64, i64, ci, P, P, sz, P],
        "fa4_linear_dgrad": [P, _QT, i64, i64, i64, ci, ci, u64, P, P, sz, P],
        "fa4_linear_wgrad": [P, P, i64, i64, i64, u32, ci, u64, P, ci, P, sz, P],
        "fa4_linear_fwd_save": [P, _QT, i64, i64, i64, ci, u32, P, _QT, P, sz, P],
        "fa4_linear_bwd": [P, _QT, _QT, i64, i64, i64, ci, ci, u64, u32, P, P, ci, P, sz, P],
        "fa4_workspace_init": [P, sz, P],
        "fa4_check_device_status": [P, P],
        "fa4_debug_convert": [P, P, i64, P, P, P, P],
        "fa4_debug_sr_bits": [u64, P, i64, P, P],
        "fa4_debug_nv_block_scale": [P, f32, i64, P, P, P],
        "fa4_debug_silu": [P, i64, P, P],
        "fa4_debug_gemm_timeout": [_QT, _QT, i64, i64, i64, ci, P, i64, ci, u64, P, sz, P],
        "fa4_quantize_nvfp4_global_noalloc": [P, i64, i64, i64, ci, ci, u64, _QT, P],
        "fa4_swiglu_quantize": [P, i64, i64, i64, ci, ci, u64, _QT, ci, ci, u32, ci, u64, _QT, P],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ci
    L.fa4_status_string.argtypes = [ci]
    L.fa4_status_string.restype = ctypes.c_char_p
    L.fa4_version.argtypes = []
    L.fa4_version.restype = ci
    return L


def _check(status: int, what: str):
    if status != 0:
        raise FA4Error(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _on_tensor_device(fn):
    """Run a binding with the device of its first CUDA tensor argument (a
    QTensor's payload counts) current: the library picks the device's SM
    count and scratch from the current device, and launches on that
    device's current stream."""
    import functools

    @functools.wraps(fn)
    def wrapped(*args, **kwargs):
        for a in list(args) + list(kwargs.values()):
            t = a.payload if isinstance(a, QTensor) else a
            if isinstance(t, torch.Tensor) and t.is_cuda:
                with torch.cuda.device(t.device):
                    return fn(*args, **kwargs)
        return fn(*args, **kwargs)
    return wrapped


@dataclass
class QTensor:
    """Quantized operand Q[R, K]: ``payload`` uint8 [R, K/2] (K-major, element
    2j in the low nibble of byte j), ``scales`` uint8 in the 128x4 atom layout
    the block-scaled MMA reads (rows padded to a multiple of 128, blocks to a
    multiple of 4), ``ts`` float32 second-level decode scales (NVFP4) or None
    (MXFP4)."""
    payload: torch.Tensor
    scales: torch.Tensor
    ts: torch.Tensor | None
    R: int
    K: int
    fmt: int

    def c(self) -> _QT:
        return _QT(self.payload.data_ptr(), self.scales.data_ptr(),
                   None if self.ts is None else self.ts.data_ptr())


def quant_sizes(rows: int, cols: int, fmt: int, orient: int = ROWWISE) -> tuple[int, int, int, int]:
    a, b, c, d = (ctypes.c_size_t() for _ in range(4))
    _check(lib().fa4_quant_sizes(rows, cols, fmt, orient, ctypes.byref(a), ctypes.byref(b),
                                 ctypes.byref(c), ctypes.byref(d)), "fa4_quant_sizes")
    return a.value, b.value, c.value, d.value


def empty_qtensor(rows: int, cols: int, fmt: int, orient: int = ROWWISE, device="cuda") -> QTensor:
    pb, sb, tc, _ = quant_sizes(rows, cols, fmt, orient)
    R, K = (rows, cols) if orient == ROWWISE else (cols, rows)
    payload = torch.empty((R, K // 2), dtype=torch.uint8, device=device)
    scales = torch.empty(sb, dtype=torch.uint8, device=device)
    ts = torch.empty(tc, dtype=torch.float32, device=device) if tc else None
    assert payload.numel() == pb
    return QTensor(payload, scales, ts, R, K, fmt)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace (the status header must start at zero)."""
    return torch.zeros(max(int(nbytes), WS_HEADER_BYTES), dtype=torch.uint8, device=device)


def _ws(ws, need, device):
    if ws is None:
        ws = workspace(need, device)
    return ws


def _as_bf16_2d(x: torch.Tensor, name: str):
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError(f"{name} must be a 2-D bf16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError(f"{name} must have unit column stride")
    return x.stride(0)


def _rowmajor_bf16(x: torch.Tensor, name: str) -> torch.Tensor:
    """x as a contiguous row-major bf16 CUDA tensor (the linear calls take no
    leading dimension).  A strided input is copied; the caller keeps the
    returned tensor alive until the call has been enqueued."""
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise ValueError(f"{name} must be a 2-D bf16 CUDA tensor")
    return x if x.is_contiguous() else x.contiguous()


def _check_qt(q: QTensor, R: int, K: int, fmt: int, device, name: str):
    """A quantized operand of Q[R, K] in `fmt` whose buffers are large enough
    for the C calls (which take no buffer sizes) and live on `device`."""
    if not isinstance(q, QTensor):
        raise ValueError(f"{name} must be a QTensor")
    if (q.R, q.K) != (R, K):
        raise ValueError(f"{name} is [{q.R}, {q.K}], the call needs [{R}, {K}]")
    same = {fmt} | ({MXFP4, MXFP4_NOCLIP} if fmt in (MXFP4, MXFP4_NOCLIP) else set())
    if q.fmt not in same:
        raise ValueError(f"{name} has format {q.fmt}, the call needs {fmt}")
    _, sb, tc, _ = quant_sizes(R, K, fmt, ROWWISE)
    for t, n, what in ((q.payload, R * (K // 2), "payload"), (q.scales, sb, "scales")):
        if t.dtype != torch.uint8 or t.device != device or not t.is_contiguous() or t.numel() < n:
            raise ValueError(f"{name}.{what} must be a contiguous uint8 tensor of >= {n} bytes on {device}")
    if tc:
        t = q.ts
        if t is None or t.dtype != torch.float32 or t.device != device or not t.is_contiguous() \
                or t.numel() < tc:
            raise ValueError(f"{name}.ts must be a contiguous float32 tensor of >= {tc} values on {device}")


def _check_out(t: torch.Tensor, shape: tuple, dtypes: tuple, device, name: str, row_stride=False):
    """A caller-supplied output: `shape`, one of `dtypes`, on `device`,
    contiguous (or, with row_stride, unit column stride and a row stride the
    C call can take)."""
    if t.dtype not in dtypes:
        raise ValueError(f"{name} must have dtype {' or '.join(str(d) for d in dtypes)}, not {t.dtype}")
    if tuple(t.shape) != tuple(shape) or t.device != device:
        raise ValueError(f"{name} must be a {list(shape)} tensor on {device}, "
                         f"not {list(t.shape)} on {t.device}")
    if row_stride:
        if t.dim() != 2 or t.stride(1) != 1 or t.stride(0) < shape[1] or t.stride(0) % 8:
            raise ValueError(f"{name} needs unit column stride and a row stride >= {shape[1]}, "
                             "a multiple of 8")
    elif not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@_on_tensor_device
def quantize(x: torch.Tensor, fmt: int, rnd: int = RNE, orient: int = ROWWISE, seed: int = 0,
             out: QTensor | None = None, ws: torch.Tensor | None = None) -> QTensor:
    ld = _as_bf16_2d(x, "x")
    rows, cols = x.shape
    if out is not None:
        _check_qt(out, *((rows, cols) if orient == ROWWISE else (cols, rows)), fmt, x.device, "out")
    out = out or empty_qtensor(rows, cols, fmt, orient, x.device)
    need = quant_sizes(rows, cols, fmt, orient)[3]
    ws = _ws(ws, need, x.device)
    _check(lib().fa4_quantize(_ptr(x), rows, cols, ld, fmt, rnd, orient, seed, out.c(), _ptr(ws),
                              ws.numel(), _stream(x.device)), "fa4_quantize")
    return out


@_on_tensor_device
def quantize_nvfp4_global_noalloc(x: torch.Tensor, rnd: int = RNE, orient: int = ROWWISE,
                                  seed: int = 0, out: QTensor | None = None) -> QTensor:
    """NVFP4-global quantization without a workspace: the amax scratch lives
    in a fixed array inside the library (see include/fa4.h)."""
    ld = _as_bf16_2d(x, "x")
    rows, cols = x.shape
    if out is not None:
        _check_qt(out, *((rows, cols) if orient == ROWWISE else (cols, rows)), NVFP4_GLOBAL,
                  x.device, "out")
    out = out or empty_qtensor(rows, cols, NVFP4_GLOBAL, orient, x.device)
    _check(lib().fa4_quantize_nvfp4_global_noalloc(_ptr(x), rows, cols, ld, rnd, orient, seed,
                                                   out.c(), _stream(x.device)),
           "fa4_quantize_nvfp4_global_noalloc")
    return out


@_on_tensor_device
def hadamard32_quantize(x: torch.Tensor, sign_mask: int, rnd: int = RNE, seed: int = 0,
                        out: QTensor | None = None, ws: torch.Tensor | None = None) -> QTensor:
    ld = _as_bf16_2d(x, "x")
    rows, cols = x.shape
    if out is not None:
        _check_qt(out, cols, rows, MXFP4, x.device, "out")
    out = out or empty_qtensor(rows, cols, MXFP4, COLWISE, x.device)
    ws = _ws(ws, WS_HEADER_BYTES, x.device)
    _check(lib().fa4_hadamard32_quantize(_ptr(x), rows, cols, ld, sign_mask & 0xFFFFFFFF, rnd, seed,
                                         out.c(), _ptr(ws), ws.numel(), _stream(x.device)),
           "fa4_hadamard32_quantize")
    return out


@_on_tensor_device
def quantize_dual(x: torch.Tensor, row_fmt: int, row_rnd: int = RNE, row_seed: int = 0,
                  col_hadamard: bool = True, sign_mask: int = 0, col_rnd: int = RNE,
                  col_seed: int = 0, row_out: QTensor | None = None,
                  col_out: QTensor | None = None,
                  ws: torch.Tensor | None = None) -> tuple[QTensor, QTensor]:
    """One read of x: the row-wise operand (any format) and the column-wise
    MXFP4 operand (with the fixed-sign Hadamard when col_hadamard)."""
    ld = _as_bf16_2d(x, "x")
    rows, cols = x.shape
    if row_out is not None:
        _check_qt(row_out, rows, cols, row_fmt, x.device, "row_out")
    if col_out is not None:
        _check_qt(col_out, cols, rows, MXFP4, x.device, "col_out")
    row_out = row_out or empty_qtensor(rows, cols, row_fmt, ROWWISE, x.device)
    col_out = col_out or empty_qtensor(rows, cols, MXFP4, COLWISE, x.device)
    need = quant_sizes(rows, cols, row_fmt, ROWWISE)[3]
    ws = _ws(ws, need, x.device)
    _check(lib().fa4_quantize_dual(_ptr(x), rows, cols, ld, row_fmt, row_rnd, row_seed,
                                   row_out.c(), 1 if col_hadamard else 0, sign_mask & 0xFFFFFFFF,
                                   col_rnd, col_seed, col_out.c(), _ptr(ws), ws.numel(),
                                   _stream(x.device)), "fa4_quantize_dual")
    return row_out, col_out


@_on_tensor_device
def swiglu_quantize(z: torch.Tensor, row_fmt: int, row_rnd: int = RNE, row_seed: int = 0,
                    col: bool = False, col_hadamard: bool = True, sign_mask: int = 0,
                    col_rnd: int = RNE, col_seed: int = 0, row_out: QTensor | None = None,
                    col_out: QTensor | None = None) -> tuple[QTensor, QTensor | None]:
    """The down projection's input h = bf16(silu(gate) * up), gate and up the
    two halves of z[T, 2F], quantized row-wise (row_fmt MXFP4, MXFP4_NOCLIP
    or NVFP4_CTA) and, with col, column-wise MXFP4 (optionally through the
    fixed-sign Hadamard) in one kernel; h is never written."""
    ld = _as_bf16_2d(z, "z")
    T, F2 = z.shape
    if F2 % 2:
        raise ValueError("z must hold gate and up halves (an even number of columns)")
    F = F2 // 2
    if row_out is not None:
        _check_qt(row_out, T, F, row_fmt, z.device, "row_out")
    if col and col_out is not None:
        _check_qt(col_out, F, T, MXFP4, z.device, "col_out")
    row_out = row_out or empty_qtensor(T, F, row_fmt, ROWWISE, z.device)
    if col:
        col_out = col_out or empty_qtensor(T, F, MXFP4, COLWISE, z.device)
    cq = col_out.c() if col else _QT(None, None, None)
    _check(lib().fa4_swiglu_quantize(_ptr(z), T, F, ld, row_fmt, row_rnd, row_seed, row_out.c(),
                                     1 if col else 0, 1 if col_hadamard else 0,
                                     sign_mask & 0xFFFFFFFF, col_rnd, col_seed, cq,
                                     _stream(z.device)), "fa4_swiglu_quantize")
    return row_out, (col_out if col else None)


@_on_tensor_device
def gemm(A: QTensor, B: QTensor, alpha: float = 1.0, out_dtype=torch.float32,
         out: torch.Tensor | None = None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """D[M, N] = alpha * A B^T on the block-scaled FP4 tensor cores."""
    if A.K != B.K or A.fmt != B.fmt:
        raise ValueError("A and B must share K and format")
    dev = A.payload.device
    if out is None:
        # leading dimension a multiple of 8 elements (the ABI's row alignment)
        ldd = -(-B.R // 8) * 8
        out = torch.empty((A.R, ldd), dtype=out_dtype, device=dev)[:, :B.R]
    _check_qt(B, B.R, A.K, A.fmt, dev, "B")
    _check_qt(A, A.R, A.K, A.fmt, dev, "A")
    _check_out(out, (A.R, B.R), (torch.bfloat16, torch.float32), dev, "out", row_stride=True)
    od = OUT_FP32 if out.dtype == torch.float32 else OUT_BF16
    ws = _ws(ws, WS_HEADER_BYTES, dev)
    _check(lib().fa4_gemm_blockscaled(A.c(), B.c(), A.R, B.R, A.K, A.fmt, float(alpha), _ptr(out),
                                      out.stride(0), od, _ptr(ws), ws.numel(), _stream(dev)),
           "fa4_gemm_blockscaled")
    return out


def linear_ws_bytes(kind: int, T: int, Cin: int, Cout: int, fmt: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().fa4_linear_ws_bytes(kind, T, Cin, Cout, fmt, ctypes.byref(n)), "fa4_linear_ws_bytes")
    return n.value


@_on_tensor_device
def linear_fwd(X: torch.Tensor, Wq: QTensor, fmt: int, out: torch.Tensor | None = None,
               ws: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X W^T; Wq is W[Cout, Cin] quantized row-wise."""
    X = _rowmajor_bf16(X, "X")
    T, Cin = X.shape
    Cout = Wq.R
    _check_qt(Wq, Cout, Cin, fmt, X.device, "Wq")
    if out is not None:
        _check_out(out, (T, Cout), (torch.bfloat16,), X.device, "out")
    out = out if out is not None else torch.empty((T, Cout), dtype=torch.bfloat16, device=X.device)
    ws = _ws(ws, linear_ws_bytes(0, T, Cin, Cout, fmt), X.device)
    _check(lib().fa4_linear_fwd(_ptr(X), Wq.c(), T, Cin, Cout, fmt, _ptr(out), _ptr(ws),
                                ws.numel(), _stream(X.device)), "fa4_linear_fwd")
    return out


@_on_tensor_device
def linear_dgrad(dY: torch.Tensor, Wq_col: QTensor, fmt: int, rnd: int = SR, seed: int = 0,
                 out: torch.Tensor | None = None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """dX = dY W; Wq_col is W[Cout, Cin] quantized column-wise ([Cin, Cout])."""
    dY = _rowmajor_bf16(dY, "dY")
    T, Cout = dY.shape
    Cin = Wq_col.R
    _check_qt(Wq_col, Cin, Cout, fmt, dY.device, "Wq_col")
    if out is not None:
        _check_out(out, (T, Cin), (torch.bfloat16,), dY.device, "out")
    out = out if out is not None else torch.empty((T, Cin), dtype=torch.bfloat16, device=dY.device)
    ws = _ws(ws, linear_ws_bytes(1, T, Cin, Cout, fmt), dY.device)
    _check(lib().fa4_linear_dgrad(_ptr(dY), Wq_col.c(), T, Cin, Cout, fmt, rnd, seed,
                                  _ptr(out), _ptr(ws), ws.numel(), _stream(dY.device)),
           "fa4_linear_dgrad")
    return out


@_on_tensor_device
def linear_wgrad(dY: torch.Tensor, X: torch.Tensor, sign_mask: int, rnd: int = RNE, seed: int = 0,
                 out_dtype=torch.float32, out: torch.Tensor | None = None,
                 ws: torch.Tensor | None = None) -> torch.Tensor:
    """dW = dY^T X through column-wise fixed-sign Hadamard MXFP4 operands."""
    dY = _rowmajor_bf16(dY, "dY")
    X = _rowmajor_bf16(X, "X")
    T, Cout = dY.shape
    TX, Cin = X.shape
    if TX != T or X.device != dY.device:
        raise ValueError(f"X must have dY's {T} rows and device")
    if out is None:
        if out_dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")
        out = torch.empty((Cout, Cin), dtype=out_dtype, device=dY.device)
    _check_out(out, (Cout, Cin), (torch.bfloat16, torch.float32), dY.device, "out")
    od = OUT_FP32 if out.dtype == torch.float32 else OUT_BF16
    ws = _ws(ws, linear_ws_bytes(2, T, Cin, Cout, MXFP4), dY.device)
    _check(lib().fa4_linear_wgrad(_ptr(dY), _ptr(X), T, Cin, Cout,
                                  sign_mask & 0xFFFFFFFF, rnd, seed, _ptr(out), od, _ptr(ws),
                                  ws.numel(), _stream(dY.device)), "fa4_linear_wgrad")
    return out


@_on_tensor_device
def check_device_status(ws: torch.Tensor) -> int:
    """Synchronize and return (and clear) the workspace's device status."""
    return lib().fa4_check_device_status(_ptr(ws), _stream(ws.device))


# ------------------------------------------------------------ diagnostics ---

def debug_convert(y: torch.Tensor, u16: torch.Tensor | None = None, e4m3: bool = False):
    """Device E2M1 RNE / SR and E4M3 conversions of fp32 values (as the
    quantizers use them)."""
    n = y.numel()
    rne = torch.empty(n, dtype=torch.uint8, device=y.device)
    sr = torch.empty(n, dtype=torch.uint8, device=y.device) if u16 is not None else None
    e4 = torch.empty(n, dtype=torch.uint8, device=y.device) if e4m3 else None
    _check(lib().fa4_debug_convert(_ptr(y), _ptr(u16), n, _ptr(rne), _ptr(sr), _ptr(e4),
                                   _stream(y.device)), "fa4_debug_convert")
    return rne, sr, e4


def debug_nv_block_scale(amax: torch.Tensor, s_enc: float):
    """Device NVFP4 block scale of each amax (float32 CUDA tensor) under the
    encode scale s_enc, as the quantizers compute it: (E4M3 codes uint8,
    element multipliers float32)."""
    n = amax.numel()
    codes = torch.empty(n, dtype=torch.uint8, device=amax.device)
    mults = torch.empty(n, dtype=torch.float32, device=amax.device)
    _check(lib().fa4_debug_nv_block_scale(_ptr(amax), float(s_enc), n, _ptr(codes), _ptr(mults),
                                          _stream(amax.device)), "fa4_debug_nv_block_scale")
    return codes, mults


def debug_silu(g: torch.Tensor) -> torch.Tensor:
    """silu(g) in binary32 exactly as the SwiGLU producer computes it, for a
    contiguous bf16 CUDA tensor g (finite values); float32 result."""
    if g.dtype != torch.bfloat16 or not g.is_cuda or not g.is_contiguous():
        raise ValueError("g must be a contiguous bf16 CUDA tensor")
    out = torch.empty(g.shape, dtype=torch.float32, device=g.device)
    _check(lib().fa4_debug_silu(_ptr(g), g.numel(), _ptr(out), _stream(g.device)), "fa4_debug_silu")
    return out


def debug_sr_bits(seed: int, idx: torch.Tensor) -> torch.Tensor:
    bits = torch.empty(idx.numel(), dtype=torch.int32, device=idx.device)
    _check(lib().fa4_debug_sr_bits(seed, _ptr(idx), idx.numel(), _ptr(bits), _stream(idx.device)),
           "fa4_debug_sr_bits")
    return bits


def debug_gemm_timeout(A: QTensor, B: QTensor, skip_k_tile: int, timeout_ns: int,
                       ws: torch.Tensor) -> torch.Tensor:
    dev = A.payload.device
    out = torch.zeros((A.R, B.R), dtype=torch.float32, device=dev)
    _check(lib().fa4_debug_gemm_timeout(A.c(), B.c(), A.R, B.R, A.K, A.fmt, _ptr(out), out.stride(0),
                                        skip_k_tile, timeout_ns, _ptr(ws), ws.numel(), _stream(dev)),
           "fa4_debug_gemm_timeout")
    return out


@_on_tensor_device
def linear_fwd_save(X: torch.Tensor, Wq: QTensor, fmt: int, sign_mask: int,
                    out: torch.Tensor | None = None, xcol: QTensor | None = None,
                    ws: torch.Tensor | None = None) -> tuple[torch.Tensor, QTensor]:
    """Y = X W^T, plus X's column-wise MXFP4 Hadamard operand for the
    backward half (one read of X)."""
    X = _rowmajor_bf16(X, "X")
    T, Cin = X.shape
    Cout = Wq.R
    _check_qt(Wq, Cout, Cin, fmt, X.device, "Wq")
    if out is not None:
        _check_out(out, (T, Cout), (torch.bfloat16,), X.device, "out")
    if xcol is not None:
        _check_qt(xcol, Cin, T, MXFP4, X.device, "xcol")
    Y = out if out is not None else torch.empty(T, Cout, dtype=torch.bfloat16, device=X.device)
    xcol = xcol or empty_qtensor(T, Cin, MXFP4, COLWISE, X.device)
    ws = _ws(ws, linear_ws_bytes(3, T, Cin, Cout, fmt), X.device)
    _check(lib().fa4_linear_fwd_save(_ptr(X), Wq.c(), T, Cin, Cout, fmt, sign_mask & 0xFFFFFFFF,
                                     _ptr(Y), xcol.c(), _ptr(ws), ws.numel(), _stream(X.device)),
           "fa4_linear_fwd_save")
    return Y, xcol


@_on_tensor_device
def linear_bwd(dY: torch.Tensor, Wq_col: QTensor, xcol: QTensor, fmt: int, rnd: int = SR,
               seed: int = 0, sign_mask: int = 0, dw_dtype=torch.float32,
               dx: torch.Tensor | None = None, dw: torch.Tensor | None = None,
               ws: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """dX = dY W and dW = dY^T X from one read of dY (xcol from
    linear_fwd_save with the same sign_mask)."""
    dY = _rowmajor_bf16(dY, "dY")
    T, Cout = dY.shape
    Cin = Wq_col.R
    _check_qt(Wq_col, Cin, Cout, fmt, dY.device, "Wq_col")
    _check_qt(xcol, Cin, T, MXFP4, dY.device, "xcol")
    if dx is not None:
        _check_out(dx, (T, Cin), (torch.bfloat16,), dY.device, "dx")
    if dw is not None:
        _check_out(dw, (Cout, Cin), (torch.bfloat16, torch.float32), dY.device, "dw")
    elif dw_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("dw_dtype must be torch.bfloat16 or torch.float32")
    dX = dx if dx is not None else torch.empty(T, Cin, dtype=torch.bfloat16, device=dY.device)
    dW = dw if dw is not None else torch.empty(Cout, Cin, dtype=dw_dtype, device=dY.device)
    od = OUT_FP32 if dW.dtype == torch.float32 else OUT_BF16
    ws = _ws(ws, linear_ws_bytes(4, T, Cin, Cout, fmt), dY.device)
    _check(lib().fa4_linear_bwd(_ptr(dY), Wq_col.c(), xcol.c(), T, Cin, Cout, fmt, rnd, seed,
                                sign_mask & 0xFFFFFFFF, _ptr(dX), _ptr(dW), od, _ptr(ws),
                                ws.numel(), _stream(dY.device)), "fa4_linear_bwd")
    return dX, dW


@_on_tensor_device
def gemm_mxout(A: QTensor, B: QTensor, alpha: float = 1.0, store_d: bool = True,
               out: torch.Tensor | None = None, qout: QTensor | None = None,
               ws: torch.Tensor | None = None) -> tuple[torch.Tensor | None, QTensor]:
    """D = alpha * A B^T (bf16, unless store_d is False) and D's row-wise
    MXFP4 operand, quantized in the GEMM's epilogue."""
    if A.K != B.K or A.fmt != B.fmt:
        raise ValueError("A and B must share K and format")
    dev = A.payload.device
    _check_qt(A, A.R, A.K, A.fmt, dev, "A")
    _check_qt(B, B.R, A.K, A.fmt, dev, "B")
    if store_d and out is not None:
        _check_out(out, (A.R, B.R), (torch.bfloat16,), dev, "out", row_stride=True)
    if qout is not None:
        _check_qt(qout, A.R, B.R, MXFP4, dev, "qout")
    if store_d and out is None:
        out = torch.empty((A.R, B.R), dtype=torch.bfloat16, device=dev)
    qout = qout or empty_qtensor(A.R, B.R, MXFP4, ROWWISE, dev)
    ws = _ws(ws, WS_HEADER_BYTES, dev)
    d_ptr = _ptr(out) if store_d else None
    ldd = out.stride(0) if store_d else B.R
    _check(lib().fa4_gemm_blockscaled_mxout(A.c(), B.c(), A.R, B.R, A.K, A.fmt, float(alpha), d_ptr,
                                            ldd, qout.c(), _ptr(ws), ws.numel(), _stream(dev)),
           "fa4_gemm_blockscaled_mxout")
    return (out if store_d else None), qout
