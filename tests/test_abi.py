"""Host-only checks of the C ABI: the library loads, exports every function
include/fa4.h declares, and rejects bad arguments before launching anything.
No call here reaches a kernel launch, so no GPU is needed."""
import ctypes
import os
import re

import pytest

import fp4_quantization_block_b200 as fa
import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "fa4.h")).read()
    return sorted(set(re.findall(r"^FA4_API[^(]*?\b(fa4_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fa4_quantize", "fa4_hadamard32_quantize", "fa4_gemm_blockscaled",
                     "fa4_linear_fwd", "fa4_linear_dgrad", "fa4_linear_wgrad"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fa.library_path)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings():
    L = fa.lib()
    assert L.fa4_version() >= 100
    for s in range(8):
        assert L.fa4_status_string(s)
    assert L.fa4_status_string(99) == b"unknown status"


@pytest.mark.parametrize("fmt", [fa.MXFP4, fa.NVFP4_GLOBAL, fa.NVFP4_CTA, fa.MXFP4_NOCLIP])
@pytest.mark.parametrize("orient", [fa.ROWWISE, fa.COLWISE])
def test_quant_sizes_match_the_layout(fmt, orient):
    rows, cols = 384, 640
    pb, sb, tc, ws = fa.quant_sizes(rows, cols, fmt, orient)
    R, K = (rows, cols) if orient == fa.ROWWISE else (cols, rows)
    assert pb == R * K // 2
    assert sb == O.sf_bytes(R, K // fa.BLOCK[fmt])
    assert tc == O.ts_count(R, K, fmt)
    assert ws >= fa.WS_HEADER_BYTES


@pytest.mark.parametrize("fmt", [fa.MXFP4, fa.NVFP4_GLOBAL, fa.NVFP4_CTA, fa.MXFP4_NOCLIP])
@pytest.mark.parametrize("rows,cols,orient", [(200, 352, fa.ROWWISE), (352, 200, fa.COLWISE),
                                              (1, 32, fa.ROWWISE), (32, 8, fa.COLWISE)])
def test_quant_sizes_of_ragged_operands(fmt, rows, cols, orient):
    """Rows of Q not a multiple of 128 and K not a multiple of 128: scale
    atoms padded as the oracle pads them."""
    pb, sb, tc, _ = fa.quant_sizes(rows, cols, fmt, orient)
    R, K = (rows, cols) if orient == fa.ROWWISE else (cols, rows)
    assert pb == R * K // 2
    assert sb == O.sf_bytes(R, K // fa.BLOCK[fmt])
    assert tc == O.ts_count(R, K, fmt)


def _qt(p=0x10000, s=0x20000, t=0x30000):
    return fa._QT(p, s, t)


DEV = 0x7F0000000000  # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("case,expect", [
    (dict(x=None), 1),
    (dict(rows=0), 2),
    (dict(cols=100), 2),        # x rows are read in 16-byte pieces
    (dict(cols=200), 2),        # K (= cols, row-wise) a multiple of 32
    (dict(rows=200, orient=1), 2),  # K (= rows, column-wise) a multiple of 32
    (dict(ld=120), 2),
    (dict(ld=132), 2),
    (dict(x=DEV + 8), 3),
    (dict(fmt=7), 1),
    (dict(fmt=4), 1),
    (dict(rnd=5), 1),
    (dict(orient=3), 1),
    (dict(ws=None), 5),
    (dict(ws_bytes=16), 5),
    (dict(out=fa._QT(0, 0x20000, 0x30000)), 1),
    (dict(out=fa._QT(0x10008, 0x20000, 0x30000)), 3),
    (dict(fmt=fa.NVFP4_GLOBAL, out=fa._QT(0x10000, 0x20000, 0)), 1),
    (dict(fmt=fa.NVFP4_GLOBAL, ws_bytes=256), 5),
])
def test_quantize_rejects_bad_arguments(case, expect):
    a = dict(x=DEV, rows=256, cols=512, ld=512, fmt=fa.MXFP4, rnd=fa.RNE, orient=fa.ROWWISE,
             out=_qt(), ws=DEV + 4096, ws_bytes=1 << 20)
    a.update(case)
    st = fa.lib().fa4_quantize(a["x"], a["rows"], a["cols"], a["ld"], a["fmt"], a["rnd"],
                               a["orient"], 0, a["out"], a["ws"], a["ws_bytes"], None)
    assert st == expect


def test_hadamard_quantize_rejects_bad_arguments():
    L = fa.lib()
    assert L.fa4_hadamard32_quantize(None, 256, 256, 256, 1, 0, 0, _qt(), DEV, 4096, None) == 1
    assert L.fa4_hadamard32_quantize(DEV, 250, 256, 256, 1, 0, 0, _qt(), DEV, 4096, None) == 2
    assert L.fa4_hadamard32_quantize(DEV, 256, 256, 256, 1, 9, 0, _qt(), DEV, 4096, None) == 1
    assert L.fa4_hadamard32_quantize(DEV, 256, 256, 256, 1, 0, 0, _qt(), DEV, 8, None) == 5


@pytest.mark.parametrize("case,expect", [
    (dict(M=0), 2),
    (dict(K=48), 2),           # K must be a multiple of 32
    (dict(ldd=100), 2),
    (dict(D=None), 1),
    (dict(D=DEV + 4), 3),
    (dict(fmt=9), 1),
    (dict(od=3), 1),
    (dict(ws=None), 5),
    (dict(ws_bytes=100), 5),
    (dict(A=fa._QT(0, 0x20000, 0)), 1),
    (dict(fmt=fa.NVFP4_CTA, B=fa._QT(0x10000, 0x20000, 0)), 1),
])
def test_gemm_rejects_bad_arguments(case, expect):
    a = dict(A=_qt(), B=_qt(), M=256, N=256, K=512, fmt=fa.MXFP4, D=DEV, ldd=256, od=1,
             ws=DEV + 65536, ws_bytes=4096)
    a.update(case)
    st = fa.lib().fa4_gemm_blockscaled(a["A"], a["B"], a["M"], a["N"], a["K"], a["fmt"], 1.0,
                                       a["D"], a["ldd"], a["od"], a["ws"], a["ws_bytes"], None)
    assert st == expect


def test_linear_workspace_sizes_and_checks():
    L = fa.lib()
    n = ctypes.c_size_t()
    assert L.fa4_linear_ws_bytes(0, 8192, 4096, 6144, fa.NVFP4_GLOBAL, ctypes.byref(n)) == 0
    assert n.value >= 8192 * 4096 // 2 + 8192 * 4096 // 16
    assert L.fa4_linear_ws_bytes(2, 8192, 4096, 6144, fa.MXFP4, ctypes.byref(n)) == 0
    assert n.value >= (4096 + 6144) * 8192 // 2
    assert L.fa4_linear_ws_bytes(5, 128, 128, 128, 0, ctypes.byref(n)) == 1
    assert L.fa4_linear_ws_bytes(0, 100, 128, 128, 0, ctypes.byref(n)) == 2
    assert L.fa4_linear_fwd(DEV, _qt(), 256, 256, 256, fa.MXFP4, DEV, DEV, 64, None) == 5
    assert L.fa4_linear_dgrad(DEV, _qt(), 256, 256, 256, fa.MXFP4, 4, 0, DEV, DEV, 1 << 20, None) == 1
    assert L.fa4_linear_wgrad(DEV, None, 256, 256, 256, 1, 0, 0, DEV, 1, DEV, 1 << 24, None) == 1


def test_debug_entry_points_reject_bad_arguments():
    L = fa.lib()
    assert L.fa4_debug_convert(None, None, 10, DEV, None, None, None) == 1
    assert L.fa4_debug_convert(DEV, None, 10, DEV, DEV, None, None) == 1
    assert L.fa4_debug_sr_bits(0, None, 10, DEV, None) == 1
    assert L.fa4_debug_nv_block_scale(None, 1.0, 10, DEV, DEV, None) == 1
    assert L.fa4_debug_nv_block_scale(DEV, 1.0, -1, DEV, DEV, None) == 1
    assert L.fa4_debug_silu(None, 10, DEV, None) == 1
    assert L.fa4_debug_silu(DEV, -1, DEV, None) == 1
    assert L.fa4_debug_gemm_timeout(_qt(), _qt(), 256, 256, 512, 0, DEV, 256, 0, 0, DEV, 4096,
                                    None) == 1
    assert L.fa4_check_device_status(None, None) == 5
    assert L.fa4_workspace_init(None, 0, None) == 5


def test_product_package_does_not_import_the_oracle():
    import ast
    pkg = os.path.join(ROOT, "fp4_quantization_block_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            path = os.path.join(dirpath, f)
            if f.endswith(".py"):
                tree = ast.parse(open(path).read())
                for node in ast.walk(tree):
                    if isinstance(node, ast.Import):
                        assert all(not a.name.startswith("oracle") for a in node.names), path
                    if isinstance(node, ast.ImportFrom):
                        assert not (node.module or "").startswith("oracle"), path
            if f.endswith((".cu", ".cuh", ".h", ".cpp")):
                assert "fa4_oracle" not in open(path).read(), path
                assert "orc_" not in open(path).read(), path


def test_noalloc_quantize_rejects_bad_arguments():
    L = fa.lib()
    q = _qt()
    assert L.fa4_quantize_nvfp4_global_noalloc(None, 256, 256, 256, 0, 0, 0, q, None) == 1
    assert L.fa4_quantize_nvfp4_global_noalloc(DEV, 256, 250, 256, 0, 0, 0, q, None) == 2
    assert L.fa4_quantize_nvfp4_global_noalloc(DEV, 240, 256, 256, 0, 1, 0, q, None) == 2
    assert L.fa4_quantize_nvfp4_global_noalloc(DEV, 256, 256, 200, 0, 0, 0, q, None) == 2
    assert L.fa4_quantize_nvfp4_global_noalloc(DEV + 4, 256, 256, 256, 0, 0, 0, q, None) == 3
    assert L.fa4_quantize_nvfp4_global_noalloc(DEV, 256, 256, 256, 3, 0, 0, q, None) == 1
    assert L.fa4_quantize_nvfp4_global_noalloc(DEV, 256, 256, 256, 0, 0, 0,
                                               fa._QT(0x10000, 0x20000, 0), None) == 1


def test_dual_quantize_rejects_bad_arguments():
    L = fa.lib()
    q = _qt()
    args = lambda **k: dict(dict(x=DEV, rows=256, cols=256, ld=256, rf=fa.MXFP4, rr=0, cr=0,
                                 row=q, col=q, ws=DEV + 4096, wsb=1 << 20), **k)

    def call(a):
        return L.fa4_quantize_dual(a["x"], a["rows"], a["cols"], a["ld"], a["rf"], a["rr"], 0,
                                   a["row"], 1, 0x1234, a["cr"], 0, a["col"], a["ws"], a["wsb"],
                                   None)
    assert call(args(x=None)) == 1
    assert call(args(rows=200)) == 2
    assert call(args(ld=136)) == 2
    assert call(args(x=DEV + 2)) == 3
    assert call(args(rf=5)) == 1
    assert call(args(rr=2)) == 1
    assert call(args(cr=7)) == 1
    assert call(args(col=fa._QT(0, 0x20000, 0))) == 1
    assert call(args(row=fa._QT(0x10000, 0x20008, 0))) == 3
    assert call(args(rf=fa.NVFP4_GLOBAL, row=fa._QT(0x10000, 0x20000, 0))) == 1
    assert call(args(rf=fa.NVFP4_GLOBAL, wsb=256)) == 5
    assert call(args(ws=None)) == 5


def test_training_linear_rejects_bad_arguments():
    L = fa.lib()
    q = _qt()
    n = ctypes.c_size_t()
    assert L.fa4_linear_ws_bytes(3, 256, 256, 384, fa.MXFP4, ctypes.byref(n)) == 0
    assert n.value >= 256 * 256 // 2
    assert L.fa4_linear_ws_bytes(4, 256, 256, 384, fa.MXFP4, ctypes.byref(n)) == 0
    assert n.value >= 2 * 256 * 384 // 2
    assert L.fa4_linear_fwd_save(None, q, 256, 256, 384, 0, 1, DEV, q, DEV, 1 << 24, None) == 1
    assert L.fa4_linear_fwd_save(DEV, q, 256, 256, 384, 0, 1, DEV, fa._QT(0, 0, 0), DEV, 1 << 24,
                                 None) == 1
    assert L.fa4_linear_fwd_save(DEV, q, 256, 256, 384, 0, 1, DEV, q, DEV, 64, None) == 5
    assert L.fa4_linear_bwd(DEV, q, q, 256, 256, 384, 0, 3, 0, 1, DEV, DEV, 1, DEV, 1 << 24,
                            None) == 1
    assert L.fa4_linear_bwd(DEV, q, q, 250, 256, 384, 0, 1, 0, 1, DEV, DEV, 1, DEV, 1 << 24,
                            None) == 2
    assert L.fa4_linear_bwd(DEV, q, q, 256, 256, 384, 0, 1, 0, 1, DEV, DEV, 1, DEV, 64, None) == 5


def test_mxout_gemm_rejects_bad_arguments():
    L = fa.lib()
    q = _qt()
    f = L.fa4_gemm_blockscaled_mxout
    assert f(q, q, 256, 256, 512, fa.NVFP4_CTA, 1.0, DEV, 256, q, DEV, 4096, None) == 4
    assert f(q, q, 256, 256, 512, 7, 1.0, DEV, 256, q, DEV, 4096, None) == 1
    assert f(q, q, 256, 256, 48, fa.MXFP4, 1.0, DEV, 256, q, DEV, 4096, None) == 2
    assert f(q, q, 256, 240, 512, fa.MXFP4, 1.0, DEV, 256, q, DEV, 4096, None) == 2  # N % 32
    assert f(q, q, 256, 256, 512, fa.MXFP4, 1.0, DEV + 8, 256, q, DEV, 4096, None) == 3
    assert f(q, q, 256, 256, 512, fa.MXFP4, 1.0, DEV, 256, fa._QT(0, 0, 0), DEV, 4096, None) == 1
    assert f(q, q, 256, 256, 512, fa.MXFP4, 1.0, None, 0, fa._QT(0x10008, 0x20000, 0), DEV, 4096,
             None) == 3
    assert f(q, q, 256, 256, 512, fa.MXFP4, 1.0, None, 0, q, DEV, 8, None) == 5


def test_header_is_plain_c_and_links_from_c(tmp_path):
    """The boundary is a C ABI: include/fa4.h compiles as strict C99 and a C
    program links against libfa4.so and calls host-only entry points."""
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(
        '#include "fa4.h"\n#include <stdio.h>\n#include <string.h>\n'
        "int main(void) {\n"
        "  size_t pb = 0, sb = 0, tc = 0, ws = 0;\n"
        "  if (fa4_version() < 100) return 1;\n"
        "  if (strcmp(fa4_status_string(FA4_OK), \"ok\") != 0) return 2;\n"
        "  if (fa4_quant_sizes(256, 512, FA4_NVFP4_GLOBAL, FA4_ROWWISE, &pb, &sb, &tc, &ws) != FA4_OK)\n"
        "    return 3;\n"
        "  if (pb != 256 * 256 || sb != 256 * 32 || tc != 1) return 4;\n"
        "  if (fa4_quantize(NULL, 256, 512, 512, FA4_MXFP4, FA4_RNE, FA4_ROWWISE, 0,\n"
        "                   (fa4_qtensor){0, 0, 0}, NULL, 0, NULL) != FA4_ERR_INVALID_ARG) return 5;\n"
        "  puts(\"c-abi ok\");\n  return 0;\n}\n")
    exe = tmp_path / "abi"
    lib_dir = os.path.dirname(fa.library_path)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                         "-L", lib_dir, "-l:libfa4.so", f"-Wl,-rpath,{lib_dir}"],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and "c-abi ok" in run.stdout, (run.returncode, run.stderr)


def test_linear_bindings_validate_inputs_before_any_call():
    """The training-form and plain linear bindings reject a non-bf16 or
    host tensor before reaching the library (the C calls take no leading
    dimension, so a strided device input is copied, never passed as is)."""
    import torch
    x = torch.zeros(32, 32, dtype=torch.float32)
    q = fa.QTensor(torch.zeros(1, dtype=torch.uint8), torch.zeros(1, dtype=torch.uint8), None, 32, 32,
                   fa.MXFP4)
    for call in (lambda: fa.linear_fwd(x, q, fa.MXFP4),
                 lambda: fa.linear_dgrad(x, q, fa.MXFP4),
                 lambda: fa.linear_wgrad(x, x, 1),
                 lambda: fa.linear_fwd_save(x, q, fa.MXFP4, 1),
                 lambda: fa.linear_bwd(x, q, q, fa.MXFP4),
                 lambda: fa.linear_fwd(x.to(torch.bfloat16), q, fa.MXFP4)):
        with pytest.raises(ValueError):
            call()


def _qt_cpu(R, K, fmt):
    import torch
    _, sb, tc, _ = fa.quant_sizes(R, K, fmt)
    return fa.QTensor(torch.zeros(R, K // 2, dtype=torch.uint8), torch.zeros(sb, dtype=torch.uint8),
                      torch.zeros(tc, dtype=torch.float32) if tc else None, R, K, fmt)


def test_operand_validation_rejects_mismatched_operands_and_outputs():
    """The bindings check every operand and caller-supplied output against the
    call's sizes before reaching the library, whose C calls take no buffer
    sizes: a quantized operand with the wrong [R, K] or format, short or
    non-contiguous buffers, a missing second-level scale, an output of the
    wrong shape, dtype (fp16 is not bf16) or layout.  The checks take the
    device to compare with, so they run here on CPU tensors."""
    import torch
    dev = torch.device("cpu")
    good = _qt_cpu(256, 512, fa.NVFP4_GLOBAL)
    fa._check_qt(good, 256, 512, fa.NVFP4_GLOBAL, dev, "q")
    bad = [
        (good, 256, 256, fa.NVFP4_GLOBAL),                     # K differs (Wq.K != Cin)
        (good, 128, 512, fa.NVFP4_GLOBAL),                     # R differs
        (good, 256, 512, fa.MXFP4),                            # format differs
        (fa.QTensor(good.payload[:100], good.scales, good.ts, 256, 512, fa.NVFP4_GLOBAL),
         256, 512, fa.NVFP4_GLOBAL),                           # short payload
        (fa.QTensor(good.payload, good.scales[:10], good.ts, 256, 512, fa.NVFP4_GLOBAL),
         256, 512, fa.NVFP4_GLOBAL),                           # short scales
        (fa.QTensor(good.payload, good.scales, None, 256, 512, fa.NVFP4_GLOBAL),
         256, 512, fa.NVFP4_GLOBAL),                           # no tensor scale
        (fa.QTensor(good.payload.t(), good.scales, good.ts, 256, 512, fa.NVFP4_GLOBAL),
         256, 512, fa.NVFP4_GLOBAL),                           # strided payload
    ]
    for q, R, K, fmt in bad:
        with pytest.raises(ValueError):
            fa._check_qt(q, R, K, fmt, dev, "q")
    # MXFP4 and its no-clip variant share layout and scale type
    fa._check_qt(_qt_cpu(256, 512, fa.MXFP4_NOCLIP), 256, 512, fa.MXFP4, dev, "q")
    # CTA-local: one decode scale per 128x128 tile
    nvc = _qt_cpu(256, 512, fa.NVFP4_CTA)
    assert nvc.ts.numel() == 8
    with pytest.raises(ValueError):
        fa._check_qt(fa.QTensor(nvc.payload, nvc.scales, nvc.ts[:4], 256, 512, fa.NVFP4_CTA),
                     256, 512, fa.NVFP4_CTA, dev, "q")
    # outputs
    bf, f32 = (torch.bfloat16,), (torch.bfloat16, torch.float32)
    fa._check_out(torch.zeros(64, 32, dtype=torch.float32), (64, 32), f32, dev, "out")
    for t, shape, dt, rs in [
        (torch.zeros(64, 32, dtype=torch.float16), (64, 32), f32, False),   # fp16 is not bf16
        (torch.zeros(64, 32, dtype=torch.float32), (64, 32), bf, False),    # dtype not allowed here
        (torch.zeros(64, 16, dtype=torch.bfloat16), (64, 32), bf, False),   # shape
        (torch.zeros(32, 64, dtype=torch.bfloat16).t(), (64, 32), bf, False),  # not contiguous
        (torch.zeros(64, 36, dtype=torch.bfloat16)[:, :32], (64, 32), bf, True),  # row stride % 8
    ]:
        with pytest.raises(ValueError):
            fa._check_out(t, shape, dt, dev, "out", row_stride=rs)
    # a row stride that is a multiple of 8 is a valid GEMM output
    fa._check_out(torch.zeros(64, 40, dtype=torch.bfloat16)[:, :32], (64, 32), bf, dev, "out",
                  row_stride=True)


def test_swiglu_quantize_rejects_bad_arguments():
    L = fa.lib()
    q, none = _qt(), fa._QT(None, None, None)

    def call(z=DEV, T=256, F=256, ld=512, fmt=fa.MXFP4, rnd=0, col=0, crnd=0, out=q, cout=none):
        return L.fa4_swiglu_quantize(z, T, F, ld, fmt, rnd, 0, out, col, 1, 1, crnd, 0, cout, None)

    assert call(z=None) == 1
    assert call(fmt=9) == 1
    assert call(rnd=4) == 1
    assert call(fmt=fa.NVFP4_GLOBAL) == 4
    assert call(F=100) == 2          # F a multiple of 32
    assert call(T=0) == 2
    assert call(ld=400) == 2         # ld >= 2F
    assert call(ld=516) == 2         # ld a multiple of 8
    assert call(col=1, T=200) == 2   # column-wise: T a multiple of 32
    assert call(z=DEV + 8) == 3
    assert call(out=fa._QT(0, 0x20000, 0x30000)) == 1
    assert call(col=1, cout=fa._QT(0x10008, 0x20000, 0)) == 3
