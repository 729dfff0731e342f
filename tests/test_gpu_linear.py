"""Linear compositions through the C ABI against oracle compositions
(quantize + GEMM), and the bounded-wait timeout path."""
import numpy as np
import pytest
import torch

import fp4_quantization_block_b200 as fa
import oracle as O
import workloads
from gpu_util import FMT_IDS, FMTS, accumulation_bound, assert_gemm_close, need_gpu, to_gpu_qt

pytestmark = pytest.mark.gpu

SIGN_MASK = 0x2545F491


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
def test_linear_fwd(fmt):
    need_gpu()
    T, Cin, Cout = 512, 1024, 768
    x = workloads.act(T, Cin, seed=3)
    w = workloads.weight(Cout, Cin, seed=4)
    Wq = O.quantize(w, fmt)
    y = fa.linear_fwd(x.cuda(), to_gpu_qt(Wq), fmt)
    torch.cuda.synchronize()
    Xq = O.quantize(x, fmt)
    want = O.gemm_sampled(Xq, Wq)
    assert_gemm_close(y.float().cpu().numpy(), want, O.gemm_tolerance(Xq, Wq), bf16=True,
                      tight=accumulation_bound(Xq, Wq))


@pytest.mark.parametrize("fmt", FMTS, ids=[FMT_IDS[f] for f in FMTS])
@pytest.mark.parametrize("rnd", [fa.RNE, fa.SR], ids=["rne", "sr"])
def test_linear_dgrad(fmt, rnd):
    need_gpu()
    T, Cin, Cout = 512, 768, 1024
    dy = workloads.grad(T, Cout, seed=5)
    w = workloads.weight(Cout, Cin, seed=6)
    Wcol = O.quantize(w, fmt, orient=O.COLWISE)        # [Cin, Cout]
    dx = fa.linear_dgrad(dy.cuda(), to_gpu_qt(Wcol), fmt, rnd, seed=1)
    torch.cuda.synchronize()
    Gq = O.quantize(dy, fmt, rnd, O.ROWWISE, seed=1)
    want = O.gemm_sampled(Gq, Wcol)
    assert_gemm_close(dx.float().cpu().numpy(), want, O.gemm_tolerance(Gq, Wcol), bf16=True,
                      tight=accumulation_bound(Gq, Wcol))


@pytest.mark.parametrize("rnd", [fa.RNE, fa.SR], ids=["rne", "sr"])
def test_linear_wgrad(rnd):
    need_gpu()
    T, Cin, Cout = 1024, 512, 384
    dy = workloads.grad(T, Cout, seed=7)
    x = workloads.act(T, Cin, seed=8)
    dw = fa.linear_wgrad(dy.cuda(), x.cuda(), SIGN_MASK, rnd, seed=9)
    torch.cuda.synchronize()
    Gq = O.quantize(dy, O.MXFP4, rnd, O.COLWISE, seed=9, hadamard_mask=SIGN_MASK)
    Xq = O.quantize(x, O.MXFP4, rnd, O.COLWISE, seed=10, hadamard_mask=SIGN_MASK)
    want = O.gemm_sampled(Gq, Xq, 1.0 / 32)
    assert_gemm_close(dw.cpu().numpy(), want, O.gemm_tolerance(Gq, Xq, 1.0 / 32),
                      tight=accumulation_bound(Gq, Xq, 1.0 / 32))
    # the Hadamard preconditioning leaves dW = dY^T X (up to FP4 error)
    exact = dy.double().T.numpy() @ x.double().numpy()
    rel = np.linalg.norm(dw.cpu().numpy() - exact) / np.linalg.norm(exact)
    assert rel < (0.2 if rnd == fa.RNE else 0.3), rel  # SR adds zero-mean noise


@pytest.mark.parametrize("layer", list(workloads.LLAMA8B_LINEARS), ids=str)
def test_llama8b_backward_shapes_sampled(layer):
    """Full 8B-shaped dgrad and wgrad (8192 tokens), sampled rows of the output."""
    need_gpu()
    cin, cout = workloads.LLAMA8B_LINEARS[layer]
    T = workloads.LLAMA8B_TOKENS
    dy = workloads.grad(T, cout, seed=11)
    x = workloads.act(T, cin, seed=12)
    w = workloads.weight(cout, cin, seed=13)
    rng = np.random.default_rng(2)
    Wcol = O.quantize(w, O.MXFP4, orient=O.COLWISE)
    dx = fa.linear_dgrad(dy.cuda(), to_gpu_qt(Wcol), fa.MXFP4, fa.SR, seed=1)
    dw = fa.linear_wgrad(dy.cuda(), x.cuda(), SIGN_MASK, fa.RNE, seed=3)
    torch.cuda.synchronize()
    rows = np.sort(rng.choice(T, 32, replace=False))
    rb = sorted({int(r) // 128 for r in rows})
    Gq = O.quantize(dy, O.MXFP4, O.SR, O.ROWWISE, seed=1)
    want = O.gemm_sampled(Gq, Wcol, 1.0, rows, None)
    assert_gemm_close(dx.float().cpu().numpy()[rows], want, O.gemm_tolerance(Gq, Wcol), bf16=True,
                      tight=accumulation_bound(Gq, Wcol, 1.0, rows, None))
    del rb
    wrows = np.sort(rng.choice(cout, 32, replace=False))
    Gc = O.quantize(dy, O.MXFP4, O.RNE, O.COLWISE, seed=3, hadamard_mask=SIGN_MASK)
    Xc = O.quantize(x, O.MXFP4, O.RNE, O.COLWISE, seed=4, hadamard_mask=SIGN_MASK)
    want_w = O.gemm_sampled(Gc, Xc, 1.0 / 32, wrows, None)
    assert_gemm_close(dw.cpu().numpy()[wrows], want_w, O.gemm_tolerance(Gc, Xc, 1.0 / 32),
                      tight=accumulation_bound(Gc, Xc, 1.0 / 32, wrows, None))


def test_bounded_wait_times_out_and_context_survives():
    """The producer never loads one k-tile, so the MMA warp's wait runs out
    after 20 ms: the kernel sets the status word and returns; the host reads
    FA4_ERR_TIMEOUT and the next GEMM on the same context is correct."""
    need_gpu()
    x = workloads.tiny(0)
    A = to_gpu_qt(O.quantize(x[:, :256].contiguous(), O.MXFP4))
    B = to_gpu_qt(O.quantize(x[:128, 256:].contiguous(), O.MXFP4))
    ws = fa.workspace(4096)
    fa.debug_gemm_timeout(A, B, skip_k_tile=0, timeout_ns=20_000_000, ws=ws)
    assert fa.check_device_status(ws) == 7
    assert fa.check_device_status(ws) == 0  # read clears it
    d = fa.gemm(A, B, ws=ws)
    assert fa.check_device_status(ws) == 0
    want = O.gemm(O.quantize(x[:, :256].contiguous(), O.MXFP4), O.quantize(x[:128, 256:].contiguous(), O.MXFP4))
    assert np.allclose(d.cpu().numpy(), want, rtol=0, atol=1e-2)


def test_bounded_wait_times_out_in_the_two_sm_kernel():
    """Same check for the cluster (2-SM) GEMM path (M and N multiples of 256):
    both CTAs of the pair give up, release their tensor memory and return."""
    need_gpu()
    x = workloads.tiny(1)
    a = torch.cat([x[:, :256], x[:, 256:]], 0)[:256].contiguous()
    b = x[:, 256:].contiguous()
    A = to_gpu_qt(O.quantize(a, O.NVFP4_GLOBAL))
    B = to_gpu_qt(O.quantize(b, O.NVFP4_GLOBAL))
    ws = fa.workspace(4096)
    fa.debug_gemm_timeout(A, B, skip_k_tile=0, timeout_ns=20_000_000, ws=ws)
    assert fa.check_device_status(ws) == 7
    d = fa.gemm(A, B, ws=ws)
    assert fa.check_device_status(ws) == 0
    Ao, Bo = O.quantize(a, O.NVFP4_GLOBAL), O.quantize(b, O.NVFP4_GLOBAL)
    assert np.abs(d.cpu().numpy() - O.gemm(Ao, Bo)).max() <= O.gemm_tolerance(Ao, Bo)


def test_linear_bindings_copy_strided_inputs():
    """The linear calls take no leading dimension, so the binding copies a
    strided input (here a column slice of a wider tensor) to a contiguous
    one: outputs are byte-identical to the same calls on contiguous copies."""
    need_gpu()
    T, Cin, Cout = 256, 384, 512
    wide_x = workloads.act(T, Cin + 64, seed=31).cuda()
    wide_dy = workloads.grad(T, Cout + 32, seed=32).cuda()
    x, dy = wide_x[:, 16:16 + Cin], wide_dy[:, 8:8 + Cout]
    assert not x.is_contiguous() and not dy.is_contiguous()
    w = workloads.weight(Cout, Cin, seed=33)
    wq = to_gpu_qt(O.quantize(w, O.NVFP4_GLOBAL))
    y1, y2 = fa.linear_fwd(x, wq, fa.NVFP4_GLOBAL), fa.linear_fwd(x.contiguous(), wq, fa.NVFP4_GLOBAL)
    dw1 = fa.linear_wgrad(dy, x, SIGN_MASK, fa.RNE, 0)
    dw2 = fa.linear_wgrad(dy.contiguous(), x.contiguous(), SIGN_MASK, fa.RNE, 0)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(dw1.view(torch.int32), dw2.view(torch.int32))
