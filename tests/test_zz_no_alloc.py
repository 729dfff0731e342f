"""The allocation-free NVFP4-global quantizer (fa4_quantize_nvfp4_global_noalloc)
against the regular entry point (fa4_quantize with a caller workspace).

Some callers cannot hand the library device scratch: a runtime that reserves
all device memory up front under a fixed plan, or code that must not call
cudaMalloc where it runs.  The no-alloc entry point keeps the amax pass's
partial maxima in a fixed array inside the library instead.  This test calls
it through the C ABI twice in a row and requires bytes identical to
fa4_quantize's each time (quantized bytes are compared exactly everywhere in
this suite).  The file is named so that pytest collects it last."""
import ctypes

import pytest
import torch

import fp4_quantization_block_b200 as fa
import workloads

pytestmark = pytest.mark.gpu


def _noalloc(x, rnd, orient, seed):
    rows, cols = x.shape
    out = fa.empty_qtensor(rows, cols, fa.NVFP4_GLOBAL, orient, x.device)
    st = fa.lib().fa4_quantize_nvfp4_global_noalloc(
        ctypes.c_void_p(x.data_ptr()), rows, cols, x.stride(0), rnd, orient, seed, out.c(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, fa.lib().fa4_status_string(st)
    return out


def _same(a: fa.QTensor, b: fa.QTensor):
    torch.cuda.synchronize()
    assert torch.equal(a.payload, b.payload)
    assert torch.equal(a.scales, b.scales)
    assert torch.equal(a.ts.view(torch.int32), b.ts.view(torch.int32))


@pytest.mark.parametrize("rnd", [fa.RNE, fa.SR], ids=["rne", "sr"])
@pytest.mark.parametrize("orient", [fa.ROWWISE, fa.COLWISE], ids=["row", "col"])
def test_noalloc_matches_workspace_quantize_twice(rnd, orient):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # two different tensors, one call each, back to back: the second call
    # reuses the library's scratch array left over from the first.  The
    # larger one needs the full 1184 partial maxima.
    xs = [workloads.sweep(4096, 8192, seed=21).cuda(), workloads.act(512, 768, seed=22).cuda()]
    for x in xs:
        got = _noalloc(x, rnd, orient, seed=5)
        want = fa.quantize(x, fa.NVFP4_GLOBAL, rnd, orient, seed=5)
        _same(got, want)
    # and the same tensor twice in a row
    a = _noalloc(xs[1], rnd, orient, seed=6)
    b = _noalloc(xs[1], rnd, orient, seed=6)
    _same(a, b)
    _same(a, fa.quantize(xs[1], fa.NVFP4_GLOBAL, rnd, orient, seed=6))


@pytest.mark.parametrize("rnd", [fa.RNE, fa.SR], ids=["rne", "sr"])
def test_noalloc_matches_the_oracle(rnd):
    """The no-alloc call on its own against the CPU oracle (not only against
    fa4_quantize): one row-wise and one column-wise tensor, bytes and the
    FP32 decode scale exact."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import numpy as np
    import oracle as O
    x = workloads.act(384, 640, seed=23)
    for orient in (fa.ROWWISE, fa.COLWISE):
        got = _noalloc(x.cuda(), rnd, orient, seed=9)
        torch.cuda.synchronize()
        want = O.quantize(x, O.NVFP4_GLOBAL, rnd, orient, seed=9)
        assert np.array_equal(got.payload.cpu().numpy(), want.payload)
        assert np.array_equal(got.scales.cpu().numpy(), want.scales)
        assert got.ts.cpu().numpy().view(np.uint32)[0] == want.ts.view(np.uint32)[0]
