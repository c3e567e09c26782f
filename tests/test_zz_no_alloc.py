"""nvfp4_quantize_noalloc gives the same bytes as nvfp4_quantize.

Some callers cannot hand the library the small workspace nvfp4_quantize needs
when it computes the tensor amax itself -- an engine plugin that receives only
its input and output buffers, or a process whose framework keeps all device
memory in its own pool, where a new cudaMalloc would fail or stall the host.
nvfp4_quantize_noalloc serves them from a fixed array of device memory built
into the library.  This test calls it through the C ABI twice in a row, the
second tensor with a far smaller amax (stale scratch from the first call would
inflate the second call's tensor scale), and compares both results with
nvfp4_quantize's, exactly.  It lives in its own file, collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [(W.ROWWISE, W.RTN, 0), (W.ROWWISE, W.MS_EDEN, 128), (W.TRANSPOSED, W.MS_EDEN, 128),
         (W.TRANSPOSED, W.SR, 32), (W.ROWWISE, W.IF4, 0), (W.ROWWISE, W.FOUR_OVER_SIX, 16),
         (W.TRANSPOSED, W.SCALE_SEARCH, 0)]


def _noalloc(x, layout, mode, g, seed, stream):
    rows, cols = x.shape
    codes, scales, gs = N.alloc_outputs(rows, cols, layout, x.device)
    P = ctypes.c_void_p
    st = N.nvfp4_quantize_noalloc(P(x.data_ptr()), rows, cols, x.stride(0), layout, mode, g, seed, None,
                                  P(codes.data_ptr()), P(scales.data_ptr()), P(gs.data_ptr()), stream)
    assert st == 0, N.nvfp4_status_string(st)
    return codes, scales, gs


@pytest.mark.parametrize("layout,mode,g", CASES)
def test_noalloc_matches_quantize_on_two_calls_in_a_row(layout, mode, g):
    gen = torch.Generator(device="cuda").manual_seed(11)
    big = (torch.randn((512, 384), generator=gen, device="cuda") * 100.0).to(torch.bfloat16)
    small = (torch.randn((512, 384), generator=gen, device="cuda") * 0.01).to(torch.bfloat16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    got = [_noalloc(x, layout, mode, g, 5, stream) for x in (big, small)]   # back to back, one stream
    ref = [N.quantize(x, layout, mode, g, 5) for x in (big, small)]
    torch.cuda.synchronize()
    for (gc, gs_, gg), (rc, rs, rg) in zip(got, ref):
        assert torch.equal(gc, rc)
        assert torch.equal(gs_, rs)
        assert gg.item() == rg.item()
    assert got[1][2].item() < got[0][2].item() * 1e-3   # the second tensor scale really is the smaller one


def test_noalloc_with_supplied_amax():
    x = W.small().tensors("cuda")["x"]
    amax = N.amax(x, W.ROWWISE, 128, 3)
    rows, cols = x.shape
    codes, scales, gs = N.alloc_outputs(rows, cols, W.ROWWISE, x.device)
    P = ctypes.c_void_p
    st = N.nvfp4_quantize_noalloc(P(x.data_ptr()), rows, cols, cols, W.ROWWISE, W.MS_EDEN, 128, 3,
                                  P(amax.data_ptr()), P(codes.data_ptr()), P(scales.data_ptr()),
                                  P(gs.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    rc, rs, rg = N.quantize(x, W.ROWWISE, W.MS_EDEN, 128, 3)
    torch.cuda.synchronize()
    assert torch.equal(codes, rc) and torch.equal(scales, rs) and gs.item() == rg.item()
