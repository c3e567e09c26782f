"""nvfp4_pack3 / nvfp4_unpack3 through the C ABI: the packed bytes of a GPU
quantization equal the oracle's packing of the same codes, bit for bit, and
unpacking restores the codes and scales exactly."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", [W.NVFP3, W.NVINT3, W.IF3, W.MXFP3])
@pytest.mark.parametrize("layout,g", [(W.ROWWISE, 0), (W.TRANSPOSED, 128)])
@pytest.mark.parametrize("shape", [(256, 384), (1024, 2048)])
def test_pack3_matches_oracle(mode, layout, g, shape):
    gen = torch.Generator().manual_seed(shape[0] + mode)
    x = torch.randn(*shape, generator=gen).to(torch.bfloat16).cuda()
    codes, scales, _ = N.quantize(x, layout, mode, g, seed=7)
    pc, ps = N.pack3(codes, scales, mode)
    vc = 2 * codes.shape[1]
    c2, s2 = N.unpack3(pc, ps, vc, mode)
    torch.cuda.synchronize()
    codes_h, scales_h = codes.cpu().numpy(), scales.cpu().numpy()
    epc, eps = oracle.pack3(codes_h, scales_h, mode)
    assert np.array_equal(pc.cpu().numpy(), epc)
    assert np.array_equal(ps.cpu().numpy(), eps)
    assert np.array_equal(c2.cpu().numpy(), codes_h)
    assert np.array_equal(s2.cpu().numpy(), scales_h)
    bits = (pc.numel() + ps.numel()) * 8 / (codes.shape[0] * vc)
    assert bits == (3.25 if mode == W.MXFP3 else 3.5)
