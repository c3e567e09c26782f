"""GPU parity at the workloads' full sizes, in the launch configuration bench.py
times (the same C-ABI call on the same shapes), on sampled output rows.  The
tensors are drawn on the GPU and copied to the host for the oracle.

For each call the oracle computes the tensor amax over the whole tensor (so the
FP32 tensor scale is checked exactly) and then only the sampled view rows; the
GPU output rows are compared with them bit for bit.  The first, the last and
randomly drawn view rows are sampled.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W

from gpu_helpers import bits

pytestmark = pytest.mark.gpu

N_SAMPLED_ROWS = 12


def _check_workload(wl):
    tensors = wl.tensors("cuda")
    host = {k: v.cpu() for k, v in tensors.items()}
    for call in wl.calls:
        x = tensors[call.tensor]
        xb = bits(host[call.tensor])
        rows, cols = x.shape
        vr, vc = N.view_shape(rows, cols, call.layout)
        codes, scales, gs = N.quantize(x, call.layout, call.mode, call.rht_group, wl.seed)
        torch.cuda.synchronize()
        A = oracle.amax(xb, call.layout, call.rht_group, wl.seed)
        assert float(gs.item()) == oracle.global_scale(A, call.mode), call.name
        rng = np.random.default_rng(abs(hash(call.name)) % (1 << 32))
        sample = sorted(set([0, vr - 1] + list(rng.integers(0, vr, N_SAMPLED_ROWS - 2))))
        codes_h, scales_h = codes.cpu().numpy(), scales.cpu().numpy()
        for r in sample:
            oc, osc, og = oracle.quantize(xb, call.layout, call.mode, call.rht_group, wl.seed, amax_in=A,
                                          row_range=(r, r + 1))
            assert np.array_equal(codes_h[r], oc[r]), (call.name, r, int(np.sum(codes_h[r] != oc[r])))
            assert np.array_equal(scales_h[r], osc[r]), (call.name, r, int(np.sum(scales_h[r] != osc[r])))
        del codes, scales, gs


@pytest.mark.parametrize("name", ["weight", "gradient", "activation", "mlp_up"])
def test_full_size_sampled(name):
    _check_workload(W.ALL[name]())
