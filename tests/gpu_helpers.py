"""Helpers shared by the GPU parity tests: run one call through the C ABI and
through the oracle on the same seeded input, and compare element by element."""
import numpy as np
import torch

import oracle
from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W


def bits(t: torch.Tensor) -> np.ndarray:
    return W.bf16_bits(t.cpu())


def to_device(x_cpu: torch.Tensor, ld_pad: int = 0) -> torch.Tensor:
    """Copy a bf16 CPU matrix to the GPU, optionally inside a wider (ld = cols + pad) buffer."""
    rows, cols = x_cpu.shape
    if ld_pad == 0:
        return x_cpu.cuda()
    buf = torch.zeros((rows, cols + ld_pad), dtype=torch.bfloat16, device="cuda")
    buf[:, :cols] = x_cpu.cuda()
    return buf[:, :cols]


def gpu_quantize(x_dev, layout, mode, g, seed, amax=None):
    amax_t = None if amax is None else torch.tensor([amax], dtype=torch.float32, device="cuda")
    codes, scales, gs = N.quantize(x_dev, layout, mode, g, seed, amax_in=amax_t)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), float(gs.item())


def mismatch_report(name, got, exp):
    bad = np.argwhere(got != exp)
    if len(bad) == 0:
        return ""
    i = tuple(bad[0])
    return f"{name}: {len(bad)} of {got.size} differ, first at {i}: got {got[i]:#x} expected {exp[i]:#x}"


def assert_same(gpu, orc, what=""):
    gc, gsc, gg = gpu
    oc, osc, og = orc
    msgs = [m for m in (mismatch_report("codes", gc, oc), mismatch_report("scales", gsc, osc)) if m]
    if gg != og and not (np.isnan(gg) and np.isnan(og)):
        msgs.append(f"global scale {gg!r} vs {og!r}")
    assert not msgs, what + ": " + "; ".join(msgs)


def compare_call(x_cpu, layout, mode, g, seed, ld_pad=0, amax=None):
    x_dev = to_device(x_cpu, ld_pad)
    gpu = gpu_quantize(x_dev, layout, mode, g, seed, amax)
    orc = oracle.quantize(bits(x_cpu), layout, mode, g, seed, amax_in=amax)
    assert_same(gpu, orc, f"layout={layout} mode={mode} g={g} shape={tuple(x_cpu.shape)} ld_pad={ld_pad}")
    return gpu
