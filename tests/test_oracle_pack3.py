"""Pins of the oracle's packed 3-bit storage (oracle_pack3 / oracle_unpack3).

The IF4 paper page's 3-bit formats table (beside Table 6) gives the bits per
parameter of MXFP3 (UE8M0 scale, E2M0, blocks of 32: 3.25), NVINT3 (E4M3,
INT3, 16: 3.5), NVFP3 (E4M3, E2M0, 16: 3.5) and IF3 (UE4M3, INT3 / E2M0, 16:
3.5): 3 bits per element plus the scale.  The bit order is this library's
reading: element i of a block at bits 3i .. 3i+2 of its 6 bytes, least
significant bit first, the sign as the top bit of the three."""
import numpy as np
import pytest

import oracle

TABLE_BITS_PER_PARAMETER = {oracle.MXFP3: 3.25, oracle.NVINT3: 3.5, oracle.NVFP3: 3.5, oracle.IF3: 3.5}


def test_hand_worked_block():
    # nibbles: e0 = +1 (0x1), e1 = -1 (0x9), e2 = +3 (0x3), e3 = -2 (0xA), the rest 0
    codes = np.zeros((1, 8), dtype=np.uint8)
    codes[0, 0] = 0x91
    codes[0, 1] = 0xA3
    scales = np.array([[0x38]], dtype=np.uint8)
    pc, ps = oracle.pack3(codes, scales, oracle.NVFP3)
    # 3-bit values 1, 5, 3, 6 at bits 0, 3, 6, 9: 0b110_011_101_001 = 0x0CE9
    assert pc.tolist() == [[0xE9, 0x0C, 0, 0, 0, 0]]
    assert ps.tolist() == [[0x38]]
    # every element -3 (0xB -> 0b111): all 48 bits set
    pc2, _ = oracle.pack3(np.full((1, 8), 0xBB, dtype=np.uint8), scales, oracle.NVINT3)
    assert pc2.tolist() == [[0xFF] * 6]


@pytest.mark.parametrize("mode", [oracle.NVFP3, oracle.NVINT3, oracle.IF3, oracle.MXFP3])
def test_round_trip_every_code(mode):
    rng = np.random.default_rng(mode)
    vr, vc = 8, 128
    valid = np.array([0, 1, 2, 3, 8, 9, 10, 11], dtype=np.uint8)   # sign bit 3, magnitude bits 0..1
    nib = valid[rng.integers(0, 8, size=(vr, vc))]
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    scales = rng.integers(0, 256, size=(vr, vc // 16)).astype(np.uint8)
    if mode == oracle.MXFP3:
        scales[:, 1::2] = scales[:, 0::2]          # one byte per 32-element group, stored in both halves
    pc, ps = oracle.pack3(codes, scales, mode)
    c2, s2 = oracle.unpack3(pc, ps, vc, mode)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)


@pytest.mark.parametrize("mode", [oracle.NVFP3, oracle.NVINT3, oracle.IF3, oracle.MXFP3])
def test_bits_per_parameter_match_the_table(mode):
    vr, vc = 4, 256
    codes = np.zeros((vr, vc // 2), dtype=np.uint8)
    scales = np.zeros((vr, vc // 16), dtype=np.uint8)
    pc, ps = oracle.pack3(codes, scales, mode)
    assert (pc.size + ps.size) * 8 / (vr * vc) == TABLE_BITS_PER_PARAMETER[mode]


@pytest.mark.parametrize("mode", [oracle.NVFP3, oracle.NVINT3, oracle.IF3, oracle.MXFP3])
def test_quantized_tensor_survives_packing(mode):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((32, 64)).astype(np.float32)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)   # bf16 truncation is fine for an input
    codes, scales, gs = oracle.quantize(xb, 0, mode, 0, 5)
    pc, ps = oracle.pack3(codes, scales, mode)
    c2, s2 = oracle.unpack3(pc, ps, 64, mode)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)
    assert np.array_equal(oracle.dequantize(c2, s2, gs, mode, 0, 5), oracle.dequantize(codes, scales, gs, mode, 0, 5))
