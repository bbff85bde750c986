"""Pins of the oracle's bf16 decode (the weight decode of the dequantise-only fallback,
closing paragraph of the "Kernels" section of "BFL (fp8r / nvfp4)").

The oracle computes bf16_rne(fl32(e2m1(code) * e4m3(sb)) * g).  It is checked here
against routes that share nothing with it: E2M1 values from the bit definition, E4M3
values from torch's float8_e4m3fn dtype, binary32 products from numpy and the bf16
rounding from torch's float32 -> bfloat16 cast."""
import numpy as np
import pytest
import torch

import oracle
import synth


def e2m1_from_bits(code: int) -> float:
    s = -1.0 if code & 0x8 else 1.0
    e, m = (code >> 1) & 3, code & 1
    return s * (m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0))


E4M3_TORCH = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
FINITE_POS_SCALES = np.array([b for b in range(0x7F)], dtype=np.uint8)   # 0x00..0x7E


def reference_bf16(codes_lin: np.ndarray, sb: np.ndarray, g: np.float32) -> np.ndarray:
    """codes_lin: one 4-bit code per element [R, K]; sb: scale byte per element."""
    e2 = np.vectorize(e2m1_from_bits)(codes_lin).astype(np.float64)
    p = (e2 * E4M3_TORCH[sb].astype(np.float64)).astype(np.float32)   # exact products
    y = p * np.float32(g)                                               # one fp32 rounding
    return torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def pack(codes_lin: np.ndarray) -> np.ndarray:
    return (codes_lin[:, 0::2] | (codes_lin[:, 1::2] << 4)).astype(np.uint8)


@pytest.mark.parametrize("g", [1.0, 2.0 ** -7, 1.0 / 2688.0, 3.0e-4, 0.37, 5.9e-39])
def test_every_code_and_scale_byte(g):
    # rows: one per finite positive scale byte; columns: the 16 codes
    R, K = len(FINITE_POS_SCALES), 16
    codes_lin = np.tile(np.arange(16, dtype=np.uint8), (R, 1))
    sf_lin = FINITE_POS_SCALES.reshape(R, 1)
    got = oracle.nvfp4_dequant_bf16(pack(codes_lin), sf_lin, g)
    want = reference_bf16(codes_lin, np.repeat(sf_lin, K, axis=1), np.float32(g))
    assert np.array_equal(got, want)


@pytest.mark.parametrize("g", [1.0, 0.5, 2.0 ** -10, 64.0])
def test_power_of_two_global_is_exact(g):
    """With g a power of two every decoded value has at most 6 significant bits, so the
    bf16 result equals the exact dequantised value."""
    rng = np.random.Generator(np.random.PCG64(5))
    codes = rng.integers(0, 256, size=(37, 64), dtype=np.uint8)
    sf = rng.integers(0, 0x7F, size=(37, 8), dtype=np.uint8)    # K = 128: 8 blocks
    got = oracle.nvfp4_dequant_bf16(codes, sf, g)
    exact = oracle.nvfp4_dequant(codes, sf, g)
    got_f = torch.from_numpy(got.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(got_f, exact)


def test_quantized_tensor_within_bf16_of_fp64_decode():
    """On a real quantized tensor the bf16 decode is the fp64 dequantised value rounded
    twice (fp32, bf16): relative error at most 2^-8 + 2^-24 (or exact zero)."""
    x = synth.bf16_normal((96, 256), 1.0, 3, 0.01, 20.0)
    g = oracle.nvfp4_global_scale(x)
    codes, sf = oracle.nvfp4_quantize(x, g)
    got = oracle.nvfp4_dequant_bf16(codes, sf, float(g))
    got_f = torch.from_numpy(got.view(np.int16)).view(torch.bfloat16).double().numpy()
    exact = oracle.nvfp4_dequant(codes, sf, float(g))
    nz = exact != 0
    assert np.all(got_f[~nz] == 0)
    rel = np.abs(got_f[nz] - exact[nz]) / np.abs(exact[nz])
    assert rel.max() <= 2.0 ** -8 + 2.0 ** -24


def test_sign_of_zero_kept():
    codes = np.array([[0x80] * 8], dtype=np.uint8)      # element 0: +0, element 1: -0
    got = oracle.nvfp4_dequant_bf16(codes, np.array([[0x38]], dtype=np.uint8), 1.0)
    assert list(got[0][:2]) == [0x0000, 0x8000]
