"""Pins for the oracle's NVFP4 and fp8r quantizers (CPU only).

The pages ("BFL (fp8r / nvfp4)", format bullets) fix: block of 16 along K, an
E4M3 scale per block, packed E2M1 codes two per byte, an fp32 global scale; for
fp8r an fp32 scale per row and E4M3 values.  These tests check the oracle against
invariants and closed-form special cases that any correct encoder must satisfy,
with the reference values computed here in fp64 from the definitions.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def bf16_from_f64(v: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.bfloat16)
    assert np.array_equal(t.float().numpy().astype(np.float64), np.asarray(v, np.float64)), \
        "test values must be exact in bf16"
    return t


def unpack(codes: np.ndarray) -> np.ndarray:
    """[R, K/2] bytes -> [R, K] 4-bit codes, element 2j from the low nibble."""
    lo = codes & 0xF
    hi = codes >> 4
    out = np.empty((codes.shape[0], codes.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def e2m1_values(c4: np.ndarray) -> np.ndarray:
    mag = E2M1_GRID[c4 & 7]
    return np.where(c4 & 8, -mag, mag)


def test_global_scale_is_amax_over_2688():
    x = synth.bf16_normal((64, 128), 1.0, 5, 0.01, 20.0)
    g = oracle.nvfp4_global_scale(x)
    amax = float(x.float().abs().max())
    assert g == np.float32(np.float32(amax) / np.float32(448 * 6))


def test_on_grid_blocks_read_off_directly():
    """Every block holds +-6g once and other values on g*{E2M1 grid}: scales decode
    to exactly 1.0 (E4M3 0x38), codes are the grid indices, dequant is exact."""
    rng = np.random.default_rng(7)
    R, K = 8, 64
    g = 2.0 ** -3
    idx = rng.integers(0, 16, size=(R, K))
    idx[:, ::16] = 7                      # one +6 per block
    x = e2m1_values(idx.astype(np.uint8)) * g
    codes, sf = oracle.nvfp4_quantize(bf16_from_f64(x), np.float32(g))
    c4 = unpack(codes)
    # a zero input may carry either sign bit; compare values, then signs of nonzeros
    assert np.array_equal(e2m1_values(c4), e2m1_values(idx.astype(np.uint8)))
    assert np.all(sf == 0x38)
    assert np.array_equal(oracle.nvfp4_dequant(codes, sf, g), x)


def test_nibble_order_element_2j_low():
    x = np.zeros((1, 16))
    x[0, 0] = 6.0      # element 0 -> low nibble of byte 0
    x[0, 3] = -3.0     # element 3 -> high nibble of byte 1
    codes, sf = oracle.nvfp4_quantize(bf16_from_f64(x), np.float32(1.0))
    assert codes[0, 0] == 0x07
    assert codes[0, 1] == (0xD << 4)
    assert sf[0, 0] == 0x38


def _blocks_reference(x64: np.ndarray, g: float):
    """Per-block quantities from the definitions, in fp64 (for the invariants)."""
    R, K = x64.shape
    xb = x64.reshape(R, K // 16, 16)
    amax = np.abs(xb).max(axis=2)
    return xb, amax


@pytest.mark.parametrize("seed,p,f", [(0, 0.01, 20.0), (3, 0.0, 1.0), (11, 0.005, 30.0)])
def test_quantizer_rounds_to_nearest_grid_point(seed, p, f):
    x = synth.bf16_normal((64, 256), 1.0, seed, p, f)
    g = oracle.nvfp4_global_scale(x)
    codes, sf = oracle.nvfp4_quantize(x, g)
    x64 = x.float().numpy().astype(np.float64)
    xb, amax = _blocks_reference(x64, float(g))
    sd = np.array([oracle.e4m3_decode(int(b)) for b in sf.ravel()]).reshape(sf.shape)
    d = sd * float(g)
    vals = e2m1_values(unpack(codes)).reshape(xb.shape)
    # scale: nearest E4M3 value of amax/(6g) (fp64), up to the binary32 rounding
    s64 = amax / (6.0 * float(g))
    for sb, s in zip(sf.ravel(), s64.ravel()):
        best = min(abs(oracle.e4m3_decode(c) - s) for c in range(0x7F))
        # two binary32 roundings (6*g and the division) move s by < 2^-22 relative
        assert abs(oracle.e4m3_decode(int(sb)) - s) <= best + 2.0 ** -22 * s
    # codes: nearest grid point to x/d (fp64), except within 1e-6 of a tie
    y = xb / d[:, :, None]
    ay = np.abs(y)
    chosen = np.abs(vals)
    err = np.abs(ay - chosen)
    best = np.abs(ay[..., None] - E2M1_GRID).min(axis=-1)
    assert np.all(err <= best + 1e-6 * np.maximum(ay, 1.0))
    # sign kept
    nz = chosen > 0
    assert np.all(np.sign(vals[nz]) == np.sign(xb[nz]))


@pytest.mark.parametrize("seed", [1, 2])
def test_quantizer_error_bound_and_block_max(seed):
    x = synth.bf16_normal((32, 512), 1.0, seed, 0.01, 20.0)
    g = oracle.nvfp4_global_scale(x)
    codes, sf = oracle.nvfp4_quantize(x, g)
    x64 = x.float().numpy().astype(np.float64)
    xh = oracle.nvfp4_dequant(codes, sf, float(g))
    xb, amax = _blocks_reference(x64, float(g))
    sd = np.array([oracle.e4m3_decode(int(b)) for b in sf.ravel()]).reshape(sf.shape)
    d = sd * float(g)
    bound = d * 1.0 + np.maximum(0.0, amax - 6.0 * d)
    errb = np.abs(xb - xh.reshape(xb.shape)).max(axis=2)
    assert np.all(errb <= bound * (1 + 1e-6))
    # the block max maps to +-6 whenever the scale is a normal E4M3 number
    c4 = unpack(codes).reshape(xb.shape)
    imax = np.abs(xb).argmax(axis=2)
    normal = (sf >= 0x08) & (sf <= 0x7E)
    top = np.take_along_axis(c4, imax[..., None], axis=2)[..., 0] & 7
    assert np.all(top[normal] == 7)


def test_idempotent_with_fixed_global():
    """Q(D(Q(x))) == Q(x) for a power-of-two g (so D(Q(x)) is exact in bf16)."""
    x = synth.bf16_normal((16, 256), 1.0, 21, 0.02, 10.0)
    g = np.float32(2.0 ** -6)
    codes, sf = oracle.nvfp4_quantize(x, g)
    xh = oracle.nvfp4_dequant(codes, sf, float(g))
    codes2, sf2 = oracle.nvfp4_quantize(bf16_from_f64(xh), g)
    assert np.array_equal(sf2, sf)
    # +0 and -0 codes decode to the same value; compare values
    assert np.array_equal(e2m1_values(unpack(codes2)), e2m1_values(unpack(codes)))


def test_zero_blocks_and_zero_global():
    x = np.zeros((2, 32))
    x[1, 16:] = 1.0
    codes, sf = oracle.nvfp4_quantize(bf16_from_f64(x), np.float32(1.0 / 6.0))
    assert np.all(codes[0] == 0) and np.all(sf[0] == 0) and np.all(codes[1, :8] == 0)
    assert sf[1, 0] == 0
    # g == 0: every block gives zero codes
    codes, sf = oracle.nvfp4_quantize(bf16_from_f64(x), np.float32(0.0))
    assert np.all(codes == 0)


def test_saturation_with_undersized_global():
    """input_scale at half the true amax/2688: the largest blocks saturate their
    scale at 448 and their largest elements at code 6."""
    x = synth.bf16_normal((16, 256), 1.0, 31, 0.01, 30.0)
    g_true = oracle.nvfp4_global_scale(x)
    g = np.float32(g_true / np.float32(2.0))
    codes, sf = oracle.nvfp4_quantize(x, g)
    x64 = x.float().numpy().astype(np.float64)
    xb, amax = _blocks_reference(x64, float(g))
    sat = amax / (6.0 * float(g)) > 464.0
    assert sat.any()
    assert np.all(sf[sat] == 0x7E)
    c4 = unpack(codes).reshape(xb.shape)
    imax = np.abs(xb).argmax(axis=2)
    top = np.take_along_axis(c4, imax[..., None], axis=2)[..., 0] & 7
    assert np.all(top[sat] == 7)


# ------------------------------------------------------------------ fp8r
def test_fp8r_row_scale_and_codes():
    x = synth.bf16_normal((32, 3072 // 8), 1.0, 40)
    q, s = oracle.fp8r_quantize(x)
    x64 = x.float().numpy().astype(np.float64)
    amax = np.abs(x64).max(axis=1)
    assert np.array_equal(s, (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32))
    vals = oracle.e4m3_decode_array(q)
    # every row's largest element encodes to +-448
    imax = np.abs(x64).argmax(axis=1)
    assert np.all(np.abs(vals[np.arange(32), imax]) == 448.0)
    # nearest E4M3 value of x/s (fp64), up to binary32 rounding of the product
    grid = np.array(sorted({abs(oracle.e4m3_decode(c)) for c in range(0x7F)}))
    y = np.abs(x64 / s.astype(np.float64)[:, None])
    best = np.abs(y[..., None] - grid).min(axis=-1)
    err = np.abs(y - np.abs(vals))
    assert np.all(err <= best + 1e-6 * np.maximum(y, 1.0))
    nz = vals != 0
    assert np.all(np.sign(vals[nz]) == np.sign(x64[nz]))


def test_fp8r_zero_row():
    x = np.zeros((2, 64))
    x[1, 5] = -3.0
    q, s = oracle.fp8r_quantize(bf16_from_f64(x))
    assert s[0] == 0 and np.all(q[0] == 0)
    assert q[1, 5] == 0xFE and s[1] == np.float32(3.0) / np.float32(448.0)
    assert math.isclose(oracle.e4m3_decode(int(q[1, 5])) * float(s[1]), -3.0, rel_tol=1e-6)
