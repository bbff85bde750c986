"""Pins for the oracle's E2M1 / E4M3 codecs and scale layouts (CPU only).

Each test checks the oracle against something other than itself: the closed form
of the bit definitions, an independent arithmetic encoder written here, or
torch's float8_e4m3fn cast.  Source of the formats: "BFL (fp8r / nvfp4)"
(Diffusers quantization doc), format bullets: packed E2M1 with E4M3 block-16
scales (nvfp4), E4M3 with fp32 row scales (fp8r).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ E2M1
def e2m1_closed_form(code: int) -> float:
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    v = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return -v if s else v


def test_e2m1_table_closed_form_and_value_set():
    for c in range(16):
        got = oracle.e2m1_decode(c)
        assert got == e2m1_closed_form(c)
        assert math.copysign(1.0, got) == (-1.0 if c & 8 else 1.0)
    mags = sorted({abs(oracle.e2m1_decode(c)) for c in range(16)})
    with open(os.path.join(GOLDEN, "e2m1_magnitudes.txt")) as f:
        golden = [float(t) for t in f.read().split("\n", 1)[1].split()]
    assert mags == golden == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e2m1_arith_encode(y: float) -> int:
    """Independent encoder: scale to the binade's quantum and round half-even."""
    sign = 8 if math.copysign(1.0, y) < 0 else 0
    a = abs(y)
    if a >= 6.0:
        return sign | 7
    if a < 1.0:
        q = 0.5                            # subnormal binade and [0.5, 1): quantum 0.5
    else:
        e = math.floor(math.log2(a))       # 0 for [1,2), 1 for [2,4), 2 for [4,6)
        q = 2.0 ** (e - 1)
    n = round(a / q)                       # Python round(): ties to even
    v = n * q
    if v >= 6.0:
        return sign | 7
    if v < 1.0:
        return sign | int(v / 0.5)         # 0, 0.5 -> codes 0, 1
    e = int(math.floor(math.log2(v)))
    m = int(round((v / 2.0 ** e - 1.0) * 2))
    if m == 2:                             # rounded up into the next binade
        e, m = e + 1, 0
    return sign | ((e + 1) << 1) | m


def _f32_neighbours(v):
    v = np.float32(v)
    return [np.nextafter(v, np.float32(-np.inf)), v, np.nextafter(v, np.float32(np.inf))]


def test_e2m1_encode_ties_table():
    # round to nearest, ties to the even code, saturate at 6, sign kept
    cases = [(0.25, 0x0), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4), (2.5, 0x4), (3.5, 0x6),
             (5.0, 0x6), (7.0, 0x7), (1e30, 0x7), (0.0, 0x0), (-0.0, 0x8), (-0.1, 0x8),
             (-0.25, 0x8), (-0.26, 0x9), (-5.0, 0xE), (-5.01, 0xF)]
    for y, code in cases:
        assert oracle.e2m1_encode(y) == code, y


def test_e2m1_encode_vs_arithmetic_encoder():
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    pts = set()
    for a, b in zip(mags[:-1], mags[1:]):
        for v in (a, b, (a + b) / 2):
            pts.update(float(t) for t in _f32_neighbours(v))
    rng = np.random.default_rng(1234)
    rnd = (2.0 ** rng.uniform(-12, 4, 20000)).astype(np.float32)
    pts.update(float(t) for t in rnd)
    pts.update([1e-45, 1e-30, 6.5, 100.0, 3.4e38])
    for y in list(pts):
        for s in (1.0, -1.0):
            v = float(np.float32(s * y))
            assert oracle.e2m1_encode(v) == e2m1_arith_encode(v), v


# ------------------------------------------------------------------ E4M3
def e4m3_closed_form(code: int) -> float:
    s, e, m = (code >> 7) & 1, (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return float("nan")
    v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -v if s else v


def test_e4m3_table_closed_form_and_library():
    lib_vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        got = oracle.e4m3_decode(c)
        ref = e4m3_closed_form(c)
        if math.isnan(ref):
            assert math.isnan(got) and math.isnan(lib_vals[c])
        else:
            assert got == ref == float(lib_vals[c])
    assert oracle.e4m3_decode(0x7E) == 448.0            # max finite
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9        # min subnormal
    assert math.isnan(oracle.e4m3_decode(0x7F)) and math.isnan(oracle.e4m3_decode(0xFF))


def e4m3_arith_encode(y: float) -> int:
    sign = 0x80 if math.copysign(1.0, y) < 0 else 0
    a = abs(y)
    if a >= 448.0:
        return sign | 0x7E
    if a < 2.0 ** -6:
        n = round(a / 2.0 ** -9)                   # subnormals, quantum 2^-9
        return sign | n                            # n == 8 is the first normal, code 8
    e = math.floor(math.log2(a))
    q = 2.0 ** (e - 3)
    n = round(a / q)                               # 8..16
    if n == 16:
        e, n = e + 1, 8
    if (e + 7) > 15 or ((e + 7) == 15 and n - 8 == 7):
        return sign | 0x7E
    return sign | ((e + 7) << 3) | (n - 8)


def test_e4m3_encode_vs_arithmetic_and_library():
    vals = [e4m3_closed_form(c) for c in range(0x7F)]
    pts = set()
    for a, b in zip(vals[:-1], vals[1:]):
        for v in (a, b, (a + b) / 2):
            pts.update(float(t) for t in _f32_neighbours(v))
    rng = np.random.default_rng(99)
    pts.update(float(t) for t in (2.0 ** rng.uniform(-12, 9, 20000)).astype(np.float32))
    pts.update([0.0, 448.0, 460.0, 464.0, 470.0, 1e6, 3.4e38, 1e-45])
    pts = sorted(pts)
    arr = np.array(pts + [-p for p in pts], dtype=np.float32)
    lib_codes = torch.from_numpy(arr).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for y, lc in zip(arr.tolist(), lib_codes.tolist()):
        got = oracle.e4m3_encode(y)
        assert got == e4m3_arith_encode(y), y
        if abs(y) <= 464.0:          # torch's cast: RNE, but NaN rather than saturation
            assert got == lc, y


def test_e4m3_saturates_and_keeps_sign():
    assert oracle.e4m3_encode(1e9) == 0x7E
    assert oracle.e4m3_encode(-1e9) == 0xFE
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00     # tie between 0 and 2^-9 -> even
    assert oracle.e4m3_encode(1.0625) == 0x38         # tie -> even mantissa
    assert oracle.e4m3_encode(1.1875) == 0x3A


# ------------------------------------------------------------------ scale layouts
def test_sf_mma_offsets_worked_examples_of_the_published_layout():
    """Worked examples of the scale-factor layout the block-scaled tensor-core MMA reads,
    as the cuBLAS documentation publishes it ("1D Block Scaling Factors Layout": the
    scales of 128 rows x 4 blocks form one 512-byte tile; inside it row r, block c sits
    at 16 * (r % 32) + 4 * (r // 32) + c; tiles are ordered along K first, then along
    rows).  Each expected offset below is read off that description for one (row,
    block) pair, not recomputed by the oracle's formula.  This is the CPU side only: the
    layout is pinned on the GPU by the single-hot GEMM tests, where the tensor cores
    themselves read it."""
    K = 256                      # 16 blocks of 16 -> 4 column tiles of 4
    assert oracle.sf_mma_offset(0, 0, K) == 0
    assert oracle.sf_mma_offset(0, 1, K) == 1
    assert oracle.sf_mma_offset(0, 3, K) == 3
    assert oracle.sf_mma_offset(1, 0, K) == 16
    assert oracle.sf_mma_offset(32, 0, K) == 4
    assert oracle.sf_mma_offset(96, 2, K) == 12 + 2
    assert oracle.sf_mma_offset(33, 5, K) == 512 + 16 + 4 + 1
    assert oracle.sf_mma_offset(128, 0, K) == 4 * 512
    assert oracle.sf_mma_offset(255, 15, K) == 7 * 512 + 31 * 16 + 3 * 4 + 3


@pytest.mark.parametrize("R,K", [(128, 64), (256, 256), (384, 3072 // 4), (200, 192)])
def test_sf_mma_layout_is_injective_and_padded(R, K):
    """Injectivity check: no two (row, block) pairs share a byte and every offset lies
    inside the padded size."""
    nb = K // 16
    total = oracle.sf_bytes(R, K, True)
    assert total == ((R + 127) // 128) * ((nb + 3) // 4) * 512
    offs = [oracle.sf_mma_offset(r, c, K) for r in range(R) for c in range(nb)]
    assert len(set(offs)) == len(offs)
    assert min(offs) >= 0 and max(offs) < total
    lin = np.arange(R * nb, dtype=np.int64).astype(np.uint8)
    mma = oracle.sf_linear_to_mma(lin, R, K)
    for r in range(0, R, 7):
        for c in range(nb):
            assert mma[oracle.sf_mma_offset(r, c, K)] == lin[r * nb + c]


def test_storage_bytes_closed_form():
    """NVFP4 = N*K/2 codes + N*K/16 scales + 2 fp32 globals; fp8r = N*K + 4*N.

    Context from the pages (golden/storage_sizes.txt): a 5.6B-parameter generator
    is 11.2 GB in BF16 and 5.6 GB in FP8, and a 4B model's NVFP4 weights are
    2-3 GB.  The per-parameter byte counts below reproduce those figures.
    """
    N = K = 3072
    nv = N * K // 2 + oracle.sf_bytes(N, K, False) + 8
    assert nv == N * K * 0.5625 + 8
    fp8 = N * K + 4 * N
    with open(os.path.join(GOLDEN, "storage_sizes.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    for params, fmt, lo_gb, hi_gb in rows:
        bpp = {"bf16": 2.0, "fp8": fp8 / (N * K), "nvfp4": nv / (N * K)}[fmt]
        gb = float(params) * bpp / 1e9
        assert float(lo_gb) <= gb <= float(hi_gb), (params, fmt, gb)
