"""Exhaustive pin of the GPU conversions against the oracle encoders.

"BFL (fp8r / nvfp4)" (Diffusers quantization doc), format bullets: E2M1 values and E4M3
scales.  The quantizers turn every binary32 product into a code with
cvt.rn.satfinite.e2m1x2.f32 / .e4m3x2.f32; the oracle encodes by nearest-value search
with ties to the even code and saturation (pinned on the CPU against independent
arithmetic encoders).  Here both are applied to every one of the 2^32 fp32 bit patterns
(NaNs excepted: non-finite inputs are out of scope) and must agree byte for byte, which
settles the sign of zero, every tie and the saturation boundary on the hardware.
"""
import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_act_b200 as bsp

pytestmark = pytest.mark.gpu

CHUNK = 1 << 28
NAN_RANGES = [(0x7F800001, 0x80000000), (0xFF800001, 0x100000000)]   # [lo, hi) bit patterns


def compare_chunk(kind, first):
    got = bsp.bsp_testing_cvt_range(kind, first, CHUNK).cpu().numpy()
    ref = oracle.encode_range(kind, first, CHUNK)
    keep = np.ones(CHUNK, dtype=bool)
    for lo, hi in NAN_RANGES:
        a, b = max(lo, first), min(hi, first + CHUNK)
        if a < b:
            keep[a - first:b - first] = False
    bad = np.nonzero((got != ref) & keep)[0]
    return bad, got, ref


@pytest.mark.parametrize("kind,name", [(0, "E2M1"), (1, "E4M3")])
def test_conversion_matches_oracle_on_all_fp32(kind, name):
    for c in range((1 << 32) // CHUNK):
        first = c * CHUNK
        bad, got, ref = compare_chunk(kind, first)
        if bad.size:
            i = bad[0]
            pytest.fail(f"{name}: {bad.size} mismatches in chunk {c}; first at bits "
                        f"{first + i:#010x}: gpu {got[i]:#04x}, oracle {ref[i]:#04x}")
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0


def test_conversion_special_points():
    """A few hand-picked patterns, readable on failure: +-0, ties, saturation."""
    vals = np.array([0.0, -0.0, 0.25, 0.75, 1.25, 2.5, 5.0, 6.0, 7.0, 1e30, -1e30,
                     np.inf, -np.inf], dtype=np.float32)
    bits = vals.view(np.uint32)
    for kind in (0, 1):
        for b in bits:
            got = int(bsp.bsp_testing_cvt_range(kind, int(b), 1).item())
            ref = int(oracle.encode_range(kind, int(b), 1)[0])
            assert got == ref, (kind, hex(int(b)), hex(got), hex(ref))
