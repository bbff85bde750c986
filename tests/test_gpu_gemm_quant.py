"""GPU checks of nvfp4_gemm_quant: the NVFP4 GEMM whose bf16 output is re-quantized in
the epilogue for the next nvfp4 linear (an MLP's up projection feeding its down
projection).

"BFL (fp8r / nvfp4)" (Diffusers quantization doc), Kernels table: every nvfp4 linear
quantizes its activations before the FP4 GEMM.  The fused epilogue must give exactly
the codes and scale bytes that the oracle's NVFP4 quantizer gives on the GEMM's bf16
output (oracle arm, every shape), and the same bytes as nvfp4_gemm followed by
nvfp4_quantize_act; the chained down projection must then match too.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_precision_act_b200 as bsp
from parity import sf_valid_mask


def assert_oracle_requantization(y, g_out, codes, sf, M, N):
    """Codes and valid MMA-layout scale bytes of the fused epilogue equal the oracle's
    quantizer run on the bf16 output y with the next layer's global scale g_out."""
    c_or, s_lin = oracle.nvfp4_quantize(y.cpu(), np.float32(g_out.item()))
    s_or = oracle.sf_linear_to_mma(s_lin, M, N)
    valid = sf_valid_mask(M, N)
    assert np.array_equal(codes.cpu().numpy(), c_or)
    assert np.array_equal(sf.cpu().numpy()[valid], s_or[valid])

pytestmark = pytest.mark.gpu


def prepared(x):
    g = bsp.nvfp4_global_scale(x)
    c, sf = bsp.nvfp4_quantize_act(x, g, layout=bsp.SF_MMA)
    return c, sf, g


@pytest.mark.parametrize("M,N,K,seed,with_bias", [
    (128, 256, 256, 0, False),
    (200, 320, 512, 1, True),        # ragged M, N not a multiple of the 256-wide tile
    (1, 64, 64, 2, False),           # one row, one 64-column group
    (384, 1024, 1280, 3, True),
    (4096, 12288, 3072, 4, False),   # the MLP up projection at 1 MP
    (2560, 2112, 256, 5, True),      # 90 tiles for 74 CTA pairs: second tiles in the ragged
                                     # last tile column, bias fetched ahead for them
    (4096, 12288, 3072, 6, True),    # the MLP up projection with bias (768 tiles)
])
def test_gemm_quant_equals_gemm_then_quantize(M, N, K, seed, with_bias):
    a = synth.bf16_normal((M, K), 1.0, seed, 0.005, 30.0).cuda()
    w = synth.bf16_normal((N, K), 0.02, seed + 100).cuda()
    bias = synth.bf16_normal((N,), 0.5, seed + 200).cuda() if with_bias else None
    ac, asf, ga = prepared(a)
    wc, wsf, gw = prepared(w)
    y = bsp.nvfp4_gemm(ac, asf, ga, wc, wsf, gw, bias=bias)
    g_out = bsp.nvfp4_global_scale(y)               # the next layer's calibrated scale
    c_ref, s_ref = bsp.nvfp4_quantize_act(y, g_out, layout=bsp.SF_MMA)
    sf_bytes = bsp.nvfp4_sf_bytes(M, N, bsp.SF_MMA)
    codes = torch.full((M, N // 2), 0x5A, dtype=torch.uint8, device="cuda")
    sf = torch.full((sf_bytes,), 0xA5, dtype=torch.uint8, device="cuda")
    bsp.nvfp4_gemm_quant(ac, asf, ga, wc, wsf, gw, g_out, bias=bias, out_codes=codes, out_sf=sf)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    assert torch.equal(codes, c_ref)
    valid = torch.from_numpy(sf_valid_mask(M, N)).cuda()
    assert torch.equal(sf[valid], s_ref[valid])
    assert_oracle_requantization(y, g_out, codes, sf, M, N)


def test_gemm_quant_with_saturating_scale():
    """A next-layer scale far below the output's amax: block scales saturate at 448 and
    codes at +-6, identically in both paths."""
    M, N, K = 256, 512, 512
    a = synth.bf16_normal((M, K), 1.0, 11).cuda()
    w = synth.bf16_normal((N, K), 0.02, 12).cuda()
    ac, asf, ga = prepared(a)
    wc, wsf, gw = prepared(w)
    y = bsp.nvfp4_gemm(ac, asf, ga, wc, wsf, gw)
    g_out = bsp.nvfp4_global_scale(y) * 0.01
    c_ref, s_ref = bsp.nvfp4_quantize_act(y, g_out, layout=bsp.SF_MMA)
    codes, sf = bsp.nvfp4_gemm_quant(ac, asf, ga, wc, wsf, gw, g_out)
    torch.cuda.synchronize()
    assert torch.equal(codes, c_ref)
    valid = torch.from_numpy(sf_valid_mask(M, N)).cuda()
    assert torch.equal(sf[valid], s_ref[valid])
    assert (s_ref[valid] == 0x7E).any()
    assert_oracle_requantization(y, g_out, codes, sf, M, N)


def test_mlp_chain_through_fused_requantization():
    """Up projection with the fused re-quantization, then the down projection on its
    codes: equal to the unfused chain bit for bit."""
    wl = synth.WORKLOADS["nvfp4_mlp_1mp"]
    M = 512
    a = wl.A_rows(M).cuda()
    w1, w2 = wl.W().cuda(), wl.W2().cuda()
    ac, asf, ga = prepared(a)
    w1c, w1sf, g1 = prepared(w1)
    w2c, w2sf, g2w = prepared(w2)
    y1 = bsp.nvfp4_gemm(ac, asf, ga, w1c, w1sf, g1)
    g2 = bsp.nvfp4_global_scale(y1)
    y1c, y1sf = bsp.nvfp4_quantize_act(y1, g2, layout=bsp.SF_MMA)
    ref = bsp.nvfp4_gemm(y1c, y1sf, g2, w2c, w2sf, g2w)
    qc, qsf = bsp.nvfp4_gemm_quant(ac, asf, ga, w1c, w1sf, g1, g2)
    out = bsp.nvfp4_gemm(qc, qsf, g2, w2c, w2sf, g2w)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    assert torch.equal(out, ref)
