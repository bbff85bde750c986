"""nvfp4_dequantize (the dequantise-only fallback's weight decode, closing paragraph of the
"Kernels" section of "BFL (fp8r / nvfp4)") against the CPU oracle: bit-exact bf16; and the
fallback linear it enables against the fused path."""
import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_precision_act_b200 as bsp

pytestmark = pytest.mark.gpu

FINITE_SCALES = np.array([b for b in range(256) if (b & 0x7F) != 0x7F], dtype=np.uint8)


def gpu_decode(codes, sf_lin, g, layout):
    rows, K = codes.shape[0], 2 * codes.shape[1]
    c = torch.from_numpy(codes).cuda()
    sf = torch.from_numpy(sf_lin).cuda()
    if layout == bsp.SF_MMA:
        sf = torch.from_numpy(oracle.sf_linear_to_mma(sf_lin, rows, K)).cuda()
    gt = torch.tensor([g], dtype=torch.float32, device="cuda")
    out = bsp.nvfp4_dequantize(c, sf, gt, layout=layout)
    torch.cuda.synchronize()
    return out.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("g", [1.0, 1.0 / 2688.0, 0.37, 5.9e-39])
def test_every_code_byte_and_scale_byte(g):
    """All 256 code bytes (512 elements) in every row, one row per finite E4M3 scale byte
    (both signs): the nibble order of the decode and every scale value are pinned."""
    rows, K = len(FINITE_SCALES), 512
    codes = np.tile(np.arange(256, dtype=np.uint8), (rows, 1))
    sf_lin = np.repeat(FINITE_SCALES.reshape(rows, 1), K // 16, axis=1)
    want = oracle.nvfp4_dequant_bf16(codes, sf_lin, np.float32(g))
    for layout in (bsp.SF_LINEAR, bsp.SF_MMA):
        got = gpu_decode(codes, sf_lin, np.float32(g), layout)
        assert np.array_equal(got, want), f"layout {layout}"


@pytest.mark.parametrize("rows,K,layout", [(200, 3072, bsp.SF_MMA), (131, 1216, bsp.SF_MMA),
                                           (7, 48, bsp.SF_LINEAR), (1, 16, bsp.SF_LINEAR)])
def test_quantized_tensor_round_trip(rows, K, layout):
    x = synth.bf16_normal((rows, K), 0.02, rows + K, 0.01, 20.0)
    g = oracle.nvfp4_global_scale(x)
    codes, sf_lin = oracle.nvfp4_quantize(x, g)
    want = oracle.nvfp4_dequant_bf16(codes, sf_lin, g)
    assert np.array_equal(gpu_decode(codes, sf_lin, g, layout), want)


def test_attention_weight_full_size():
    """The 1 MP attention weight [3072, 3072], quantized on the GPU, decoded on the GPU
    from the MMA layout: bit-exact with the oracle's decode of the same codes."""
    wl = synth.WORKLOADS["nvfp4_attn_1mp"]
    w = wl.W().cuda()
    gw = bsp.nvfp4_global_scale(w)
    wc, wsf = bsp.nvfp4_quantize_act(w, gw, layout=bsp.SF_LINEAR)
    out = bsp.nvfp4_dequantize(wc, wsf, gw, layout=bsp.SF_LINEAR)
    wsf_mma = bsp.nvfp4_sf_convert(wsf, wl.N, wl.K, bsp.SF_LINEAR, bsp.SF_MMA)
    out_mma = bsp.nvfp4_dequantize(wc, wsf_mma, gw, layout=bsp.SF_MMA)
    torch.cuda.synchronize()
    want = oracle.nvfp4_dequant_bf16(wc.cpu().numpy(), wsf.cpu().numpy().reshape(wl.N, wl.K // 16),
                                     float(gw.item()))
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, want)
    assert torch.equal(out, out_mma)


def test_fallback_differs_slightly_from_fused():
    """The closing paragraph of the Kernels section: the fallback (bf16 weights decoded
    from NVFP4, bf16 activations not quantized, a plain bf16 GEMM) gives outputs that
    differ slightly from the fused path.  On sampled rows of the 1 MP attention linear,
    both stay close to the unquantized bf16 product, the fallback closer (it carries only
    the weight's quantization error), and the two are not identical."""
    wl = synth.WORKLOADS["nvfp4_attn_1mp"]
    a_cpu, w_cpu, b_cpu = wl.A(), wl.W(), wl.bias_vec()
    a, w, b = a_cpu.cuda(), w_cpu.cuda(), b_cpu.cuda()
    ga, gw = bsp.nvfp4_global_scale(a), bsp.nvfp4_global_scale(w)
    wc, wsf = bsp.nvfp4_quantize_act(w, gw, layout=bsp.SF_MMA)
    y_fused = bsp.nvfp4_linear(a, ga, wc, wsf, gw, bias=b)
    w_hat = bsp.nvfp4_dequantize(wc, wsf, gw, layout=bsp.SF_MMA)
    y_fb = (a @ w_hat.t() + b).to(torch.bfloat16)            # library bf16 GEMM
    torch.cuda.synchronize()
    rows = np.arange(0, wl.M, 61)
    A = a_cpu.double().numpy()[rows]
    W = w_cpu.double().numpy()
    ref = A @ W.T + b_cpu.double().numpy()[None, :]
    denom = np.linalg.norm(A, axis=1)[:, None] * np.linalg.norm(W, axis=1)[None, :]
    e_fused = np.abs(y_fused.float().cpu().numpy()[rows] - ref) / denom
    e_fb = np.abs(y_fb.float().cpu().numpy()[rows] - ref) / denom
    rms = lambda e: float(np.sqrt(np.mean(e ** 2)))
    print(f"fallback vs bf16 product: rms {rms(e_fb):.3e} max {e_fb.max():.3e}; "
          f"fused: rms {rms(e_fused):.3e} max {e_fused.max():.3e}")
    assert rms(e_fb) < rms(e_fused) < 0.1
    assert not torch.equal(y_fused, y_fb)
