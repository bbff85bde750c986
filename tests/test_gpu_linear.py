"""GPU checks of nvfp4_linear, the one-call nvfp4 linear forward.

"BFL (fp8r / nvfp4)" (Diffusers quantization doc), Kernels table: the nvfp4 linear
quantizes its activations at run time and runs the block-scaled FP4 GEMM.
nvfp4_linear runs exactly those two kernels (the GEMM as a programmatic dependent of
the quantizer), so its output must equal the two separate calls bit for bit; the
quantized activations it leaves in the workspace must equal the oracle's codes; and
the output must meet the oracle within the tolerances of tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_precision_act_b200 as bsp
from parity import bf16_bias_np, compare_gemm, nvfp4_dequant_rows, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["pair", "single"], autouse=True)
def gemm_kernel(request):
    old = bsp.bsp_testing_set_gemm_kernel({"pair": 1, "single": 2}[request.param])
    yield request.param
    bsp.bsp_testing_set_gemm_kernel(old)


def prepared_weight(w):
    gw = bsp.nvfp4_global_scale(w)
    wc, wsf = bsp.nvfp4_quantize_act(w, gw, layout=bsp.SF_MMA)
    return wc, wsf, gw


def two_calls(a, ga, wc, wsf, gw, bias):
    ac, asf = bsp.nvfp4_quantize_act(a, ga, layout=bsp.SF_MMA)
    return bsp.nvfp4_gemm(ac, asf, ga, wc, wsf, gw, bias=bias), ac


@pytest.mark.parametrize("M,N,K,seed,with_bias", [
    (128, 256, 256, 0, False),
    (200, 136, 320, 3, True),        # ragged M and N
    (1, 8, 64, 4, False),            # one row
    (130, 264, 1216, 5, True),
    (384, 512, 1280, 7, False),
    (1024, 3072, 3072, 10, True),    # the attention projection's N and K
])
def test_linear_equals_two_calls(M, N, K, seed, with_bias):
    a = synth.bf16_normal((M, K), 1.0, seed, 0.01, 20.0).cuda()
    w = synth.bf16_normal((N, K), 0.02, seed + 100).cuda()
    bias = synth.bf16_normal((N,), 0.5, seed + 200).cuda() if with_bias else None
    wc, wsf, gw = prepared_weight(w)
    ga = bsp.nvfp4_global_scale(a)
    ws = torch.full((bsp.nvfp4_linear_workspace_bytes(M, K),), 0xAB, dtype=torch.uint8,
                    device="cuda")
    y1 = bsp.nvfp4_linear(a, ga, wc, wsf, gw, bias=bias, workspace=ws)
    y2, ac = two_calls(a, ga, wc, wsf, gw, bias)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    assert torch.equal(y1, y2)
    assert torch.equal(ws[: M * K // 2].view(M, K // 2), ac)


def test_linear_against_oracle():
    wl = synth.WORKLOADS["nvfp4_tiny"]
    a_cpu, w_cpu = wl.A(), wl.W()
    bias_cpu = synth.bf16_normal((wl.N,), 0.5, 77)
    a, w, bias = a_cpu.cuda(), w_cpu.cuda(), bias_cpu.cuda()
    wc, wsf, gw = prepared_weight(w)
    ga = bsp.nvfp4_global_scale(a)
    y = bsp.nvfp4_linear(a, ga, wc, wsf, gw, bias=bias)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    ga_r, gw_r = oracle.nvfp4_global_scale(a_cpu), oracle.nvfp4_global_scale(w_cpu)
    ac, asf = oracle.nvfp4_quantize(a_cpu, ga_r)
    wcr, wsfr = oracle.nvfp4_quantize(w_cpu, gw_r)
    b = bf16_bias_np(bias_cpu)
    Y = oracle.nvfp4_linear(ac, asf, ga_r, wcr, wsfr, gw_r, b)
    compare_gemm(y.cpu(), Y, nvfp4_dequant_rows(ac, asf, ga_r),
                 nvfp4_dequant_rows(wcr, wsfr, gw_r), b)


def test_linear_reuses_one_workspace():
    """Consecutive calls on one workspace with different activations: each result is
    that of its own input (the workspace is fully rewritten by every call)."""
    M, N, K = 512, 768, 1024
    w = synth.bf16_normal((N, K), 0.02, 301).cuda()
    wc, wsf, gw = prepared_weight(w)
    ws = torch.empty((bsp.nvfp4_linear_workspace_bytes(M, K),), dtype=torch.uint8, device="cuda")
    outs, refs = [], []
    for seed in (302, 303, 304):
        a = synth.bf16_normal((M, K), 1.0, seed).cuda()
        ga = bsp.nvfp4_global_scale(a)
        outs.append(bsp.nvfp4_linear(a, ga, wc, wsf, gw, workspace=ws))
        refs.append(two_calls(a, ga, wc, wsf, gw, None)[0])
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    for y, r in zip(outs, refs):
        assert torch.equal(y, r)
    assert not torch.equal(outs[0], outs[1])


def test_linear_rejects_small_workspace():
    M, N, K = 128, 128, 256
    a = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((bsp.nvfp4_sf_bytes(N, K),), dtype=torch.uint8, device="cuda")
    g = torch.ones((1,), dtype=torch.float32, device="cuda")
    ws = torch.empty((bsp.nvfp4_linear_workspace_bytes(M, K) - 16,), dtype=torch.uint8,
                     device="cuda")
    with pytest.raises(bsp.BSPError):
        bsp.nvfp4_linear(a, g, w, sf, g, workspace=ws)


def test_linear_dynamic_scale():
    """The dynamic variant: g = amax(x)/2688 of this call's x (the oracle's value, bit
    for bit), and the output of nvfp4_linear with that g."""
    M, N, K = 300, 512, 1024
    a_cpu = synth.bf16_normal((M, K), 1.0, 400, 0.01, 20.0)
    a = a_cpu.cuda()
    w = synth.bf16_normal((N, K), 0.02, 401).cuda()
    wc, wsf, gw = prepared_weight(w)
    y, g = bsp.nvfp4_linear_dynamic(a, wc, wsf, gw)
    ref = bsp.nvfp4_linear(a, bsp.nvfp4_global_scale(a), wc, wsf, gw)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    assert g.item() == float(oracle.nvfp4_global_scale(a_cpu))
    assert torch.equal(y, ref)
    # a second call on a scaled input recomputes g
    y2, g2 = bsp.nvfp4_linear_dynamic(a * 4, wc, wsf, gw)
    torch.cuda.synchronize()
    assert g2.item() == 4 * g.item()


@pytest.mark.parametrize("kernel", [1, 2])        # grid-stride / staged quantizer
@pytest.mark.parametrize("M,N,K", [(300, 512, 1024), (1, 8, 64), (4096, 256, 3072)])
def test_linear_dynamic_scale_both_quantizer_kernels(kernel, M, N, K):
    """Both quantizer kernels reduce the per-CTA maxima of the amax pass themselves and
    publish g: g is the oracle's value bit for bit, and the output equals nvfp4_linear with
    the separately computed scale."""
    old = bsp.bsp_testing_set_quant_kernel(kernel)
    try:
        a_cpu = synth.bf16_normal((M, K), 1.0, 410 + M, 0.01, 20.0)
        a = a_cpu.cuda()
        w = synth.bf16_normal((N, K), 0.02, 411).cuda()
        wc, wsf, gw = prepared_weight(w)
        y, g = bsp.nvfp4_linear_dynamic(a, wc, wsf, gw)
        ref = bsp.nvfp4_linear(a, bsp.nvfp4_global_scale(a), wc, wsf, gw)
        torch.cuda.synchronize()
        assert bsp.bsp_last_device_status() == 0
        assert g.item() == float(oracle.nvfp4_global_scale(a_cpu))
        assert torch.equal(y, ref)
    finally:
        bsp.bsp_testing_set_quant_kernel(old)


@pytest.mark.parametrize("kernel", [1, 2])
def test_linear_dynamic_all_zero_activations(kernel):
    """amax = 0 gives g = 0: every activation code and block scale is zero, the product
    vanishes (alpha = 0) and the output is the bias, exactly."""
    old = bsp.bsp_testing_set_quant_kernel(kernel)
    try:
        M, N, K = 256, 384, 512
        a = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
        w = synth.bf16_normal((N, K), 0.02, 420).cuda()
        b = synth.bf16_normal((N,), 0.1, 421).cuda()
        wc, wsf, gw = prepared_weight(w)
        y, g = bsp.nvfp4_linear_dynamic(a, wc, wsf, gw, bias=b)
        torch.cuda.synchronize()
        assert bsp.bsp_last_device_status() == 0
        assert g.item() == 0.0
        assert torch.equal(y, b.expand(M, N))
    finally:
        bsp.bsp_testing_set_quant_kernel(old)
