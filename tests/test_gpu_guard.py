"""Guard bands around every output: ragged shapes must not write outside their buffers.

Each output tensor is a contiguous slice in the middle of a larger buffer filled with a
sentinel; after the call the bytes on both sides must still hold the sentinel.  Run on
both GEMM kernels and both quantizer kernels, at shapes whose M, N and K are not
multiples of the tiles (the pages fix no shapes; these are the tails the kernels mask).
"""
import pytest
import torch

import synth
import block_scaled_precision_act_b200 as bsp

pytestmark = pytest.mark.gpu

GUARD = 4096            # bytes on each side, a multiple of 16
SENT = 0xA7


class Guarded:
    def __init__(self, nbytes):
        self.n = nbytes
        self.buf = torch.full((GUARD + nbytes + GUARD,), SENT, dtype=torch.uint8, device="cuda")

    def view(self, dtype, shape):
        return self.buf[GUARD:GUARD + self.n].view(dtype).view(shape)

    def intact(self):
        return bool((self.buf[:GUARD] == SENT).all()) and bool((self.buf[GUARD + self.n:] == SENT).all())


@pytest.fixture(params=[(1, 1), (2, 2)], ids=["pair+grid", "single+staged"], autouse=True)
def kernels(request):
    g, q = request.param
    old_g = bsp.bsp_testing_set_gemm_kernel(g)
    old_q = bsp.bsp_testing_set_quant_kernel(q)
    yield
    bsp.bsp_testing_set_gemm_kernel(old_g)
    bsp.bsp_testing_set_quant_kernel(old_q)


@pytest.mark.parametrize("M,N,K", [(200, 136, 320), (1, 8, 64), (130, 264, 1216), (257, 520, 192)])
def test_nvfp4_outputs_stay_in_bounds(M, N, K):
    a = synth.bf16_normal((M, K), 1.0, 700).cuda()
    w = synth.bf16_normal((N, K), 0.02, 701).cuda()
    bias = synth.bf16_normal((N,), 0.5, 702).cuda()
    ga, gw = bsp.nvfp4_global_scale(a), bsp.nvfp4_global_scale(w)
    ac_g = Guarded(M * K // 2)
    asf_g = Guarded(bsp.nvfp4_sf_bytes(M, K, bsp.SF_MMA))
    ac, asf = bsp.nvfp4_quantize_act(a, ga, codes=ac_g.view(torch.uint8, (M, K // 2)),
                                     scales=asf_g.view(torch.uint8, (-1,)))
    wc, wsf = bsp.nvfp4_quantize_act(w, gw)
    y_g = Guarded(M * N * 2)
    bsp.nvfp4_gemm(ac, asf, ga, wc, wsf, gw, bias=bias, out=y_g.view(torch.bfloat16, (M, N)))
    lin_g = Guarded(bsp.nvfp4_linear_workspace_bytes(M, K))
    y2_g = Guarded(M * N * 2)
    bsp.nvfp4_linear(a, ga, wc, wsf, gw, bias=bias, out=y2_g.view(torch.bfloat16, (M, N)),
                     workspace=lin_g.view(torch.uint8, (-1,)))
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    for name, g in [("codes", ac_g), ("scales", asf_g), ("gemm out", y_g), ("linear workspace", lin_g),
                    ("linear out", y2_g)]:
        assert g.intact(), name


@pytest.mark.parametrize("M,N,K", [(200, 320, 320), (1, 64, 64), (257, 576, 192)])
def test_gemm_quant_outputs_stay_in_bounds(M, N, K):
    a = synth.bf16_normal((M, K), 1.0, 710).cuda()
    w = synth.bf16_normal((N, K), 0.02, 711).cuda()
    ga, gw = bsp.nvfp4_global_scale(a), bsp.nvfp4_global_scale(w)
    ac, asf = bsp.nvfp4_quantize_act(a, ga)
    wc, wsf = bsp.nvfp4_quantize_act(w, gw)
    g_out = torch.full((1,), 0.01, dtype=torch.float32, device="cuda")
    c_g = Guarded(M * N // 2)
    s_g = Guarded(bsp.nvfp4_sf_bytes(M, N, bsp.SF_MMA))
    bsp.nvfp4_gemm_quant(ac, asf, ga, wc, wsf, gw, g_out, out_codes=c_g.view(torch.uint8, (M, N // 2)),
                         out_sf=s_g.view(torch.uint8, (-1,)))
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    assert c_g.intact() and s_g.intact()


@pytest.mark.parametrize("M,N,K", [(200, 136, 320), (1, 8, 16), (300, 520, 384), (7, 24, 40000)])
def test_fp8r_outputs_stay_in_bounds(M, N, K):
    a = synth.bf16_normal((M, K), 1.0, 720).cuda()
    w = synth.bf16_normal((N, K), 0.02, 721).cuda()
    q_g = Guarded(M * K)
    s_g = Guarded(M * 4)
    aq, as_ = bsp.fp8r_quantize_rows(a, q=q_g.view(torch.uint8, (M, K)),
                                     row_scale=s_g.view(torch.float32, (M,)))
    wq, ws = bsp.fp8r_quantize_rows(w)
    y_g = Guarded(M * N * 2)
    if K % 16 == 0:
        bsp.fp8r_gemm(aq, as_, wq, ws, out=y_g.view(torch.bfloat16, (M, N)))
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    assert q_g.intact() and s_g.intact() and y_g.intact()
