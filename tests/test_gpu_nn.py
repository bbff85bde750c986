"""GPU checks of QuantLinear: its forward is the library's linear (bit-identical to the
direct calls), it round-trips through its state dict, and it meets the oracle.

"BFL (fp8r / nvfp4)" (Diffusers quantization doc), format bullets and Kernels table.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_precision_act_b200 as bsp
from block_scaled_precision_act_b200.nn import QuantLinear
from parity import bf16_bias_np, compare_gemm, fp8r_dequant_rows, nvfp4_dequant_rows

pytestmark = pytest.mark.gpu


def bf16_linear(K, N, seed, bias=True):
    lin = torch.nn.Linear(K, N, bias=bias)
    with torch.no_grad():
        lin.weight.copy_(synth.bf16_normal((N, K), 0.02, seed).float())
        if bias:
            lin.bias.copy_(synth.bf16_normal((N,), 0.5, seed + 1).float())
    return lin.to(torch.bfloat16).cuda()


def test_nvfp4_forward_equals_direct_calls_and_oracle():
    K, N = 3072, 1024
    lin = bf16_linear(K, N, 40)
    x = synth.bf16_normal((2, 300, K), 1.0, 41, 0.005, 30.0).cuda()     # [B, T, K]
    m = QuantLinear.from_linear(lin, "nvfp4", calibration=x)
    y = m(x)
    assert y.shape == (2, 300, N) and y.dtype == torch.bfloat16
    # the same forward through the library's entry points
    x2 = x.reshape(-1, K)
    W = lin.weight.detach()
    gw = bsp.nvfp4_global_scale(W)
    wc, wsf = bsp.nvfp4_quantize_act(W, gw, layout=bsp.SF_MMA)
    ref = bsp.nvfp4_linear(x2, m.input_scale.view(1), wc, wsf, gw, bias=m.bias)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    assert torch.equal(y.reshape(-1, N), ref)
    # and against the oracle on every 7th row
    rows = np.arange(0, x2.shape[0], 7)
    xs = x2.cpu()[torch.from_numpy(rows)].contiguous()
    ga = np.float32(m.input_scale.item())
    ac, asf = oracle.nvfp4_quantize(xs, ga)
    gw_r = oracle.nvfp4_global_scale(W.cpu())
    wcr, wsfr = oracle.nvfp4_quantize(W.cpu(), gw_r)
    b = bf16_bias_np(m.bias.cpu())
    Y = oracle.nvfp4_linear(ac, asf, ga, wcr, wsfr, gw_r, b)
    compare_gemm(y.reshape(-1, N).cpu()[torch.from_numpy(rows)], Y,
                 nvfp4_dequant_rows(ac, asf, ga), nvfp4_dequant_rows(wcr, wsfr, gw_r), b)


def test_fp8r_forward_against_oracle():
    K, N = 3072, 1024
    lin = bf16_linear(K, N, 50, bias=False)
    m = QuantLinear.from_linear(lin, "fp8r")
    x = synth.bf16_normal((257, K), 1.0, 51).cuda()
    y = m(x)
    torch.cuda.synchronize()
    aq, as_ = oracle.fp8r_quantize(x.cpu())
    wq, ws = oracle.fp8r_quantize(lin.weight.detach().cpu())
    Y = oracle.fp8r_linear(aq, as_, wq, ws)
    compare_gemm(y.cpu(), Y, fp8r_dequant_rows(aq, as_), fp8r_dequant_rows(wq, ws))


@pytest.mark.parametrize("scheme", ["nvfp4", "fp8r"])
def test_state_dict_round_trip(scheme):
    K, N = 1024, 512
    lin = bf16_linear(K, N, 60)
    x = synth.bf16_normal((129, K), 1.0, 61).cuda()
    m = QuantLinear.from_linear(lin, scheme, input_scale=0.01)
    y = m(x)
    sd = {k: v.cpu() for k, v in m.state_dict().items()}
    m2 = QuantLinear.from_state_dict(sd, device="cuda")
    assert m2.scheme == scheme
    m3 = QuantLinear(K, N, scheme).cuda()
    m3(x)                                      # builds the scale copy for the zero weights
    m3.load_state_dict(m.state_dict())         # the copy is rebuilt after a load
    torch.cuda.synchronize()
    assert torch.equal(m2(x), y) and torch.equal(m3(x), y)
