"""GPU checks of fp8r_linear: the fp8r linear in one call.

"BFL (fp8r / nvfp4)" (Diffusers quantization doc), fp8r bullet and Kernels table:
activations quantized to E4M3 per row at run time, then the row-scaled FP8 GEMM.  The
codes it leaves in the workspace must equal the oracle's bit for bit, the output must
meet the oracle within the tolerances of tests/parity.py and equal fp8r_quantize_rows +
fp8r_gemm bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_precision_act_b200 as bsp
from parity import bf16_bias_np, compare_gemm, fp8r_dequant_rows, sample_rows

pytestmark = pytest.mark.gpu


def run(M, N, K, seed, with_bias):
    a_cpu = synth.bf16_normal((M, K), 1.0, seed, 0.005, 30.0)
    w_cpu = synth.bf16_normal((N, K), 0.02, seed + 1)
    bias_cpu = synth.bf16_normal((N,), 0.5, seed + 2) if with_bias else None
    a, w = a_cpu.cuda(), w_cpu.cuda()
    bias = None if bias_cpu is None else bias_cpu.cuda()
    wq, ws = bsp.fp8r_quantize_rows(w)
    work = torch.full((bsp.fp8r_linear_workspace_bytes(M, K),), 0x3C, dtype=torch.uint8,
                      device="cuda")
    y = bsp.fp8r_linear(a, wq, ws, bias=bias, workspace=work)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    return a_cpu, w_cpu, bias_cpu, a, wq, ws, bias, work, y


@pytest.mark.parametrize("M,N,K,seed,with_bias", [
    (256, 3072, 3072, 600, True),     # the sweep's smallest M
    (1024, 3072, 3072, 610, False),
    (200, 1000, 1024, 620, True),     # ragged M and N
    (1, 64, 256, 630, False),         # one row
    (300, 520, 384, 640, True),       # ragged, 3 K-stages
])
def test_fp8r_linear_against_oracle(M, N, K, seed, with_bias):
    a_cpu, w_cpu, bias_cpu, a, wq, ws, bias, work, y = run(M, N, K, seed, with_bias)
    rows = sample_rows(M, 1 if M <= 512 else 5)
    aq_r, as_r = oracle.fp8r_quantize(a_cpu)
    wq_r, ws_r = oracle.fp8r_quantize(w_cpu)
    # the quantized activations in the workspace: codes bit for bit
    assert np.array_equal(work[: M * K].view(M, K).cpu().numpy(), aq_r)
    b = bf16_bias_np(bias_cpu)
    Y = oracle.fp8r_linear(aq_r[rows], as_r[rows], wq_r, ws_r, b)
    compare_gemm(y.cpu()[torch.from_numpy(rows)], Y, fp8r_dequant_rows(aq_r[rows], as_r[rows]),
                 fp8r_dequant_rows(wq_r, ws_r), b)


@pytest.mark.parametrize("M", [256, 4096])
def test_fp8r_linear_equals_two_calls(M):
    N, K = 3072, 3072
    a = synth.bf16_normal((M, K), 1.0, 650 + M).cuda()
    w = synth.bf16_normal((N, K), 0.02, 651).cuda()
    bias = synth.bf16_normal((N,), 0.5, 652).cuda()
    wq, ws = bsp.fp8r_quantize_rows(w)
    y = bsp.fp8r_linear(a, wq, ws, bias=bias)
    aq, as_ = bsp.fp8r_quantize_rows(a)
    ref = bsp.fp8r_gemm(aq, as_, wq, ws, bias=bias)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    assert torch.equal(y, ref)
