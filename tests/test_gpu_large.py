"""The largest inputs: the activation quantizer past 2^31 blocks of 16 elements, and the
GEMM over those rows.

Both quantizer kernels find a block's row with 32-bit arithmetic (a multiply-high by the
blocks per row) while every block index of the launch stays below 2^31, and by 64-bit
division beyond.  An input of 2^21 + 64 rows of K = 16384 (1024 blocks per row, so
2^31 + 65536 blocks, 64 GiB of bf16) takes the 64-bit path; row 2^21 starts exactly at
block 2^31.  Rows on both sides of it must match the oracle bit for bit (codes, and the
MMA-layout scale bytes at the offsets the oracle's index function gives), and the GEMM's
outputs on those rows must meet the oracle within the tolerances of tests/parity.py.
It needs about 95 GB of free device memory and skips when less is free.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_precision_act_b200 as bsp
from parity import compare_gemm, nvfp4_dequant_rows

pytestmark = pytest.mark.gpu

K = 16384
M = (1 << 31) // (K // 16) + 64
ROWS = [0, 1, (1 << 21) - 2, (1 << 21) - 1, 1 << 21, (1 << 21) + 1, M - 64, M - 1]
G = np.float32(8.0 / 2688.0)          # decode-side global scale for |x| up to 8


@pytest.fixture(scope="module")
def big_input():
    free, _ = torch.cuda.mem_get_info()
    need = M * K * 2 + M * K // 2 + bsp.nvfp4_sf_bytes(M, K) + M * 256 * 2 + (4 << 30)
    if free < need:
        pytest.skip(f"needs {need / 1e9:.0f} GB of free device memory, {free / 1e9:.0f} free")
    gen = torch.Generator(device="cuda").manual_seed(2024)
    x = torch.randn((M, K), dtype=torch.bfloat16, device="cuda", generator=gen)
    rows = torch.tensor(ROWS, device="cuda")
    yield x, rows, x[rows].cpu()
    del x
    torch.cuda.empty_cache()


def gather_mma_scales(sf: torch.Tensor, rows) -> np.ndarray:
    """Scale bytes of `rows` ([len(rows), K/16], linear order) from an MMA-layout array."""
    idx = [oracle.sf_mma_offset(r, kb, K) for r in rows for kb in range(K // 16)]
    got = sf[torch.tensor(idx, device=sf.device)].cpu().numpy()
    return got.reshape(len(rows), K // 16)


@pytest.mark.parametrize("kernel", [1, 2])        # grid-stride / staged quantizer
def test_quantizer_past_2_31_blocks(big_input, kernel):
    x, rows, x_rows = big_input
    g = torch.tensor([G], device="cuda")
    old = bsp.bsp_testing_set_quant_kernel(kernel)
    try:
        codes, sf = bsp.nvfp4_quantize_act(x, g, layout=bsp.SF_MMA)
        torch.cuda.synchronize()
    finally:
        bsp.bsp_testing_set_quant_kernel(old)
    assert bsp.bsp_last_device_status() == 0
    rc, rsf = oracle.nvfp4_quantize(x_rows, G)
    assert np.array_equal(codes[rows].cpu().numpy(), rc)
    assert np.array_equal(gather_mma_scales(sf, ROWS), rsf)
    del codes, sf
    torch.cuda.empty_cache()


def test_gemm_over_2_31_blocks_of_activations(big_input):
    x, rows, x_rows = big_input
    N = 256
    w_cpu = synth.bf16_normal((N, K), 0.02, 2025)
    gw = oracle.nvfp4_global_scale(w_cpu)
    wcr, wsfr = oracle.nvfp4_quantize(w_cpu, gw)
    g = torch.tensor([G], device="cuda")
    gw_t = torch.tensor([gw], device="cuda")
    wc, wsf = bsp.nvfp4_quantize_act(w_cpu.cuda(), gw_t, layout=bsp.SF_MMA)
    codes, sf = bsp.nvfp4_quantize_act(x, g, layout=bsp.SF_MMA)
    y = bsp.nvfp4_gemm(codes, sf, g, wc, wsf, gw_t)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    rc, rsf = oracle.nvfp4_quantize(x_rows, G)
    Y = oracle.nvfp4_linear(rc, rsf, G, wcr, wsfr, gw)
    compare_gemm(y[rows].cpu(), Y, nvfp4_dequant_rows(rc, rsf, G),
                 nvfp4_dequant_rows(wcr, wsfr, gw))
    del codes, sf, y
    torch.cuda.empty_cache()
