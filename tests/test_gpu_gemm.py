"""GPU parity of the fused quantized linear against the fp64 oracle.

"BFL (fp8r / nvfp4)" (Diffusers quantization doc), Kernels table: the nvfp4 linear
quantizes activations and runs a block-scaled FP4 GEMM; fp8r runs a row-scaled FP8
GEMM.  The CUDA path and the oracle each run their whole path from the same seeded
bf16 tensors; codes and scales must agree bit for bit (checked again here) and the
outputs within the tolerances described in tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_precision_act_b200 as bsp
from parity import (bf16_bias_np, compare_gemm, fp8r_dequant_rows, nvfp4_dequant_rows,
                    sample_rows)

pytestmark = pytest.mark.gpu

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


@pytest.fixture(params=["pair", "single"], autouse=True)
def gemm_kernel(request):
    """Run every GEMM test on both kernels: CTA pairs (256x256 tiles, cta_group::2)
    and single CTAs (128-row tiles)."""
    old = bsp.bsp_testing_set_gemm_kernel({"pair": 1, "single": 2}[request.param])
    yield request.param
    bsp.bsp_testing_set_gemm_kernel(old)


# ------------------------------------------------------------------ NVFP4 path
def gpu_nvfp4_linear(a_cpu, w_cpu, bias_cpu=None):
    """Whole CUDA path: device global scales, both quantizers, the GEMM."""
    a, w = a_cpu.cuda(), w_cpu.cuda()
    ga = bsp.nvfp4_global_scale(a)
    gw = bsp.nvfp4_global_scale(w)
    wc, wsf = bsp.nvfp4_quantize_act(w, gw, layout=bsp.SF_MMA)      # offline weight prep
    ac, asf = bsp.nvfp4_quantize_act(a, ga, layout=bsp.SF_MMA)      # run-time activations
    bias = None if bias_cpu is None else bias_cpu.cuda()
    y = bsp.nvfp4_gemm(ac, asf, ga, wc, wsf, gw, bias=bias)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    return y.cpu(), ga.item(), gw.item(), ac.cpu().numpy()


def oracle_nvfp4_linear(a_cpu, w_cpu, bias_cpu, rows):
    ga = oracle.nvfp4_global_scale(a_cpu)
    gw = oracle.nvfp4_global_scale(w_cpu)
    a_rows = a_cpu[torch.from_numpy(rows)].contiguous()
    ac, asf = oracle.nvfp4_quantize(a_rows, ga)
    wc, wsf = oracle.nvfp4_quantize(w_cpu, gw)
    bias = bf16_bias_np(bias_cpu)
    Y = oracle.nvfp4_linear(ac, asf, ga, wc, wsf, gw, bias)
    return Y, ga, gw, ac, nvfp4_dequant_rows(ac, asf, ga), nvfp4_dequant_rows(wc, wsf, gw), bias


def check_nvfp4(a_cpu, w_cpu, bias_cpu=None, step=1):
    M = a_cpu.shape[0]
    rows = sample_rows(M, step)
    y, ga, gw, ac_gpu = gpu_nvfp4_linear(a_cpu, w_cpu, bias_cpu)
    Y, ga_r, gw_r, ac_ref, A_hat, W_hat, bias = oracle_nvfp4_linear(a_cpu, w_cpu, bias_cpu, rows)
    assert ga == float(ga_r) and gw == float(gw_r)
    assert np.array_equal(ac_gpu[rows], ac_ref)
    return compare_gemm(y[torch.from_numpy(rows)], Y, A_hat, W_hat, bias)


@pytest.mark.parametrize("M,N,K,seed", [
    (128, 256, 256, 0),      # the tiny workload's shape
    (128, 128, 64, 1),       # one MMA K-step
    (256, 384, 512, 2),      # several tiles, N tail of a 256-wide tile
    (200, 136, 320, 3),      # ragged M, N, and K not a multiple of the 256-wide stage
    (1, 8, 64, 4),           # degenerate: one row, one 8-column group
    (130, 264, 1216, 5),     # ragged everything, 19 K-blocks of 64
    (200, 136, 768, 6),      # 3 K-atoms of 128 bytes: the pair kernel's last stage is half empty
    (384, 512, 1280, 7),     # 5 K-atoms, N two full tiles
])
def test_nvfp4_linear_small(M, N, K, seed):
    a = synth.bf16_normal((M, K), 1.0, seed, 0.01, 20.0)
    w = synth.bf16_normal((N, K), 0.02, seed + 100)
    bias = synth.bf16_normal((N,), 0.1, seed + 200) if seed % 2 == 0 else None
    check_nvfp4(a, w, bias)


def test_nvfp4_bias_tiles_beyond_one_wave():
    """80 output tiles of 256 x 256 for the 74 CTA pairs of a B200: the first pairs take
    a second tile, which here is in the ragged last column of tiles (N = 2000), so the
    epilogue's bias columns fetched ahead for a later tile are checked, guard included."""
    a = synth.bf16_normal((2560, 256), 1.0, 71, 0.01, 20.0)
    w = synth.bf16_normal((2000, 256), 0.02, 171)
    bias = synth.bf16_normal((2000,), 0.1, 271)
    print("nvfp4 80 tiles", check_nvfp4(a, w, bias))


def test_nvfp4_tiny_workload():
    wl = synth.WORKLOADS["nvfp4_tiny"]
    stats = check_nvfp4(wl.A(), wl.W())
    print("tiny", stats)


def test_nvfp4_attn_1mp_sampled_rows():
    wl = synth.WORKLOADS["nvfp4_attn_1mp"]
    stats = check_nvfp4(wl.A(), wl.W(), wl.bias_vec(), step=61)
    print("attn_1mp", stats)


def test_nvfp4_mlp_up_and_down_sampled_rows():
    wl = synth.WORKLOADS["nvfp4_mlp_1mp"]
    print("mlp_up", check_nvfp4(wl.A(), wl.W(), step=127))
    print("mlp_down", check_nvfp4(wl.A2(), wl.W2(), step=127))


def test_nvfp4_4k_sampled_rows():
    wl = synth.WORKLOADS["nvfp4_4k"]
    print("4k", check_nvfp4(wl.A(), wl.W(), step=1021))


def test_nvfp4_mlp_chain_small():
    """GEMM1 -> global scale of its output -> re-quantize -> GEMM2, on 128 tokens.
    The oracle runs the same chain from the same bf16 inputs; its intermediate is the
    fp64 GEMM1 output rounded to bf16, so a few codes may differ from the GPU's (1-ulp
    bf16 differences in GEMM1); GEMM2 is checked within tolerance."""
    wl = synth.WORKLOADS["nvfp4_mlp_1mp"]
    a = wl.A()[:128].contiguous()
    w1, w2 = wl.W(), wl.W2()
    # CUDA path
    y1, _, _, _ = gpu_nvfp4_linear(a, w1)
    y2, _, _, _ = gpu_nvfp4_linear(y1, w2)
    # oracle path
    Y1, *_ = oracle_nvfp4_linear(a, w1, None, np.arange(128))
    y1_ref = torch.from_numpy(Y1.astype(np.float32)).to(torch.bfloat16)
    mism = (y1_ref.view(torch.int16) != y1.view(torch.int16)).float().mean().item()
    assert mism < 0.05, mism
    Y2, _, _, _, A_hat, W_hat, _ = oracle_nvfp4_linear(y1_ref, w2, None, np.arange(128))
    stats = compare_gemm(y2, Y2, A_hat, W_hat)
    print("chain", stats, "intermediate bf16 mismatch", mism)


def test_nvfp4_integer_valued_exact():
    """On-grid E2M1 values with every scale 1 and global scales 1: the sums are
    multiples of 1/4 well inside fp32, so the output is exactly bf16(Y_ref)."""
    rng = np.random.default_rng(11)
    M, N, K = 256, 256, 256
    ia = rng.integers(0, 16, (M, K)).astype(np.uint8)
    iw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    pack = lambda c: (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    sf_a = oracle.sf_linear_to_mma(np.full((M, K // 16), 0x38, np.uint8), M, K)
    sf_w = oracle.sf_linear_to_mma(np.full((N, K // 16), 0x38, np.uint8), N, K)
    one = torch.ones((1,), dtype=torch.float32, device="cuda")
    y = bsp.nvfp4_gemm(torch.from_numpy(pack(ia)).cuda(), torch.from_numpy(sf_a).cuda(), one,
                       torch.from_numpy(pack(iw)).cuda(), torch.from_numpy(sf_w).cuda(), one)
    va = np.where(ia & 8, -1.0, 1.0) * E2M1[ia & 7]
    vw = np.where(iw & 8, -1.0, 1.0) * E2M1[iw & 7]
    ref = torch.from_numpy((va @ vw.T).astype(np.float32)).to(torch.bfloat16)
    assert torch.equal(y.cpu(), ref)


@pytest.mark.parametrize("k0", [0, 1, 2, 15, 16, 17, 63, 64, 65, 127, 200, 255])
def test_nvfp4_single_hot_nibble_and_scale_layout(k0):
    """One nonzero code in A at (m0, k0) with its block scale set to 2: exactly row m0
    of Y changes, by 2 * e2m1(a) * e2m1(W[n, k0]) * scale of W's block."""
    M, N, K = 256, 256, 256
    rng = np.random.default_rng(k0)
    m0 = int(rng.integers(0, M))
    ia = np.zeros((M, K), np.uint8)
    ia[m0, k0] = 0x3                                   # +1.5
    iw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sfa_lin = np.full((M, K // 16), 0x38, np.uint8)     # 1.0
    sfa_lin[m0, k0 // 16] = 0x40                        # 2.0
    sfw_lin = rng.integers(0x30, 0x48, (N, K // 16)).astype(np.uint8)
    pack = lambda c: (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    one = torch.ones((1,), dtype=torch.float32, device="cuda")
    y = bsp.nvfp4_gemm(torch.from_numpy(pack(ia)).cuda(),
                       torch.from_numpy(oracle.sf_linear_to_mma(sfa_lin, M, K)).cuda(), one,
                       torch.from_numpy(pack(iw)).cuda(),
                       torch.from_numpy(oracle.sf_linear_to_mma(sfw_lin, N, K)).cuda(), one)
    y = y.float().cpu().numpy()
    vw = np.where(iw[:, k0] & 8, -1.0, 1.0) * E2M1[iw[:, k0] & 7]
    sw = np.array([oracle.e4m3_decode(int(b)) for b in sfw_lin[:, k0 // 16]])
    expect = 2.0 * 1.5 * vw * sw
    assert np.array_equal(np.delete(y, m0, axis=0), np.zeros((M - 1, N)))
    ref = torch.from_numpy(expect.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(y[m0], ref)


def test_nvfp4_single_hot_weight_rows():
    """One nonzero code in W at (n0, k0) for several n0 (both 128-row halves of a
    256-wide tile and the second N tile): exactly column n0 of Y changes."""
    M, N, K = 128, 512, 128
    rng = np.random.default_rng(5)
    ia = rng.integers(0, 16, (M, K)).astype(np.uint8)
    sfa_lin = rng.integers(0x30, 0x48, (M, K // 16)).astype(np.uint8)
    pack = lambda c: (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    one = torch.ones((1,), dtype=torch.float32, device="cuda")
    a_c = torch.from_numpy(pack(ia)).cuda()
    a_s = torch.from_numpy(oracle.sf_linear_to_mma(sfa_lin, M, K)).cuda()
    for n0, k0 in [(0, 0), (31, 5), (127, 64), (128, 1), (200, 99), (255, 127), (300, 77),
                   (511, 126)]:
        iw = np.zeros((N, K), np.uint8)
        iw[n0, k0] = 0xC                                # -2.0
        sfw_lin = np.full((N, K // 16), 0x38, np.uint8)
        sfw_lin[n0, k0 // 16] = 0x30                    # 0.5
        y = bsp.nvfp4_gemm(a_c, a_s, one, torch.from_numpy(pack(iw)).cuda(),
                           torch.from_numpy(oracle.sf_linear_to_mma(sfw_lin, N, K)).cuda(), one)
        y = y.float().cpu().numpy()
        va = np.where(ia[:, k0] & 8, -1.0, 1.0) * E2M1[ia[:, k0] & 7]
        sa = np.array([oracle.e4m3_decode(int(b)) for b in sfa_lin[:, k0 // 16]])
        expect = -2.0 * 0.5 * va * sa
        assert np.array_equal(np.delete(y, n0, axis=1), np.zeros((M, N - 1))), (n0, k0)
        ref = torch.from_numpy(expect.astype(np.float32)).to(torch.bfloat16).float().numpy()
        assert np.array_equal(y[:, n0], ref), (n0, k0)


# ------------------------------------------------------------------ fp8r path
def check_fp8r(a_cpu, w_cpu, bias_cpu=None, step=1):
    M = a_cpu.shape[0]
    rows = sample_rows(M, step)
    a, w = a_cpu.cuda(), w_cpu.cuda()
    wq, ws = bsp.fp8r_quantize_rows(w)
    aq, as_ = bsp.fp8r_quantize_rows(a)
    y = bsp.fp8r_gemm(aq, as_, wq, ws, bias=None if bias_cpu is None else bias_cpu.cuda())
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    a_rows = a_cpu[torch.from_numpy(rows)].contiguous()
    aq_r, as_r = oracle.fp8r_quantize(a_rows)
    wq_r, ws_r = oracle.fp8r_quantize(w_cpu)
    assert np.array_equal(aq.cpu().numpy()[rows], aq_r)
    assert np.array_equal(ws.cpu().numpy(), ws_r)
    bias = bf16_bias_np(bias_cpu)
    Y = oracle.fp8r_linear(aq_r, as_r, wq_r, ws_r, bias)
    return compare_gemm(y.cpu()[torch.from_numpy(rows)], Y, fp8r_dequant_rows(aq_r, as_r),
                        fp8r_dequant_rows(wq_r, ws_r), bias)


@pytest.mark.parametrize("M,N,K,seed", [
    (128, 256, 256, 0), (128, 128, 32, 1), (200, 136, 336, 2), (1, 8, 16, 3),
    (300, 520, 1040, 4), (300, 520, 384, 5), (260, 264, 640, 6),
])
def test_fp8r_linear_small(M, N, K, seed):
    a = synth.bf16_normal((M, K), 1.0, seed, 0.01, 20.0)
    w = synth.bf16_normal((N, K), 0.02, seed + 100)
    bias = synth.bf16_normal((N,), 0.1, seed + 200) if seed % 2 == 0 else None
    check_fp8r(a, w, bias)


def test_fp8r_bias_tiles_beyond_one_wave():
    """As the NVFP4 case: 80 tiles for 74 pairs, the later tiles in the ragged last
    column of tiles, with bias; the row scales of a pair's next tile are fetched ahead."""
    a = synth.bf16_normal((2560, 256), 1.0, 72, 0.01, 20.0)
    w = synth.bf16_normal((2000, 256), 0.02, 172)
    bias = synth.bf16_normal((2000,), 0.1, 272)
    print("fp8r 80 tiles", check_fp8r(a, w, bias))


@pytest.mark.parametrize("M", synth.FP8R_M_SWEEP)
def test_fp8r_sweep_sampled_rows(M):
    wl = synth.WORKLOADS["fp8r_1mp"]
    print("fp8r", M, check_fp8r(wl.A_rows(M), wl.W(), step=max(1, M // 64)))


def test_fp8r_integer_valued_exact():
    rng = np.random.default_rng(12)
    M, N, K = 128, 256, 128
    vals = np.array([0x38, 0x40, 0x44, 0xB8, 0xC0, 0x30, 0x00], np.uint8)  # 1,2,3,-1,-2,.5,0
    qa = vals[rng.integers(0, len(vals), (M, K))]
    qw = vals[rng.integers(0, len(vals), (N, K))]
    one_a = torch.ones((M,), dtype=torch.float32, device="cuda")
    one_w = torch.ones((N,), dtype=torch.float32, device="cuda")
    y = bsp.fp8r_gemm(torch.from_numpy(qa).cuda(), one_a, torch.from_numpy(qw).cuda(), one_w)
    ref = oracle.e4m3_decode_array(qa) @ oracle.e4m3_decode_array(qw).T
    assert torch.equal(y.cpu(), torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16))


# ------------------------------------------------------------------ edge cases
def test_zero_sized_gemms_are_noops():
    e = torch.empty((0,), dtype=torch.uint8, device="cuda")
    one = torch.ones((1,), dtype=torch.float32, device="cuda")
    assert bsp.lib().nvfp4_gemm(None, None, one.data_ptr(), None, None, one.data_ptr(), None,
                                None, 0, 128, 256, None) == 0
    assert bsp.lib().fp8r_gemm(None, None, None, None, None, None, 128, 0, 256, None) == 0
    del e
    torch.cuda.synchronize()


def test_bounded_wait_times_out_and_context_survives():
    """The producer stops after one stage; the MMA thread's wait on the next stage can
    never complete.  The kernel must report BSP_ERR_TIMEOUT within its limit, free its
    resources, and leave the context usable (a normal GEMM runs right after)."""
    M, N, K = 128, 256, 1024
    a = synth.bf16_normal((M, K), 1.0, 7)
    w = synth.bf16_normal((N, K), 0.02, 8)
    ad, wd = a.cuda(), w.cuda()
    ga, gw = bsp.nvfp4_global_scale(ad), bsp.nvfp4_global_scale(wd)
    ac, asf = bsp.nvfp4_quantize_act(ad, ga)
    wc, wsf = bsp.nvfp4_quantize_act(wd, gw)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert bsp.bsp_last_device_status() == 0
    st = bsp.bsp_testing_gemm_stall(1, ac, asf, ga, wc, wsf, gw, out, K, 1, 200)
    assert st == 0
    assert bsp.bsp_last_device_status() == -6
    assert bsp.bsp_last_device_status() == 0            # cleared on read
    # the fp8r kernel's waits are bounded the same way
    aq, as_ = bsp.fp8r_quantize_rows(ad)
    wq, ws = bsp.fp8r_quantize_rows(wd)
    assert bsp.bsp_testing_gemm_stall(0, aq, None, as_, wq, None, ws, out, K, 2, 200) == 0
    assert bsp.bsp_last_device_status() == -6
    # the same context still computes correct results
    y = bsp.nvfp4_gemm(ac, asf, ga, wc, wsf, gw)
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
    ref = check_nvfp4(a, w)
    assert ref["max_norm_err"] < 1e-2
    assert torch.isfinite(y.float()).all()
