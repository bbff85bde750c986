"""GPU parity of the quantizers against the oracle: codes and scale bytes must be
bit-identical ("BFL (fp8r / nvfp4)", format bullets; the quantizer steps are the
ones written in include/bsp.h and in the oracle)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import block_scaled_precision_act_b200 as bsp
from parity import sf_valid_mask

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["grid", "staged"], autouse=True)
def quant_kernel(request):
    """Run every quantizer test on both NVFP4 quantizer kernels: the grid-stride one and
    the staged one (bulk copies into a shared-memory ring); the size-based default picks
    the staged kernel only for inputs of 96 M elements and more."""
    old = bsp.bsp_testing_set_quant_kernel({"grid": 1, "staged": 2}[request.param])
    yield request.param
    bsp.bsp_testing_set_quant_kernel(old)


def gpu_quant(x_cpu, g, layout):
    x = x_cpu.cuda()
    gd = torch.tensor([float(g)], dtype=torch.float32, device="cuda")
    codes, sf = bsp.nvfp4_quantize_act(x, gd, layout=layout)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), sf.cpu().numpy()


def assert_nvfp4_equal(x_cpu, g, layout):
    M, K = x_cpu.shape
    c_ref, s_ref = oracle.nvfp4_quantize(x_cpu, g)
    c, s = gpu_quant(x_cpu, g, layout)
    bad = np.argwhere(c != c_ref)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:4].tolist()}"
    if layout == bsp.SF_LINEAR:
        assert np.array_equal(s.reshape(M, K // 16), s_ref)
    else:
        ref = oracle.sf_linear_to_mma(s_ref, M, K)
        valid = sf_valid_mask(M, K)
        assert s.shape == ref.shape
        assert np.array_equal(s[valid], ref[valid])


@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("M,K,seed", [(128, 256, 0), (200, 320, 1), (1, 64, 2), (37, 1024, 3),
                                      (4096, 3072, 10), (4096, 12288, 24)])
def test_nvfp4_quantizer_bit_exact(M, K, seed, layout):
    x = synth.bf16_normal((M, K), 1.0, seed, 0.005, 30.0)
    g = oracle.nvfp4_global_scale(x)
    assert_nvfp4_equal(x, g, layout)


def test_nvfp4_quantizer_linear_layout_ragged_k():
    x = synth.bf16_normal((33, 48), 1.0, 5, 0.02, 10.0)
    assert_nvfp4_equal(x, oracle.nvfp4_global_scale(x), bsp.SF_LINEAR)


def special_blocks() -> np.ndarray:
    """Blocks that hit every E2M1 tie, both zero signs, small negatives, saturation,
    E4M3 scale ties, subnormal scales and all-zero blocks, under g = 2^-3."""
    rows = []
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5,
            -5.0, -0.0]
    # amax 0.75 -> s = 1 exactly, d = 2^-3 ; element value y*d
    rows.append([0.75] + [t / 8.0 for t in ties])
    rows.append([-0.75] + [t / 8.0 for t in ties[::-1]])
    rows.append([0.75, -0.0, 0.0, -0.01, 0.01, -0.03, 0.03, 0.0625, -0.0625, 0.7,
                 0.74, 0.6, -0.6, 0.5, 0.4, 0.3])
    # E4M3 scale ties: s = 1.0625 (-> 1.0) and s = 1.1875 (-> 1.25): amax = s * 0.75
    rows.append([1.0625 * 0.75] + [0.05 * i for i in range(15)])
    rows.append([1.1875 * 0.75] + [-0.05 * i for i in range(15)])
    # tiny block: subnormal E4M3 scale
    rows.append([1e-4 * (i - 7) for i in range(16)])
    rows.append([0.0] * 16)
    rows.append([-0.0] * 16)
    # saturating block: amax / (6g) > 448
    rows.append([500.0] + [37.5 * i for i in range(15)])
    return np.array(rows, dtype=np.float32)


def test_nvfp4_quantizer_special_values():
    blocks = special_blocks()                 # [9, 16]
    x = torch.from_numpy(np.tile(blocks.reshape(1, -1), (128, 4))).to(torch.bfloat16)
    assert x.shape == (128, 9 * 16 * 4)
    x = x[:, : (x.shape[1] // 64) * 64].contiguous()
    g = np.float32(2.0 ** -3)
    for layout in (bsp.SF_LINEAR, bsp.SF_MMA):
        assert_nvfp4_equal(x, g, layout)
    # g = 0: everything quantizes to zero
    assert_nvfp4_equal(x, np.float32(0.0), bsp.SF_LINEAR)


def test_nvfp4_quantizer_subnormal_and_infinite_inputs():
    """bf16 subnormal inputs (no flush to zero anywhere) and +-inf (the block scale
    saturates to 448, the infinite element to +-6)."""
    sub = np.float32(2.0 ** -130)                       # bf16 subnormal
    rows = [[sub * (i - 7) for i in range(16)],          # a block of subnormals only
            [np.inf] + [0.1 * i for i in range(15)],
            [-np.inf, 1.0, -2.0, 3.0] + [0.0] * 12,
            [sub, -sub, 1e-3, -1e-3] + [0.25 * i for i in range(12)]]
    blocks = np.array(rows, dtype=np.float32)
    x = torch.from_numpy(np.tile(blocks.reshape(1, -1), (64, 1))).to(torch.bfloat16)
    assert x.shape == (64, 64)
    for g in (np.float32(2.0 ** -3), np.float32(2.0 ** -140), np.float32(1.0)):
        for layout in (bsp.SF_LINEAR, bsp.SF_MMA):
            assert_nvfp4_equal(x, g, layout)
    # a tensor of subnormals only: its global scale is itself subnormal in binary32
    xs = torch.from_numpy(np.tile(blocks[:1], (128, 4))).to(torch.bfloat16)
    gs = oracle.nvfp4_global_scale(xs)
    assert 0.0 < float(gs) < 1.2e-38
    assert_nvfp4_equal(xs, gs, bsp.SF_MMA)


@pytest.mark.parametrize("M,K,seed", [(256, 3072, 30), (1000, 3072, 31), (4096, 3072, 32),
                                      (7, 24, 33), (64, 12288, 34), (3, 40000, 35)])
def test_fp8r_quantizer_bit_exact(M, K, seed):
    x = synth.bf16_normal((M, K), 1.0, seed, 0.01, 50.0)
    q_ref, s_ref = oracle.fp8r_quantize(x)
    q, s = bsp.fp8r_quantize_rows(x.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), s_ref)
    q = q.cpu().numpy()
    bad = np.argwhere(q != q_ref)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[:4].tolist()}"


def test_fp8r_quantizer_zero_and_special_rows():
    blocks = special_blocks()
    x = torch.from_numpy(np.tile(blocks, (1, 8))).to(torch.bfloat16)   # 9 rows x 128
    q_ref, s_ref = oracle.fp8r_quantize(x)
    q, s = bsp.fp8r_quantize_rows(x.cuda())
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("shape,seed", [((128, 256), 0), ((4096, 3072), 10), ((3, 8), 4),
                                        ((65536, 3072), 40)])
def test_global_scale_bit_exact(shape, seed):
    x = synth.bf16_normal(shape, 1.0, seed, 0.005, 30.0)
    g_ref = oracle.nvfp4_global_scale(x)
    g = bsp.nvfp4_global_scale(x.cuda())
    assert g.item() == float(g_ref)


@pytest.mark.parametrize("R,K", [(128, 256), (200, 320), (4096, 3072)])
def test_sf_convert_matches_oracle_layout(R, K):
    rng = np.random.default_rng(R + K)
    lin = rng.integers(0, 256, size=(R, K // 16), dtype=np.uint8)
    ref = oracle.sf_linear_to_mma(lin, R, K)
    src = torch.from_numpy(lin.reshape(-1)).cuda()
    mma = bsp.nvfp4_sf_convert(src, R, K, bsp.SF_LINEAR, bsp.SF_MMA)
    assert np.array_equal(mma.cpu().numpy(), ref)           # padding written as 0 too
    back = bsp.nvfp4_sf_convert(mma, R, K, bsp.SF_MMA, bsp.SF_LINEAR)
    assert np.array_equal(back.cpu().numpy().reshape(R, K // 16), lin)


def test_empty_inputs_are_noops():
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    g = torch.ones((1,), dtype=torch.float32, device="cuda")
    codes = torch.empty((0, 128), dtype=torch.uint8, device="cuda")
    sf = torch.empty((16,), dtype=torch.uint8, device="cuda")
    bsp.nvfp4_quantize_act(x, g, codes=codes, scales=sf)
    q, s = bsp.fp8r_quantize_rows(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"),
                                  q=torch.empty((16,), dtype=torch.uint8, device="cuda"),
                                  row_scale=torch.empty((4,), dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert bsp.bsp_last_device_status() == 0
