"""Pins for the oracle's fp64 GEMMs (CPU only).

"BFL (fp8r / nvfp4)", Kernels table: the NVFP4 path is a block-scaled GEMM on
quantized activations and weights; the fp8r path is a row-scaled FP8 GEMM.  The
oracle sums dequantised products in fp64.  Here it is checked against brute-force
exactly-rounded sums (math.fsum) on tiny inputs, against numpy's independent fp64
matmul, and on integer-valued cases where every method must agree exactly.
"""
import math

import numpy as np
import pytest

import oracle
import synth

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def decode_nvfp4(codes, sf_lin):
    """Independent decode: nibbles by hand, E4M3 from the bit formula."""
    R, K2 = codes.shape
    K = 2 * K2
    out = np.zeros((R, K))
    for r in range(R):
        for k in range(K):
            b = int(codes[r, k // 2])
            c = (b & 0xF) if k % 2 == 0 else (b >> 4)
            v = E2M1_GRID[c & 7] * (-1.0 if c & 8 else 1.0)
            sb = int(sf_lin[r, k // 16])
            e, m = (sb >> 3) & 15, sb & 7
            sd = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            out[r, k] = v * sd
    return out


@pytest.mark.parametrize("M,N,K", [(3, 5, 32), (4, 4, 64), (2, 7, 48)])
def test_nvfp4_linear_brute_force(M, N, K):
    a = synth.bf16_normal((M, K), 1.0, 100 + M, 0.05, 10.0)
    w = synth.bf16_normal((N, K), 0.02, 200 + N)
    bias = synth.bf16_normal((N,), 0.1, 300).float().numpy().astype(np.float64)
    ga, gw = oracle.nvfp4_global_scale(a), oracle.nvfp4_global_scale(w)
    ac, asf = oracle.nvfp4_quantize(a, ga)
    wc, wsf = oracle.nvfp4_quantize(w, gw)
    Y = oracle.nvfp4_linear(ac, asf, ga, wc, wsf, gw, bias)
    A = decode_nvfp4(ac, asf)
    W = decode_nvfp4(wc, wsf)
    alpha = float(ga) * float(gw)
    for m in range(M):
        for n in range(N):
            ref = alpha * math.fsum(A[m, k] * W[n, k] for k in range(K)) + bias[n]
            scale = alpha * math.fsum(abs(A[m, k] * W[n, k]) for k in range(K)) + abs(bias[n])
            assert abs(Y[m, n] - ref) <= 1e-14 * scale + 1e-300


def test_nvfp4_linear_matches_numpy_matmul():
    w_ = synth.WORKLOADS["nvfp4_tiny"]
    a, w = w_.A(), w_.W()
    ga, gw = oracle.nvfp4_global_scale(a), oracle.nvfp4_global_scale(w)
    ac, asf = oracle.nvfp4_quantize(a, ga)
    wc, wsf = oracle.nvfp4_quantize(w, gw)
    Y = oracle.nvfp4_linear(ac, asf, ga, wc, wsf, gw)
    A = oracle.nvfp4_dequant(ac, asf, float(ga))
    W = oracle.nvfp4_dequant(wc, wsf, float(gw))
    ref = A @ W.T
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_integer_valued_gemm_is_exact():
    """All scales 1 (g = 1/6 * 6 ... chosen so sd = 1) and on-grid values: sums of
    products of E2M1 values are multiples of 1/4, exact in fp64 and fp32."""
    rng = np.random.default_rng(3)
    M, N, K = 4, 6, 64
    ia = rng.integers(0, 16, (M, K)).astype(np.uint8)
    iw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    ia[:, ::16] = 7
    iw[:, ::16] = 15                          # -6 in every block of W
    import torch
    xa = np.where(ia & 8, -1, 1) * E2M1_GRID[ia & 7]
    xw = np.where(iw & 8, -1, 1) * E2M1_GRID[iw & 7]
    ta = torch.from_numpy(xa.astype(np.float32)).to(torch.bfloat16)
    tw = torch.from_numpy(xw.astype(np.float32)).to(torch.bfloat16)
    g = np.float32(1.0)
    ac, asf = oracle.nvfp4_quantize(ta, g)
    wc, wsf = oracle.nvfp4_quantize(tw, g)
    assert np.all(asf == 0x38) and np.all(wsf == 0x38)
    Y = oracle.nvfp4_linear(ac, asf, g, wc, wsf, g)
    ref = np.array([[sum(int(4 * xa[m, k]) * int(4 * xw[n, k]) for k in range(K)) / 16.0
                     for n in range(N)] for m in range(M)])
    assert np.array_equal(Y, ref)


@pytest.mark.parametrize("M,N,K", [(3, 4, 32), (5, 2, 80)])
def test_fp8r_linear_brute_force(M, N, K):
    a = synth.bf16_normal((M, K), 1.0, 400 + M)
    w = synth.bf16_normal((N, K), 0.02, 500 + N)
    aq, as_ = oracle.fp8r_quantize(a)
    wq, ws = oracle.fp8r_quantize(w)
    bias = np.linspace(-0.3, 0.3, N)
    Y = oracle.fp8r_linear(aq, as_, wq, ws, bias)

    def dec(c):
        s, e, m = (c >> 7) & 1, (c >> 3) & 15, c & 7
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        return -v if s else v

    for m in range(M):
        for n in range(N):
            prods = [dec(int(aq[m, k])) * dec(int(wq[n, k])) for k in range(K)]
            ref = math.fsum(prods) * float(as_[m]) * float(ws[n]) + bias[n]
            scale = math.fsum(abs(p) for p in prods) * float(as_[m]) * float(ws[n]) + abs(bias[n])
            assert abs(Y[m, n] - ref) <= 1e-14 * scale


def test_gemm_f64_against_numpy_and_transpose_sensitivity():
    rng = np.random.default_rng(5)
    A = rng.standard_normal((7, 33))
    W = rng.standard_normal((9, 33))
    b = rng.standard_normal(9)
    Y = oracle.gemm_f64(A, W, b, alpha=0.5)
    assert np.allclose(Y, 0.5 * A @ W.T + b, rtol=1e-13, atol=1e-13)
    # a transposed operand (a plausible mistake) would not pass
    assert not np.allclose(Y[:7, :7], 0.5 * (W[:7] @ A.T[:, :7]) + b[:7])
