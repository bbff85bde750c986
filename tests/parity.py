"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on the
same seeded bf16 inputs and compare.

Tolerance of the GEMM outputs (both asserted):
  (1) the stated one: |Y - Y_ref| / (||A_m|| ||W_n|| + |bias_n|) <= 1e-2, with A_m, W_n
      the dequantised rows including their global or row scales;
  (2) a tighter one derived from the arithmetic: bf16 rounding of the output
      (2^-9 relative, 2^-8 allowed) plus fp32 accumulation over K on the tensor cores,
      bounded by 2^-12 * sum_k |a_k w_k|.  A wrong scale on a single 16-element block
      or a swapped nibble moves Y by far more than this, while (1) alone would not see
      it at K = 3072.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_STATED = 1e-2
REL_OUT = 2.0 ** -8
REL_ACC = 2.0 ** -12


def sf_valid_mask(R: int, K: int) -> np.ndarray:
    ones = np.ones((R, K // 16), dtype=np.uint8)
    return oracle.sf_linear_to_mma(ones, R, K).astype(bool)


def compare_gemm(y_gpu: torch.Tensor, Y_ref: np.ndarray, A_hat: np.ndarray, W_hat: np.ndarray,
                 bias=None) -> dict:
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    assert y.shape == Y_ref.shape
    assert np.all(np.isfinite(y)), "non-finite output"
    b = np.zeros(Y_ref.shape[1]) if bias is None else np.abs(np.asarray(bias, np.float64))
    na = np.linalg.norm(A_hat, axis=1)
    nw = np.linalg.norm(W_hat, axis=1)
    diff = np.abs(y - Y_ref)
    denom = na[:, None] * nw[None, :] + b[None, :]
    err = diff / np.where(denom > 0, denom, 1.0)
    S = np.abs(A_hat) @ np.abs(W_hat).T
    bound = REL_OUT * np.abs(Y_ref) + REL_ACC * S + 2.0 ** -9 * b[None, :] + 1e-30
    stats = {"max_norm_err": float(err.max()), "max_ratio_to_bound": float((diff / bound).max())}
    assert stats["max_norm_err"] <= TOL_STATED, stats
    assert np.all(diff <= bound), stats
    return stats


def nvfp4_dequant_rows(codes, sf_lin, g) -> np.ndarray:
    return oracle.nvfp4_dequant(codes, sf_lin, float(g))


def fp8r_dequant_rows(q, s) -> np.ndarray:
    return oracle.e4m3_decode_array(q) * np.asarray(s, np.float64)[:, None]


def sample_rows(M: int, step: int) -> np.ndarray:
    rows = np.arange(0, M, step)
    if rows[-1] != M - 1:
        rows = np.append(rows, M - 1)
    return rows


def bf16_bias_np(bias_t):
    return None if bias_t is None else bias_t.float().numpy().astype(np.float64)
