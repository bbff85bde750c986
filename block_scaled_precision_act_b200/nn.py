"""QuantLinear: the quantized linear as a torch module, with the checkpoint tensor names.

"BFL (fp8r / nvfp4)" (Diffusers quantization doc), format bullets: an nvfp4 linear
stores `weight` (E2M1 codes, two per byte), `weight_scale` (one E4M3 scale per 16
weights), `weight_scale_2` (fp32 global) and `input_scale` (fp32, calibrated for the
activations); an fp8r linear stores `weight` (E4M3) and one fp32 `weight_scale` per
row, and quantizes its activations per row at run time.  The scheme is read from the
tensors present, as that page's loader does.

The module only marshals: forward() is one nvfp4_linear call (activation quantizer +
FP4 GEMM) or fp8r_quantize_rows + fp8r_gemm, all in libbsp.so.  `weight_scale` is kept
in the checkpoint's row-major [N][K/16] layout (the state-dict form); the tensor-core
layout the GEMM reads is built from it on the device once and rebuilt after a load.
"""
from __future__ import annotations

import torch

from . import (SF_LINEAR, SF_MMA, BSPError, fp8r_gemm, fp8r_quantize_rows, nvfp4_global_scale,
               nvfp4_linear, nvfp4_linear_workspace_bytes, nvfp4_quantize_act, nvfp4_sf_convert)

__all__ = ["QuantLinear"]

_E4M3 = getattr(torch, "float8_e4m3fn", None)


def _u8(t: torch.Tensor) -> torch.Tensor:
    return t if t.dtype == torch.uint8 else t.view(torch.uint8)


class QuantLinear(torch.nn.Module):
    """y = x W^T (+ bias) with W stored as nvfp4 or fp8r; x is bf16 [..., in_features]."""

    def __init__(self, in_features: int, out_features: int, scheme: str = "nvfp4",
                 bias: bool = True, device=None):
        super().__init__()
        if scheme not in ("nvfp4", "fp8r"):
            raise ValueError(f"unknown scheme {scheme!r} (nvfp4 or fp8r)")
        K, N = in_features, out_features
        if scheme == "nvfp4" and K % 64 != 0:
            raise ValueError("nvfp4 needs in_features % 64 == 0 (16-element blocks, four per "
                             "tensor-core scale column)")
        if scheme == "fp8r" and K % 16 != 0:
            raise ValueError("fp8r needs in_features % 16 == 0")
        if N % 8 != 0:
            raise ValueError("out_features must be a multiple of 8")
        self.in_features, self.out_features, self.scheme = K, N, scheme
        e4m3 = _E4M3 if _E4M3 is not None else torch.uint8
        if scheme == "nvfp4":
            self.register_buffer("weight", torch.zeros((N, K // 2), dtype=torch.uint8,
                                                       device=device))
            self.register_buffer("weight_scale", torch.zeros((N, K // 16), dtype=e4m3,
                                                             device=device))
            self.register_buffer("weight_scale_2", torch.ones((), dtype=torch.float32,
                                                              device=device))
            self.register_buffer("input_scale", torch.ones((), dtype=torch.float32,
                                                           device=device))
        else:
            self.register_buffer("weight", torch.zeros((N, K), dtype=e4m3, device=device))
            self.register_buffer("weight_scale", torch.ones((N,), dtype=torch.float32,
                                                            device=device))
        if bias:
            self.register_buffer("bias", torch.zeros((N,), dtype=torch.bfloat16, device=device))
        else:
            self.bias = None
        self._sf_mma = None          # weight_scale in the tensor-core layout (nvfp4)
        self._workspace = None       # quantized activations (nvfp4), grown on demand

    # ------------------------------------------------------------------ construction
    @classmethod
    def from_linear(cls, linear: torch.nn.Linear, scheme: str = "nvfp4",
                    input_scale=None, calibration: torch.Tensor | None = None) -> "QuantLinear":
        """Quantize a bf16 nn.Linear on its (CUDA) device with the library's quantizers:
        weight_scale_2 = amax(W) / (448*6); the nvfp4 input_scale is `input_scale` if
        given, else calibrated as amax(calibration) / (448*6)."""
        W = linear.weight.detach().to(torch.bfloat16).contiguous()
        if not W.is_cuda:
            raise BSPError("QuantLinear.from_linear (weight not on a CUDA device)", -1)
        N, K = W.shape
        m = cls(K, N, scheme, bias=linear.bias is not None, device=W.device)
        if scheme == "nvfp4":
            g = nvfp4_global_scale(W)
            codes, sf = nvfp4_quantize_act(W, g, layout=SF_LINEAR)
            m.weight.copy_(codes)
            _u8(m.weight_scale).copy_(sf.view(N, K // 16))
            m.weight_scale_2.copy_(g.view(()))
            if input_scale is not None:
                m.input_scale.fill_(float(input_scale))
            elif calibration is not None:
                x = calibration.detach().to(torch.bfloat16).reshape(-1, K).contiguous()
                m.input_scale.copy_(nvfp4_global_scale(x).view(()))
            else:
                raise ValueError("nvfp4 needs input_scale or a calibration activation")
        else:
            q, s = fp8r_quantize_rows(W)
            _u8(m.weight).copy_(q)
            m.weight_scale.copy_(s)
        if linear.bias is not None:
            m.bias.copy_(linear.bias.detach().to(torch.bfloat16))
        return m

    @classmethod
    def from_state_dict(cls, state: dict, prefix: str = "", device=None) -> "QuantLinear":
        """Build from checkpoint tensors; the scheme follows from the names present."""
        w = state[prefix + "weight"]
        nvfp4 = (prefix + "weight_scale_2") in state
        N = w.shape[0]
        K = w.shape[1] * 2 if nvfp4 else w.shape[1]
        m = cls(K, N, "nvfp4" if nvfp4 else "fp8r", bias=(prefix + "bias") in state,
                device=device if device is not None else w.device)
        sub = {k[len(prefix):]: v for k, v in state.items() if k.startswith(prefix)}
        m.load_state_dict(sub)
        return m

    def _load_from_state_dict(self, *args, **kwargs):
        self._sf_mma = None
        return super()._load_from_state_dict(*args, **kwargs)

    def extra_repr(self) -> str:
        return (f"in_features={self.in_features}, out_features={self.out_features}, "
                f"scheme={self.scheme}, bias={self.bias is not None}")

    # ------------------------------------------------------------------ forward
    def forward(self, x: torch.Tensor) -> torch.Tensor:
        K, N = self.in_features, self.out_features
        if x.shape[-1] != K:
            raise ValueError(f"expected last dimension {K}, got {x.shape[-1]}")
        lead = x.shape[:-1]
        x2 = x.reshape(-1, K)
        if x2.dtype != torch.bfloat16:
            raise TypeError("QuantLinear takes bf16 activations")
        x2 = x2.contiguous()
        M = x2.shape[0]
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
        if self.scheme == "nvfp4":
            if self._sf_mma is None:
                self._sf_mma = nvfp4_sf_convert(_u8(self.weight_scale).contiguous(), N, K,
                                                SF_LINEAR, SF_MMA)
            need = nvfp4_linear_workspace_bytes(M, K)
            if self._workspace is None or self._workspace.numel() < need \
                    or self._workspace.device != x.device:
                self._workspace = torch.empty((need,), dtype=torch.uint8, device=x.device)
            nvfp4_linear(x2, self.input_scale, self.weight, self._sf_mma, self.weight_scale_2,
                         bias=self.bias, out=y, workspace=self._workspace)
        else:
            aq, asc = fp8r_quantize_rows(x2)
            fp8r_gemm(aq, asc, _u8(self.weight), self.weight_scale, bias=self.bias, out=y)
        return y.reshape(*lead, N)
