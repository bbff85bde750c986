"""Python binding of ``libbsp.so``: the NVFP4 / fp8r quantized linear on B200.

Argument marshalling only.  Every step of the path runs in the library's CUDA
kernels; torch supplies device memory and the current stream.  There is no CPU
fallback: importing works without a GPU (so the ABI can be inspected), but every
compute call needs the built library and a compute-capability-10.0 device, and
raises ``BSPError`` otherwise.

The C entry points and their semantics are declared in ``include/bsp.h``; the
functions here carry the same names.  Formats ("BFL (fp8r / nvfp4)", Diffusers
quantization doc, format bullets): nvfp4 = packed E2M1 codes, E4M3 scale per 16
elements, fp32 global scales; fp8r = E4M3 values with an fp32 scale per row.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "BSPError", "SF_LINEAR", "SF_MMA", "lib", "library_path",
    "nvfp4_quantize_act", "nvfp4_gemm", "nvfp4_gemm_quant", "fp8r_quantize_rows", "fp8r_gemm",
    "nvfp4_linear", "nvfp4_linear_dynamic", "nvfp4_linear_workspace_bytes", "nvfp4_linear_noalloc",
    "nvfp4_linear_noalloc_max_bytes", "fp8r_linear", "fp8r_linear_workspace_bytes",
    "nvfp4_global_scale", "nvfp4_sf_convert", "nvfp4_sf_bytes", "nvfp4_dequantize",
    "bsp_last_device_status", "bsp_set_wait_limit_ms", "bsp_status_string", "bsp_version",
    "bsp_testing_gemm_stall", "bsp_testing_set_gemm_kernel", "bsp_testing_set_quant_kernel",
    "bsp_testing_cvt_range",
]

SF_LINEAR = 0
SF_MMA = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libbsp.so")

_c_i64 = ctypes.c_int64
_c_int = ctypes.c_int
_c_vp = ctypes.c_void_p

_SIGS = {
    "nvfp4_quantize_act": ([_c_vp, _c_i64, _c_i64, _c_vp, _c_vp, _c_vp, _c_int, _c_vp], _c_int),
    "nvfp4_gemm": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64,
                    _c_i64, _c_vp], _c_int),
    "nvfp4_gemm_quant": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp,
                          _c_i64, _c_i64, _c_i64, _c_vp], _c_int),
    "nvfp4_linear": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64, _c_i64,
                      _c_vp, _c_i64, _c_vp], _c_int),
    "nvfp4_linear_workspace_bytes": ([_c_i64, _c_i64], _c_i64),
    "nvfp4_linear_dynamic": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64,
                              _c_i64, _c_vp, _c_i64, _c_vp], _c_int),
    "nvfp4_linear_noalloc": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64,
                              _c_i64, _c_vp], _c_int),
    "nvfp4_linear_noalloc_max_bytes": ([], _c_i64),
    "fp8r_quantize_rows": ([_c_vp, _c_i64, _c_i64, _c_vp, _c_vp, _c_vp], _c_int),
    "fp8r_linear": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64, _c_i64, _c_vp, _c_i64,
                     _c_vp], _c_int),
    "fp8r_linear_workspace_bytes": ([_c_i64, _c_i64], _c_i64),
    "fp8r_gemm": ([_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64, _c_i64, _c_vp],
                  _c_int),
    "nvfp4_global_scale": ([_c_vp, _c_i64, _c_vp, _c_vp], _c_int),
    "nvfp4_sf_convert": ([_c_vp, _c_vp, _c_i64, _c_i64, _c_int, _c_int, _c_vp], _c_int),
    "nvfp4_dequantize": ([_c_vp, _c_vp, _c_int, _c_vp, _c_i64, _c_i64, _c_vp, _c_vp], _c_int),
    "nvfp4_sf_bytes": ([_c_i64, _c_i64, _c_int], _c_i64),
    "bsp_last_device_status": ([_c_vp], _c_int),
    "bsp_set_wait_limit_ms": ([_c_i64], _c_i64),
    "bsp_status_string": ([_c_int], ctypes.c_char_p),
    "bsp_version": ([], _c_int),
    "bsp_testing_set_gemm_kernel": ([_c_int], _c_int),
    "bsp_testing_set_quant_kernel": ([_c_int], _c_int),
    "bsp_testing_cvt_range": ([_c_int, ctypes.c_uint32, _c_i64, _c_vp, _c_vp], _c_int),
    "bsp_testing_gemm_stall": ([_c_int, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i64,
                                _c_i64, _c_i64, _c_i64, _c_i64, _c_vp], _c_int),
}

_lib = None


class BSPError(RuntimeError):
    """A libbsp call returned a negative bsp_status."""

    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_name(status)} ({status})")


def lib() -> ctypes.CDLL:
    """Load ``libbsp.so`` (raises if it has not been built: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise BSPError("load", -5) from FileNotFoundError(
                f"{library_path} is missing; build it with "
                "`python -m block_scaled_precision_act_b200.build` (or __graft_entry__.build())")
        L = ctypes.CDLL(library_path)
        for name, (argtypes, restype) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = argtypes
            fn.restype = restype
        _lib = L
    return _lib


def status_name(status: int) -> str:
    names = {0: "BSP_OK", -1: "BSP_ERR_INVALID_ARG", -2: "BSP_ERR_UNSUPPORTED_SHAPE",
             -3: "BSP_ERR_MISALIGNED", -4: "BSP_ERR_UNSUPPORTED_DEVICE", -5: "BSP_ERR_CUDA",
             -6: "BSP_ERR_TIMEOUT"}
    return names.get(status, "BSP_ERR_UNKNOWN")


def _check(fn: str, st: int) -> None:
    if st != 0:
        raise BSPError(fn, st)


def _require_current_device(index: int, current: int | None = None) -> None:
    """The C calls run on the current CUDA device and stream (cudaGetDevice): a tensor on
    any other device would be handed to that device's kernels as a peer address, so it
    is refused here."""
    cur = torch.cuda.current_device() if current is None else current
    if index != cur:
        raise BSPError(f"argument check (tensor on cuda:{index}, but the current device is "
                       f"cuda:{cur}; use torch.cuda.device)", -1)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise BSPError("argument check (tensor not on a CUDA device)", -1)
    _require_current_device(t.device.index)
    if not t.is_contiguous():
        raise BSPError("argument check (tensor not contiguous)", -1)
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dtype(t, dt, what):
    if t.dtype != dt:
        raise TypeError(f"{what} must be {dt}, got {t.dtype}")


def _buf(t, dt, what, min_numel: int):
    """A buffer the library reads or writes `min_numel` elements of: dtype and size are
    checked here, since the C calls receive only its address."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what} must be a torch.Tensor")
    _dtype(t, dt, what)
    if t.numel() < min_numel:
        raise BSPError(f"argument check ({what} holds {t.numel()} elements, needs {min_numel})",
                       -1)


def _mat(t, dt, what, cols=None):
    """A 2-D operand whose shape gives the problem size; returns (rows, cols)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what} must be a torch.Tensor")
    _dtype(t, dt, what)
    if t.dim() != 2:
        raise BSPError(f"argument check ({what} must be 2-D, got {tuple(t.shape)})", -1)
    if cols is not None and t.shape[1] != cols:
        raise BSPError(f"argument check ({what} has {t.shape[1]} columns, needs {cols})", -1)
    return t.shape[0], t.shape[1]


# ------------------------------------------------------------------ entry points
def nvfp4_sf_bytes(rows: int, K: int, layout: int = SF_MMA) -> int:
    n = lib().nvfp4_sf_bytes(rows, K, layout)
    if n < 0:
        raise BSPError("nvfp4_sf_bytes", int(n))
    return int(n)


def nvfp4_quantize_act(x: torch.Tensor, global_scale: torch.Tensor, codes=None, scales=None,
                       layout: int = SF_MMA, stream=None):
    """bf16 [M, K] -> (codes uint8 [M, K/2], block scales uint8 in `layout`)."""
    M, K = _mat(x, torch.bfloat16, "x")
    _buf(global_scale, torch.float32, "global_scale", 1)
    if codes is None:
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((max(nvfp4_sf_bytes(M, K, layout), 0),), dtype=torch.uint8,
                             device=x.device)
    _buf(codes, torch.uint8, "codes", M * (K // 2))
    _buf(scales, torch.uint8, "scales", max(nvfp4_sf_bytes(M, K, layout), 0))
    _check("nvfp4_quantize_act",
           lib().nvfp4_quantize_act(_ptr(x), M, K, _ptr(global_scale), _ptr(codes),
                                    _ptr(scales), layout, _stream(stream)))
    return codes, scales


def _nvfp4_operands(M, N, K, a_sf, a_global, w_sf, w_global, bias):
    _buf(a_sf, torch.uint8, "a_sf", max(nvfp4_sf_bytes(M, K, SF_MMA), 0))
    _buf(a_global, torch.float32, "a_global", 1)
    _buf(w_sf, torch.uint8, "w_sf", max(nvfp4_sf_bytes(N, K, SF_MMA), 0))
    _buf(w_global, torch.float32, "w_global", 1)
    _buf(bias, torch.bfloat16, "bias", N)


def nvfp4_gemm(a_codes, a_sf, a_global, w_codes, w_sf, w_global, bias=None, out=None,
               stream=None):
    """Y[M, N] bf16 = (a_global*w_global) * (A_q . W_q^T) (+ bias); scales in SF_MMA layout."""
    M, K2 = _mat(a_codes, torch.uint8, "a_codes")
    N, _ = _mat(w_codes, torch.uint8, "w_codes", K2)
    _nvfp4_operands(M, N, 2 * K2, a_sf, a_global, w_sf, w_global, bias)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a_codes.device)
    _buf(out, torch.bfloat16, "out", M * N)
    _check("nvfp4_gemm",
           lib().nvfp4_gemm(_ptr(a_codes), _ptr(a_sf), _ptr(a_global), _ptr(w_codes),
                            _ptr(w_sf), _ptr(w_global), _ptr(bias), _ptr(out), M, N, 2 * K2,
                            _stream(stream)))
    return out


def nvfp4_gemm_quant(a_codes, a_sf, a_global, w_codes, w_sf, w_global, out_global, bias=None,
                     out_codes=None, out_sf=None, stream=None):
    """nvfp4_gemm whose bf16 output is re-quantized in the epilogue for the next nvfp4
    linear: returns (codes uint8 [M, N/2], MMA-layout scales) under `out_global`."""
    M, K2 = _mat(a_codes, torch.uint8, "a_codes")
    N, _ = _mat(w_codes, torch.uint8, "w_codes", K2)
    _nvfp4_operands(M, N, 2 * K2, a_sf, a_global, w_sf, w_global, bias)
    _buf(out_global, torch.float32, "out_global", 1)
    if out_codes is None:
        out_codes = torch.empty((M, N // 2), dtype=torch.uint8, device=a_codes.device)
    if out_sf is None:
        out_sf = torch.empty((max(nvfp4_sf_bytes(M, N, SF_MMA), 0),), dtype=torch.uint8,
                             device=a_codes.device)
    _buf(out_codes, torch.uint8, "out_codes", M * (N // 2))
    _buf(out_sf, torch.uint8, "out_sf", max(nvfp4_sf_bytes(M, N, SF_MMA), 0))
    _check("nvfp4_gemm_quant",
           lib().nvfp4_gemm_quant(_ptr(a_codes), _ptr(a_sf), _ptr(a_global), _ptr(w_codes),
                                  _ptr(w_sf), _ptr(w_global), _ptr(bias), _ptr(out_global),
                                  _ptr(out_codes), _ptr(out_sf), M, N, 2 * K2, _stream(stream)))
    return out_codes, out_sf


def nvfp4_linear_workspace_bytes(M: int, K: int) -> int:
    n = lib().nvfp4_linear_workspace_bytes(M, K)
    if n < 0:
        raise BSPError("nvfp4_linear_workspace_bytes", int(n))
    return int(n)


def nvfp4_linear(x: torch.Tensor, input_scale: torch.Tensor, w_codes, w_sf, w_scale, bias=None,
                 out=None, workspace=None, stream=None):
    """Y[M, N] bf16 = nvfp4 linear of bf16 x [M, K]: activation quantizer + FP4 GEMM in one
    call (the GEMM overlaps the quantizer's tail).  `workspace` (uint8, at least
    nvfp4_linear_workspace_bytes(M, K) bytes) is allocated here when not given."""
    M, K = _mat(x, torch.bfloat16, "x")
    _buf(input_scale, torch.float32, "input_scale", 1)
    N, _ = _mat(w_codes, torch.uint8, "w_codes", K // 2)
    _nvfp4_operands(0, N, K, None, None, w_sf, w_scale, bias)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _buf(out, torch.bfloat16, "out", M * N)
    if workspace is None:
        workspace = torch.empty((max(nvfp4_linear_workspace_bytes(M, K), 0),), dtype=torch.uint8,
                                device=x.device)
    _buf(workspace, torch.uint8, "workspace", 0)
    _check("nvfp4_linear",
           lib().nvfp4_linear(_ptr(x), _ptr(input_scale), _ptr(w_codes), _ptr(w_sf),
                              _ptr(w_scale), _ptr(bias), _ptr(out), M, N, K, _ptr(workspace),
                              workspace.numel(), _stream(stream)))
    return out


def nvfp4_linear_noalloc_max_bytes() -> int:
    return int(lib().nvfp4_linear_noalloc_max_bytes())


def nvfp4_linear_noalloc(x: torch.Tensor, input_scale: torch.Tensor, w_codes, w_sf, w_scale,
                         out: torch.Tensor, bias=None, stream=None):
    """nvfp4_linear with the library's own per-device buffer as workspace; allocates
    nothing, so `out` ([M, N] bf16) must be given.  Calls that can run concurrently on
    one device race on that buffer (see include/bsp.h)."""
    M, K = _mat(x, torch.bfloat16, "x")
    _buf(input_scale, torch.float32, "input_scale", 1)
    N, _ = _mat(w_codes, torch.uint8, "w_codes", K // 2)
    _nvfp4_operands(0, N, K, None, None, w_sf, w_scale, bias)
    _dtype(out, torch.bfloat16, "out")
    if tuple(out.shape) != (M, N):
        raise BSPError("nvfp4_linear_noalloc (shape mismatch)", -1)
    _check("nvfp4_linear_noalloc",
           lib().nvfp4_linear_noalloc(_ptr(x), _ptr(input_scale), _ptr(w_codes), _ptr(w_sf),
                                      _ptr(w_scale), _ptr(bias), _ptr(out), M, N, K,
                                      _stream(stream)))
    return out


def nvfp4_linear_dynamic(x: torch.Tensor, w_codes, w_sf, w_scale, bias=None, out=None,
                         input_scale_out=None, workspace=None, stream=None):
    """nvfp4_linear with input_scale = amax(x) / (448*6) computed on the device for this
    call; returns (out, input_scale_out)."""
    M, K = _mat(x, torch.bfloat16, "x")
    N, _ = _mat(w_codes, torch.uint8, "w_codes", K // 2)
    _nvfp4_operands(0, N, K, None, None, w_sf, w_scale, bias)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _buf(out, torch.bfloat16, "out", M * N)
    if input_scale_out is None:
        input_scale_out = torch.empty((1,), dtype=torch.float32, device=x.device)
    _buf(input_scale_out, torch.float32, "input_scale_out", 1)
    if workspace is None:
        workspace = torch.empty((max(nvfp4_linear_workspace_bytes(M, K), 0),), dtype=torch.uint8,
                                device=x.device)
    _buf(workspace, torch.uint8, "workspace", 0)
    _check("nvfp4_linear_dynamic",
           lib().nvfp4_linear_dynamic(_ptr(x), _ptr(input_scale_out), _ptr(w_codes), _ptr(w_sf),
                                      _ptr(w_scale), _ptr(bias), _ptr(out), M, N, K,
                                      _ptr(workspace), workspace.numel(), _stream(stream)))
    return out, input_scale_out


def fp8r_quantize_rows(x: torch.Tensor, q=None, row_scale=None, stream=None):
    """bf16 [M, K] -> (E4M3 codes uint8 [M, K], fp32 row scales [M])."""
    M, K = _mat(x, torch.bfloat16, "x")
    if q is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if row_scale is None:
        row_scale = torch.empty((M,), dtype=torch.float32, device=x.device)
    _buf(q, torch.uint8, "q", M * K)
    _buf(row_scale, torch.float32, "row_scale", M)
    _check("fp8r_quantize_rows",
           lib().fp8r_quantize_rows(_ptr(x), M, K, _ptr(q), _ptr(row_scale), _stream(stream)))
    return q, row_scale


def fp8r_linear_workspace_bytes(M: int, K: int) -> int:
    n = lib().fp8r_linear_workspace_bytes(M, K)
    if n < 0:
        raise BSPError("fp8r_linear_workspace_bytes", int(n))
    return int(n)


def fp8r_linear(x: torch.Tensor, w_q, w_row_scale, bias=None, out=None, workspace=None,
                stream=None):
    """Y[M, N] bf16 = fp8r linear of bf16 x [M, K]: row quantizer + FP8 GEMM in one call.
    `workspace` (uint8, at least fp8r_linear_workspace_bytes(M, K) bytes) is allocated here
    when not given."""
    M, K = _mat(x, torch.bfloat16, "x")
    N, _ = _mat(w_q, torch.uint8, "w_q", K)
    _buf(w_row_scale, torch.float32, "w_row_scale", N)
    _buf(bias, torch.bfloat16, "bias", N)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _buf(out, torch.bfloat16, "out", M * N)
    if workspace is None:
        workspace = torch.empty((max(fp8r_linear_workspace_bytes(M, K), 0),),
                                dtype=torch.uint8, device=x.device)
    _buf(workspace, torch.uint8, "workspace", 0)
    _check("fp8r_linear",
           lib().fp8r_linear(_ptr(x), _ptr(w_q), _ptr(w_row_scale), _ptr(bias), _ptr(out), M, N, K,
                             _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def fp8r_gemm(a_q, a_row_scale, w_q, w_row_scale, bias=None, out=None, stream=None):
    """Y[M, N] bf16 = (A_q . W_q^T) * sA[m] * sW[n] (+ bias)."""
    M, K = _mat(a_q, torch.uint8, "a_q")
    N, _ = _mat(w_q, torch.uint8, "w_q", K)
    _buf(a_row_scale, torch.float32, "a_row_scale", M)
    _buf(w_row_scale, torch.float32, "w_row_scale", N)
    _buf(bias, torch.bfloat16, "bias", N)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a_q.device)
    _buf(out, torch.bfloat16, "out", M * N)
    _check("fp8r_gemm",
           lib().fp8r_gemm(_ptr(a_q), _ptr(a_row_scale), _ptr(w_q), _ptr(w_row_scale),
                           _ptr(bias), _ptr(out), M, N, K, _stream(stream)))
    return out


def nvfp4_global_scale(x: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """fp32 [1] = amax(x) / (448*6), computed on the device."""
    _dtype(x, torch.bfloat16, "x")
    if out is None:
        out = torch.empty((1,), dtype=torch.float32, device=x.device)
    _buf(out, torch.float32, "out", 1)
    _check("nvfp4_global_scale",
           lib().nvfp4_global_scale(_ptr(x), x.numel(), _ptr(out), _stream(stream)))
    return out


def nvfp4_sf_convert(src, rows: int, K: int, from_layout: int, to_layout: int, dst=None,
                     stream=None):
    _buf(src, torch.uint8, "src", nvfp4_sf_bytes(rows, K, from_layout))
    if dst is None:
        dst = torch.empty((nvfp4_sf_bytes(rows, K, to_layout),), dtype=torch.uint8,
                          device=src.device)
    _buf(dst, torch.uint8, "dst", nvfp4_sf_bytes(rows, K, to_layout))
    _check("nvfp4_sf_convert",
           lib().nvfp4_sf_convert(_ptr(src), _ptr(dst), rows, K, from_layout, to_layout,
                                  _stream(stream)))
    return dst


def nvfp4_dequantize(codes: torch.Tensor, scales: torch.Tensor, global_scale: torch.Tensor,
                     layout: int = SF_MMA, out=None, stream=None) -> torch.Tensor:
    """NVFP4 codes [rows, K/2] + block scales + fp32 global scale -> bf16 [rows, K]
    (the dequantise-only fallback's weight decode; see nvfp4_dequantize in bsp.h)."""
    rows, K2 = _mat(codes, torch.uint8, "codes")
    K = 2 * K2
    _buf(scales, torch.uint8, "scales", max(nvfp4_sf_bytes(rows, K, layout), 0))
    _buf(global_scale, torch.float32, "global_scale", 1)
    if out is None:
        out = torch.empty((rows, K), dtype=torch.bfloat16, device=codes.device)
    _buf(out, torch.bfloat16, "out", rows * K)
    _check("nvfp4_dequantize",
           lib().nvfp4_dequantize(_ptr(codes), _ptr(scales), layout, _ptr(global_scale), rows, K,
                                  _ptr(out), _stream(stream)))
    return out


def bsp_last_device_status(stream=None) -> int:
    return int(lib().bsp_last_device_status(_stream(stream)))


def bsp_set_wait_limit_ms(ms: int) -> int:
    return int(lib().bsp_set_wait_limit_ms(ms))


def bsp_status_string(status: int) -> str:
    return lib().bsp_status_string(status).decode()


def bsp_version() -> int:
    return int(lib().bsp_version())


def bsp_testing_gemm_stall(scheme: int, a, a_sf, a_scale, w, w_sf, w_scale, out, K: int,
                           stop_after_stages: int, wait_limit_ms: int, stream=None) -> int:
    """Test hook (include/bsp_testing.h): returns the launch status, not the device status."""
    M = a.shape[0]
    N = w.shape[0]
    return int(lib().bsp_testing_gemm_stall(scheme, _ptr(a), _ptr(a_sf), _ptr(a_scale), _ptr(w),
                                            _ptr(w_sf), _ptr(w_scale), _ptr(out), M, N, K,
                                            stop_after_stages, wait_limit_ms, _stream(stream)))


def bsp_testing_set_gemm_kernel(choice: int) -> int:
    """Test hook: 0 = automatic, 1 = CTA-pair kernel, 2 = single-CTA kernel."""
    old = int(lib().bsp_testing_set_gemm_kernel(choice))
    if old < 0:
        raise BSPError("bsp_testing_set_gemm_kernel", old)
    return old


def bsp_testing_set_quant_kernel(choice: int) -> int:
    """Test hook: 0 = by size, 1 = grid-stride quantizer kernel, 2 = staged kernel."""
    old = int(lib().bsp_testing_set_quant_kernel(choice))
    if old < 0:
        raise BSPError("bsp_testing_set_quant_kernel", old)
    return old


def bsp_testing_cvt_range(kind: int, first: int, n: int, out=None, stream=None):
    """Test hook: the quantizers' E2M1 (kind 0) / E4M3 (kind 1) conversion of the fp32
    values with bit patterns first .. first+n-1, as uint8 on the current device."""
    if out is None:
        out = torch.empty((n,), dtype=torch.uint8, device="cuda")
    _check("bsp_testing_cvt_range",
           lib().bsp_testing_cvt_range(kind, first, n, _ptr(out), _stream(stream)))
    return out
