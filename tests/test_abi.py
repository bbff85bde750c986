"""CPU-only checks of the C ABI: the library loads, exports every symbol that
include/*.h declares, and rejects bad arguments on the host before any launch.
No compute call is made (there is no GPU here)."""
import ctypes
import glob
import os
import re

import pytest

import oracle
import block_scaled_precision_act_b200 as bsp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, SHAPE, MISALIGNED = 0, -1, -2, -3


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(",
                             src, flags=re.M):
            if m.group(1) not in ("if", "defined"):
                names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_four_hot_calls():
    names = declared_functions()
    for n in ("nvfp4_quantize_act", "nvfp4_gemm", "fp8r_quantize_rows", "fp8r_gemm"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(bsp.library_path)
    names = declared_functions()
    assert len(names) >= 12
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    # and the binding wraps each of them under the same name
    for n in names:
        assert hasattr(bsp, n), n


def test_sf_bytes_matches_closed_form():
    for rows, K in [(1, 64), (128, 256), (4096, 3072), (200, 320), (65536, 12288)]:
        for layout in (bsp.SF_LINEAR, bsp.SF_MMA):
            assert bsp.nvfp4_sf_bytes(rows, K, layout) == oracle.sf_bytes(rows, K, layout == 1)
    assert bsp.lib().nvfp4_sf_bytes(128, 20, 1) == INVALID
    assert bsp.lib().nvfp4_sf_bytes(128, 64, 7) == INVALID


def test_status_strings():
    for code, name in [(0, "BSP_OK"), (-1, "BSP_ERR_INVALID_ARG"), (-2, "BSP_ERR_UNSUPPORTED_SHAPE"),
                       (-3, "BSP_ERR_MISALIGNED"), (-4, "BSP_ERR_UNSUPPORTED_DEVICE"),
                       (-5, "BSP_ERR_CUDA"), (-6, "BSP_ERR_TIMEOUT")]:
        assert bsp.bsp_status_string(code) == name
    assert bsp.bsp_version() >= 100


P = 1 << 20          # a fake, 16-byte aligned "device" address: never dereferenced here


def test_quantize_validation_on_host():
    L = bsp.lib()
    q = L.nvfp4_quantize_act
    assert q(None, 128, 256, P, P, P, 1, None) == INVALID
    assert q(P, -1, 256, P, P, P, 1, None) == INVALID
    assert q(P, 128, 256, P, P, P, 5, None) == INVALID
    assert q(P, 128, 24, P, P, P, 0, None) == SHAPE           # K % 16
    assert q(P, 128, 80, P, P, P, 1, None) == SHAPE           # MMA layout needs K % 64
    assert q(P + 8, 128, 256, P, P, P, 1, None) == MISALIGNED
    assert q(P, 128, 256, P + 2, P, P, 1, None) == MISALIGNED  # fp32 scalar alignment
    f = L.fp8r_quantize_rows
    assert f(None, 1, 64, P, P, None) == INVALID
    assert f(P, 1, 12, P, P, None) == SHAPE
    assert f(P, 1, 64, P + 4, P, None) == MISALIGNED
    g = L.nvfp4_global_scale
    assert g(P, 12, P, None) == SHAPE
    assert g(None, 16, P, None) == INVALID


def test_dequantize_validation_on_host():
    d = bsp.lib().nvfp4_dequantize
    assert d(None, P, 1, P, 8, 64, P, None) == INVALID
    assert d(P, P, 7, P, 8, 64, P, None) == INVALID            # unknown layout
    assert d(P, P, 1, P, -1, 64, P, None) == INVALID
    assert d(P, P, 0, P, 8, 24, P, None) == SHAPE              # K % 16
    assert d(P, P, 1, P, 8, 80, P, None) == SHAPE              # MMA layout needs K % 64
    assert d(P + 8, P, 1, P, 8, 64, P, None) == MISALIGNED
    assert d(P, P, 1, P + 2, 8, 64, P, None) == MISALIGNED     # fp32 scalar alignment
    assert d(P, P, 1, P, 8, 64, P + 4, None) == MISALIGNED
    assert d(P, P, 1, P, 0, 64, P, None) == 0                  # nothing to do


def test_gemm_validation_on_host():
    L = bsp.lib()
    n = L.nvfp4_gemm
    assert n(None, P, P, P, P, P, None, P, 128, 128, 256, None) == INVALID
    assert n(P, None, P, P, P, P, None, P, 128, 128, 256, None) == INVALID
    assert n(P, P, P, P, P, P, None, P, 128, 128, 96, None) == SHAPE     # K % 64
    assert n(P, P, P, P, P, P, None, P, 128, 12, 256, None) == SHAPE     # N % 8
    assert n(P, P, P, P, P, P, P + 8, P, 128, 128, 256, None) == MISALIGNED
    assert n(P, P, P, P, P, P, None, P, -5, 128, 256, None) == INVALID
    f = L.fp8r_gemm
    assert f(P, P, P, P, None, P, 128, 128, 24, None) == SHAPE          # K % 16
    assert f(P, P, P, P, None, P, 128, 128, 0, None) == SHAPE
    assert f(P, P + 4, P, P, None, P, 128, 128, 256, None) == MISALIGNED
    c = L.nvfp4_sf_convert
    assert c(P, P, 128, 256, 1, 1, None) == INVALID
    assert c(P, P, 128, 48, 0, 1, None) == SHAPE


def test_linear_workspace_and_validation_on_host():
    L = bsp.lib()
    for M, K in [(1, 64), (4096, 3072), (200, 320), (0, 128)]:
        codes = M * K // 2
        scales_end = (codes + 255) // 256 * 256 + oracle.sf_bytes(M, K, True)
        expect = (scales_end + 255) // 256 * 256 + 8192      # + per-CTA maxima (dynamic)
        assert bsp.nvfp4_linear_workspace_bytes(M, K) == expect
    assert L.nvfp4_linear_workspace_bytes(128, 96) == INVALID
    assert L.nvfp4_linear_workspace_bytes(-1, 64) == INVALID
    lin = L.nvfp4_linear
    need = bsp.nvfp4_linear_workspace_bytes(128, 256)
    assert lin(P, P, P, P, P, None, P, 128, 128, 256, None, need, None) == INVALID
    assert lin(P, P, P, P, P, None, P, 128, 128, 256, P, need - 1, None) == INVALID
    assert lin(P, P, P, P, P, None, P, 128, 128, 96, P, need, None) == SHAPE
    assert lin(P, P, P, P, P, None, P, 128, 128, 256, P + 8, need, None) == MISALIGNED
    assert lin(P, P, P, P, P, None, P, 0, 128, 256, None, 0, None) == OK   # empty problem


def test_noalloc_size_limit_on_host():
    L = bsp.lib()
    cap = bsp.nvfp4_linear_noalloc_max_bytes()
    assert cap == 128 << 20
    K = 3072
    rows_ok = 4096
    assert bsp.nvfp4_linear_workspace_bytes(rows_ok, K) <= cap
    rows_big = cap // (K // 2) + 1
    assert L.nvfp4_linear_noalloc(P, P, P, P, P, None, P, rows_big, 256, K, None) == SHAPE
    assert L.nvfp4_linear_noalloc(P, P, P, P, P, None, P, 128, 128, 96, None) == SHAPE
    assert L.nvfp4_linear_noalloc(P, P, P, P, P, None, P, 0, 128, 256, None) == OK


def test_gemm_quant_validation_on_host():
    L = bsp.lib()
    gq = L.nvfp4_gemm_quant
    assert gq(P, P, P, P, P, P, None, None, P, P, 128, 128, 256, None) == INVALID   # no out_global
    assert gq(P, P, P, P, P, P, None, P, P, None, 128, 128, 256, None) == INVALID   # no out_sf
    assert gq(P, P, P, P, P, P, None, P, None, P, 128, 128, 256, None) == INVALID   # no codes
    assert gq(P, P, P, P, P, P, None, P, P, P, 128, 96, 256, None) == SHAPE         # N % 64
    assert gq(P, P, P, P, P, P, None, P, P, P + 8, 128, 128, 256, None) == MISALIGNED
    assert gq(P, P, P, P, P, P, None, P + 2, P, P, 128, 128, 256, None) == MISALIGNED
    assert gq(P, P, P, P, P, P, None, P, P, P, 0, 128, 256, None) == OK             # empty


def test_linear_dynamic_validation_on_host():
    L = bsp.lib()
    d = L.nvfp4_linear_dynamic
    need = bsp.nvfp4_linear_workspace_bytes(128, 256)
    assert d(P, None, P, P, P, None, P, 128, 128, 256, P, need, None) == INVALID   # no g out
    assert d(P, P, P, P, P, None, P, 128, 128, 256, P, need - 1, None) == INVALID
    assert d(P, P, P, P, P, None, P, 128, 128, 96, P, need, None) == SHAPE
    assert d(P, P, P, P, P, None, P, 0, 128, 256, None, 0, None) == OK


def test_fp8r_linear_workspace_and_validation_on_host():
    L = bsp.lib()
    a256 = lambda v: (v + 255) // 256 * 256
    assert bsp.fp8r_linear_workspace_bytes(256, 3072) == a256(256 * 3072) + a256(1024)
    assert bsp.fp8r_linear_workspace_bytes(4096, 3072) == a256(4096 * 3072) + a256(4 * 4096)
    assert L.fp8r_linear_workspace_bytes(256, 12) == INVALID
    f = L.fp8r_linear
    need = bsp.fp8r_linear_workspace_bytes(128, 256)
    assert f(P, P, P, None, P, 128, 128, 256, None, need, None) == INVALID
    assert f(P, P, P, None, P, 128, 128, 256, P, need - 1, None) == INVALID
    assert f(P, P, P, None, P, 128, 128, 256, P + 8, need, None) == MISALIGNED
    assert f(P, P, P, None, P, 0, 128, 256, None, 0, None) == OK


def test_testing_hook_validation():
    L = bsp.lib()
    h = L.bsp_testing_gemm_stall
    assert h(1, P, P, P, P, P, P, P, 128, 128, 256, -1, 100, None) == INVALID
    assert h(1, P, P, P, P, P, P, P, 128, 128, 256, 1, 0, None) == INVALID
    assert h(7, P, P, P, P, P, P, P, 128, 128, 256, 1, 100, None) == INVALID
    assert L.bsp_testing_set_quant_kernel(7) == INVALID
    assert L.bsp_testing_cvt_range(2, 0, 16, P, None) == INVALID
    assert L.bsp_testing_cvt_range(0, 0xFFFFFFF0, 32, P, None) == INVALID    # past 2^32
    assert L.bsp_testing_cvt_range(0, 0, 0, None, None) == OK
    assert bsp.bsp_testing_set_quant_kernel(0) == 0


def test_python_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros((128, 256), dtype=torch.bfloat16)
    g = torch.ones((1,), dtype=torch.float32)
    with pytest.raises(bsp.BSPError, match="not on a CUDA device"):
        bsp.nvfp4_quantize_act(x, g, codes=torch.empty((128, 128), dtype=torch.uint8),
                               scales=torch.empty((bsp.nvfp4_sf_bytes(128, 256),),
                                                  dtype=torch.uint8))
