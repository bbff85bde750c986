"""The Python binding checks every buffer it hands to the C calls, which receive only
addresses: dtypes, and sizes against what the call reads or writes for the problem the
operands' shapes define.  A buffer that is too small is refused before anything reaches
the device; buffers of exactly the right size pass every check and are refused only for
being on the CPU, which pins the binding's size formulas without a GPU."""
import pytest
import torch

import block_scaled_precision_act_b200 as bsp

ON_CPU = "not on a CUDA device"
TOO_SMALL = "elements, needs"

M, N, K = 200, 136, 320            # ragged against the tiles


def u8(*shape):
    return torch.zeros(shape, dtype=torch.uint8)


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def f32(*shape):
    return torch.ones(shape, dtype=torch.float32)


def nvfp4_operands():
    return dict(a_codes=u8(M, K // 2), a_sf=u8(bsp.nvfp4_sf_bytes(M, K)), a_global=f32(1),
                w_codes=u8(N, K // 2), w_sf=u8(bsp.nvfp4_sf_bytes(N, K)), w_global=f32(1))


def test_quantizer_buffers():
    x, g = bf16(M, K), f32(1)
    ok = dict(codes=u8(M, K // 2), scales=u8(bsp.nvfp4_sf_bytes(M, K)))
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.nvfp4_quantize_act(x, g, **ok)
    with pytest.raises(bsp.BSPError, match=ON_CPU):            # linear layout sizes too
        bsp.nvfp4_quantize_act(x, g, codes=ok["codes"],
                               scales=u8(M * K // 16), layout=bsp.SF_LINEAR)
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_quantize_act(x, g, codes=u8(M - 1, K // 2), scales=ok["scales"])
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_quantize_act(x, g, codes=ok["codes"],
                               scales=u8(bsp.nvfp4_sf_bytes(M, K) - 1))
    with pytest.raises(TypeError):
        bsp.nvfp4_quantize_act(x.float(), g, **ok)
    with pytest.raises(TypeError):
        bsp.nvfp4_quantize_act(x, g.double(), **ok)
    with pytest.raises(bsp.BSPError, match="2-D"):
        bsp.nvfp4_quantize_act(bf16(M * K), g, **ok)
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_quantize_act(x, f32(0), **ok)


def test_gemm_buffers():
    ops = nvfp4_operands()
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.nvfp4_gemm(**ops, bias=bf16(N), out=bf16(M, N))
    for name, bad in [("a_sf", u8(bsp.nvfp4_sf_bytes(M, K) - 1)),
                      ("w_sf", u8(bsp.nvfp4_sf_bytes(N, K) - 16)), ("a_global", f32(0))]:
        with pytest.raises(bsp.BSPError, match=TOO_SMALL):
            bsp.nvfp4_gemm(**{**ops, name: bad}, out=bf16(M, N))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_gemm(**ops, bias=bf16(N - 8), out=bf16(M, N))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_gemm(**ops, out=bf16(M, N - 8))
    with pytest.raises(TypeError):
        bsp.nvfp4_gemm(**ops, bias=f32(N), out=bf16(M, N))
    with pytest.raises(TypeError):
        bsp.nvfp4_gemm(**ops, out=f32(M, N))
    with pytest.raises(bsp.BSPError, match="columns"):
        bsp.nvfp4_gemm(**{**ops, "w_codes": u8(N, K // 2 - 32)}, out=bf16(M, N))


def test_gemm_quant_buffers():
    ops = nvfp4_operands()
    N2 = 192                                       # N % 64 == 0 for the re-quantized output
    ops["w_codes"], ops["w_sf"] = u8(N2, K // 2), u8(bsp.nvfp4_sf_bytes(N2, K))
    out_codes, out_sf = u8(M, N2 // 2), u8(bsp.nvfp4_sf_bytes(M, N2))
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.nvfp4_gemm_quant(**ops, out_global=f32(1), out_codes=out_codes, out_sf=out_sf)
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_gemm_quant(**ops, out_global=f32(1), out_codes=u8(M, N2 // 2 - 1),
                             out_sf=out_sf)
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_gemm_quant(**ops, out_global=f32(1), out_codes=out_codes, out_sf=u8(16))


def test_linear_buffers():
    x, g = bf16(M, K), torch.ones((), dtype=torch.float32)        # 0-dim, as QuantLinear's
    w, wsf, gw = u8(N, K // 2), u8(bsp.nvfp4_sf_bytes(N, K)), torch.ones((), dtype=torch.float32)
    ws = u8(bsp.nvfp4_linear_workspace_bytes(M, K))
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.nvfp4_linear(x, g, w, wsf, gw, bias=bf16(N), out=bf16(M, N), workspace=ws)
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.nvfp4_linear_dynamic(x, w, wsf, gw, out=bf16(M, N), input_scale_out=f32(1),
                                 workspace=ws)
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.nvfp4_linear_noalloc(x, g, w, wsf, gw, out=bf16(M, N))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_linear(x, g, w, u8(bsp.nvfp4_sf_bytes(N, K) - 1), gw, out=bf16(M, N),
                         workspace=ws)
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_linear(x, g, w, wsf, gw, out=bf16(M - 1, N), workspace=ws)
    with pytest.raises(TypeError):
        bsp.nvfp4_linear(x, g, w, wsf, gw, out=bf16(M, N), workspace=f32(ws.numel()))
    with pytest.raises(bsp.BSPError, match="columns"):
        bsp.nvfp4_linear(bf16(M, K + 64), g, w, wsf, gw, out=bf16(M, N), workspace=ws)


def test_fp8r_buffers():
    x = bf16(M, K)
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.fp8r_quantize_rows(x, q=u8(M, K), row_scale=f32(M))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.fp8r_quantize_rows(x, q=u8(M, K - 1), row_scale=f32(M))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.fp8r_quantize_rows(x, q=u8(M, K), row_scale=f32(M - 1))
    aq, asc, wq, wsc = u8(M, K), f32(M), u8(N, K), f32(N)
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.fp8r_gemm(aq, asc, wq, wsc, bias=bf16(N), out=bf16(M, N))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.fp8r_gemm(aq, f32(M - 1), wq, wsc, out=bf16(M, N))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.fp8r_gemm(aq, asc, wq, f32(N - 1), out=bf16(M, N))
    ws = u8(bsp.fp8r_linear_workspace_bytes(M, K))
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.fp8r_linear(x, wq, wsc, bias=bf16(N), out=bf16(M, N), workspace=ws)
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.fp8r_linear(x, wq, wsc, out=bf16(M, N - 8), workspace=ws)


def test_helper_buffers():
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.nvfp4_global_scale(bf16(M, K), out=f32(1))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_global_scale(bf16(M, K), out=f32(0))
    src = u8(M * K // 16)
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.nvfp4_sf_convert(src, M, K, bsp.SF_LINEAR, bsp.SF_MMA,
                             dst=u8(bsp.nvfp4_sf_bytes(M, K)))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_sf_convert(src, M, K, bsp.SF_LINEAR, bsp.SF_MMA, dst=u8(16))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_sf_convert(u8(10), M, K, bsp.SF_LINEAR, bsp.SF_MMA)
    codes, sf = u8(M, K // 2), u8(bsp.nvfp4_sf_bytes(M, K))
    with pytest.raises(bsp.BSPError, match=ON_CPU):
        bsp.nvfp4_dequantize(codes, sf, f32(1), out=bf16(M, K))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_dequantize(codes, u8(16), f32(1), out=bf16(M, K))
    with pytest.raises(bsp.BSPError, match=TOO_SMALL):
        bsp.nvfp4_dequantize(codes, sf, f32(1), out=bf16(M, K - 16))


def test_tensor_on_another_device_is_refused():
    """The C calls launch on the current device (cudaGetDevice) and its stream; a tensor
    of another GPU would reach that device's kernels as a peer address.  The binding
    refuses it: pinned on the decision itself, with the current device given."""
    bsp._require_current_device(0, current=0)
    bsp._require_current_device(3, current=3)
    with pytest.raises(bsp.BSPError, match="current device is cuda:0"):
        bsp._require_current_device(1, current=0)
    with pytest.raises(bsp.BSPError, match="tensor on cuda:0"):
        bsp._require_current_device(0, current=2)
