"""CPU checks of QuantLinear's state-dict form (no GPU compute).

"BFL (fp8r / nvfp4)" (Diffusers quantization doc), format bullets: nvfp4 linears carry
`weight`, `weight_scale`, `weight_scale_2`, `input_scale`; fp8r linears carry `weight`
and a per-row `weight_scale`; the scheme is read from the checkpoint.
"""
import pytest
import torch

from block_scaled_precision_act_b200.nn import QuantLinear


def test_nvfp4_state_dict_names_shapes_and_storage():
    m = QuantLinear(3072, 1024, "nvfp4", bias=True)
    sd = m.state_dict()
    assert sorted(sd) == ["bias", "input_scale", "weight", "weight_scale", "weight_scale_2"]
    assert sd["weight"].shape == (1024, 1536) and sd["weight"].dtype == torch.uint8
    assert sd["weight_scale"].shape == (1024, 192)
    assert sd["weight_scale"].element_size() == 1
    assert sd["weight_scale_2"].shape == () and sd["weight_scale_2"].dtype == torch.float32
    assert sd["input_scale"].shape == () and sd["bias"].dtype == torch.bfloat16
    # storage: N*K/2 + N*K/16 bytes + two fp32 scalars = 0.5625 B per weight + 8 B
    nbytes = sum(t.numel() * t.element_size() for k, t in sd.items() if k != "bias")
    assert nbytes == 1024 * 3072 * 9 // 16 + 8


def test_fp8r_state_dict_names_and_shapes():
    m = QuantLinear(3072, 3072, "fp8r", bias=False)
    sd = m.state_dict()
    assert sorted(sd) == ["weight", "weight_scale"]
    assert sd["weight"].shape == (3072, 3072) and sd["weight"].element_size() == 1
    assert sd["weight_scale"].shape == (3072,) and sd["weight_scale"].dtype == torch.float32


def test_scheme_read_from_the_tensors_present():
    nv = QuantLinear(256, 128, "nvfp4", bias=False).state_dict()
    f8 = QuantLinear(256, 128, "fp8r", bias=True).state_dict()
    a = QuantLinear.from_state_dict({"blk.proj." + k: v for k, v in nv.items()}, "blk.proj.")
    b = QuantLinear.from_state_dict(f8)
    assert a.scheme == "nvfp4" and a.in_features == 256 and a.out_features == 128
    assert a.bias is None
    assert b.scheme == "fp8r" and b.in_features == 256 and b.bias is not None


def test_unsupported_shapes_are_refused():
    with pytest.raises(ValueError):
        QuantLinear(96, 128, "nvfp4")          # K % 64
    with pytest.raises(ValueError):
        QuantLinear(256, 100, "fp8r")          # N % 8
    with pytest.raises(ValueError):
        QuantLinear(256, 128, "int4")
