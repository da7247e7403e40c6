"""The Python binding's argument checks, on the CPU: a tensor whose dtype or layout the call
cannot take, or one in host memory, raises before its pointer reaches the library (which
would take it as device memory)."""
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl


def bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def u8(*shape):
    return torch.zeros(*shape, dtype=torch.uint8)


def test_host_tensors_are_refused():
    with pytest.raises(ValueError, match="CUDA tensor"):
        fl.nvfp4_quantize(bf16(16, 64))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fl.mxfp4_quantize(bf16(16, 64))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fl.nvfp4_gemm(u8(16, 32), u8(512), torch.ones(1), u8(64, 32), u8(512), torch.ones(1))
    with pytest.raises(ValueError, match="CUDA tensor"):
        fl.kv_nvfp4_load_fp8(u8(1, 1, 4, 64), u8(1, 1, 4, 8), torch.ones(1), 4)


def test_wrong_dtypes_are_refused():
    with pytest.raises(TypeError, match="x must be torch.bfloat16"):
        fl.nvfp4_quantize(torch.zeros(16, 64))
    with pytest.raises(TypeError, match="x must be torch.bfloat16"):
        fl.mxfp4_quantize(torch.zeros(16, 64, dtype=torch.float16))
    with pytest.raises(TypeError, match="a_codes must be torch.uint8"):
        fl.nvfp4_gemm(torch.zeros(16, 32, dtype=torch.int8), u8(512), torch.ones(1), u8(64, 32), u8(512),
                      torch.ones(1))
    with pytest.raises(TypeError, match="x must be torch.float32"):
        fl.convert_selftest(torch.zeros(8, dtype=torch.float64))
    with pytest.raises(TypeError, match="kv_new must be torch.bfloat16"):
        fl.kv_nvfp4_store(torch.zeros(1, 1, 1, 64), torch.zeros(1, dtype=torch.int32), torch.ones(1),
                          u8(1, 1, 4, 32), u8(1, 1, 4, 4))


def test_layouts_the_calls_cannot_take_are_refused():
    # a row-strided activation view is fine for the layout check (it then fails on the device)
    with pytest.raises(ValueError, match="CUDA tensor"):
        fl.nvfp4_quantize(bf16(16, 128)[:, :64])
    # a transposed one is not
    with pytest.raises(ValueError, match="unit stride along its rows"):
        fl.nvfp4_quantize(bf16(64, 16).t())
    with pytest.raises(ValueError, match="unit stride along its rows"):
        fl.nvfp4_quantize(bf16(2, 16, 64))
    # codes and scales are read with fixed strides: they must be contiguous
    with pytest.raises(ValueError, match="a_codes must be contiguous"):
        fl.nvfp4_gemm(u8(16, 64)[:, :32], u8(512), torch.ones(1), u8(64, 32), u8(512), torch.ones(1))
    with pytest.raises(ValueError, match="2-D codes tensor"):
        fl.nvfp4_gemm(u8(512), u8(512), torch.ones(1), u8(64, 32), u8(512), torch.ones(1))
    with pytest.raises(ValueError, match="fmt must be"):
        fl.gptq_quantize(bf16(16, 64), torch.zeros(64, 64), "int4")
