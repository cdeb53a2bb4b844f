"""GPU parity of mxfp4_quantize / mxfp4_dequantize against the CPU oracle.

Exactly one correct output exists for codes, scales and dequantized values, so
every comparison is bit-exact (NaN payloads excepted: only NaN-ness is compared).
"""
import numpy as np
import pytest
import torch

import oracle
import moe_expert_gemm_mxfp4_b200 as mx
from moe_expert_gemm_mxfp4_b200 import inputs
from helpers import bits_of, from_bits

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _gpu_quant(x_cpu, rule):
    c, s = mx.mxfp4_quantize(x_cpu.to(DEV), rule)
    torch.cuda.synchronize()
    return c.cpu().numpy(), s.cpu().numpy()


def _oracle_quant(x_cpu, rule):
    if x_cpu.dtype == torch.bfloat16:
        return oracle.quantize(bits_of(x_cpu), rule, dtype="bf16")
    return oracle.quantize(x_cpu.numpy(), rule)


@pytest.mark.parametrize("rule", [mx.SCALE_FLOOR, mx.SCALE_CEIL])
def test_quantize_every_bf16_pattern(rule):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(64, 1024)
    x = from_bits(bits)
    c, s = _gpu_quant(x, rule)
    rc, rs = _oracle_quant(x, rule)
    assert np.array_equal(s, rs)
    assert np.array_equal(c, rc)


@pytest.mark.parametrize("rule", [mx.SCALE_FLOOR, mx.SCALE_CEIL])
def test_quantize_f32_random_and_special(rule):
    g = torch.Generator().manual_seed(7)
    x = torch.randn(37, 320, generator=g) * torch.exp(torch.randn(37, 320, generator=g) * 6)
    x[0, :32] = 0.0
    x[1, :32] = -0.0
    x[2, 5] = float("inf")
    x[3, 40] = float("nan")
    x[4, :32] = torch.tensor([1e-40] * 32)              # fp32 subnormals
    x[5, :32] = 6.0 * 2.0 ** torch.arange(-16, 16).float()
    x[6, 64:96] = 3.4e38
    c, s = _gpu_quant(x, rule)
    rc, rs = _oracle_quant(x, rule)
    assert np.array_equal(s, rs)
    assert np.array_equal(c, rc)


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 96), (7, 4160), (129, 64), (1000, 2880)])
def test_quantize_ragged_shapes(rows, cols):
    x = inputs.seeded_bf16((rows, cols), seed=rows * 7 + cols) * 3
    c, s = _gpu_quant(x, mx.SCALE_FLOOR)
    rc, rs = _oracle_quant(x, mx.SCALE_FLOOR)
    assert np.array_equal(s, rs) and np.array_equal(c, rc)


def test_quantize_full_size_workload():
    """The bf16 [4096, 11520] workload with outliers and all-zero blocks."""
    x = inputs.quant_tensor()
    c, s = _gpu_quant(x, mx.SCALE_FLOOR)
    rc, rs = _oracle_quant(x, mx.SCALE_FLOOR)
    assert np.array_equal(s, rs)
    assert np.array_equal(c, rc)
    # and the dequantized roundtrip, bit-exact
    d = mx.mxfp4_dequantize(torch.from_numpy(c).to(DEV), torch.from_numpy(s).to(DEV))
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(d), oracle.dequantize_bf16(rc, rs))


def test_dequantize_every_scale_and_code():
    codes = np.tile(np.array([c | (c << 4) for c in range(16)], dtype=np.uint8), (256, 1))
    scales = np.arange(256, dtype=np.uint8).reshape(256, 1)
    d = mx.mxfp4_dequantize(torch.from_numpy(codes).to(DEV), torch.from_numpy(scales).to(DEV))
    torch.cuda.synchronize()
    got = bits_of(d)
    ref = oracle.dequantize_bf16(codes, scales)
    nan_ref = (ref & 0x7FFF) > 0x7F80
    nan_got = (got & 0x7FFF) > 0x7F80
    assert np.array_equal(nan_ref, nan_got)
    assert np.array_equal(got[~nan_ref], ref[~nan_ref])


@pytest.mark.parametrize("rows,cols", [(1, 32), (5, 96), (333, 2880)])
def test_dequantize_random_codes(rows, cols):
    g = torch.Generator().manual_seed(rows + cols)
    codes = torch.randint(0, 256, (rows, cols // 2), generator=g, dtype=torch.uint8)
    scales = torch.randint(0, 255, (rows, cols // 32), generator=g, dtype=torch.uint8)
    d = mx.mxfp4_dequantize(codes.to(DEV), scales.to(DEV))
    torch.cuda.synchronize()
    assert np.array_equal(bits_of(d), oracle.dequantize_bf16(codes.numpy(), scales.numpy()))
