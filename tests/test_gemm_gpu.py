"""GPU parity of mxfp4_gemm (W4A16 and W4A4) against the fp64 oracle, within
|gpu - ref| <= 8e-3 * max(|ref|, rms(ref)) per element."""
import numpy as np
import pytest
import torch

import oracle
import moe_expert_gemm_mxfp4_b200 as mx
from moe_expert_gemm_mxfp4_b200 import inputs
from helpers import assert_close_tol, bits_of, f64_of, oracle_quantize_weights

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _run(x_bf16, wc, ws, mode=mx.W4A16):
    y = mx.mxfp4_gemm(x_bf16.to(DEV), torch.from_numpy(wc).to(DEV), torch.from_numpy(ws).to(DEV), mode)
    torch.cuda.synchronize()
    assert mx.mxfp4_get_device_status() == 0
    return f64_of(y)


def test_gemm_small_workload():
    """x bf16 [8, 256] x MXFP4 W [512, 256] (the single-GEMM workload)."""
    x, w = inputs.gemm_small()
    wc, ws = oracle_quantize_weights(w)
    y = _run(x, wc, ws)
    ref = oracle.gemm_w4a16(bits_of(x), wc, ws)
    assert_close_tol(y, ref, what="gemm 8x256x512")


@pytest.mark.parametrize("M,K,N", [(1, 64, 1), (3, 64, 130), (16, 128, 128), (17, 192, 200),
                                   (40, 256, 256), (64, 320, 384), (100, 512, 129),
                                   (257, 704, 640), (500, 512, 384), (777, 1024, 256),
                                   (1024, 2880, 2880)])
def test_gemm_shapes(M, K, N):
    g = torch.Generator().manual_seed(M * 7 + K + N)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = torch.randn(N, K, generator=g) * 0.05
    wc, ws = oracle_quantize_weights(w)
    y = _run(x, wc, ws)
    assert_close_tol(y, oracle.gemm_w4a16(bits_of(x), wc, ws), what=f"gemm {M}x{K}x{N}")


def test_gemm_closed_form_rowsum():
    """All codes 1.0, scale S: y = 2^(S-127) * rowsum(x) (exact products)."""
    M, K, N = 8, 256, 256
    g = torch.Generator().manual_seed(3)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    wc = np.full((N, K // 2), 0x22, dtype=np.uint8)
    ws = np.full((N, K // 32), 120, dtype=np.uint8)
    y = _run(x, wc, ws)
    ref = np.repeat(x.double().numpy().sum(axis=1, keepdims=True) * 2.0 ** -7, N, axis=1)
    assert_close_tol(y, ref, what="rowsum")


def test_gemm_one_hot_selects_weight_column():
    M, K, N = 16, 128, 300
    g = torch.Generator().manual_seed(4)
    w = torch.randn(N, K, generator=g) * 0.05
    wc, ws = oracle_quantize_weights(w)
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    for m in range(M):
        x[m, (m * 37) % K] = 1.0
    y = _run(x, wc, ws)
    W = oracle.dequantize_f64(wc, ws)
    for m in range(M):
        col = W[:, (m * 37) % K]
        assert np.array_equal(y[m], oracle.bf16_to_f64(oracle.f64_to_bf16(col)))


def test_gemm_extreme_scales_use_exact_path():
    """Scale bytes 0 and 1 (subnormal results) take the exact dequant path, 2 and
    250..252 the fast one; with a one-hot x every output is one weight (kept
    finite: an Inf weight would turn the zero products into NaN)."""
    M, K, N = 16, 64, 128
    g = torch.Generator().manual_seed(5)
    wc = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8).numpy()
    ws = np.array([[0, 1], [2, 250], [251, 252]] * 43, dtype=np.uint8)[:N]
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    for m in range(M):
        x[m, m * 4] = 1.0
    y = mx.mxfp4_gemm(x.to(DEV), torch.from_numpy(wc).to(DEV), torch.from_numpy(ws).to(DEV))
    torch.cuda.synchronize()
    got = f64_of(y)
    deq = oracle.bf16_to_f64(oracle.dequantize_bf16(wc, ws))
    for m in range(M):
        assert np.array_equal(got[m], deq[:, m * 4])


@pytest.mark.parametrize("M,K,N", [(1, 64, 1), (8, 256, 512), (16, 128, 128), (17, 192, 200),
                                   (33, 448, 130), (64, 320, 384), (300, 1024, 512),
                                   (257, 704, 640), (1024, 2880, 2880)])
def test_gemm_w4a4(M, K, N):
    g = torch.Generator().manual_seed(M + K + N + 1)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = torch.randn(N, K, generator=g) * 0.05
    wc, ws = oracle_quantize_weights(w)
    y = _run(x, wc, ws, mx.W4A4)
    assert_close_tol(y, oracle.gemm_w4a4(bits_of(x), wc, ws), what=f"w4a4 {M}x{K}x{N}")


@pytest.mark.parametrize("M", [5, 40, 100, 200])
def test_gemm_w4a4_one_hot_selects_weight_column(M):
    """x rows with a single 1.0 are on the MXFP4 grid (block scale 2^-2, code 4):
    every output is one product of block-scaled E2M1 values, so y[m] equals the
    bf16 of dequantized weight column k exactly; a misplaced weight or activation
    block scale shows up as a power-of-two error."""
    K, N = 512, 300
    g = torch.Generator().manual_seed(40 + M)
    w = torch.randn(N, K, generator=g) * 0.05
    wc, ws = oracle_quantize_weights(w)
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    for m in range(M):
        x[m, (m * 37) % K] = 1.0
    y = _run(x, wc, ws, mx.W4A4)
    W = oracle.dequantize_f64(wc, ws)
    for m in range(M):
        col = W[:, (m * 37) % K]
        assert np.array_equal(y[m], oracle.bf16_to_f64(oracle.f64_to_bf16(col))), m


def test_gemm_w4a4_equals_w4a16_on_grid_activations():
    """Activations already on the MXFP4 grid (dequantized random codes) quantize to
    themselves, so W4A4 and W4A16 compute the same products; they differ only in
    fp32 summation order."""
    M, K, N = 96, 768, 384
    g = torch.Generator().manual_seed(11)
    xc = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.uint8).numpy()
    xs = torch.randint(118, 130, (M, K // 32), generator=g, dtype=torch.uint8).numpy()
    x = torch.from_numpy(oracle.dequantize_bf16(xc, xs).view(np.int16)).view(torch.bfloat16)
    w = torch.randn(N, K, generator=g) * 0.05
    wc, ws = oracle_quantize_weights(w)
    y4 = _run(x, wc, ws, mx.W4A4)
    y16 = _run(x, wc, ws, mx.W4A16)
    assert_close_tol(y4, y16, what="w4a4 vs w4a16 on grid")


@pytest.mark.parametrize("M", [20, 100, 400])   # 32-, 128- and 192-row token tiles
@pytest.mark.parametrize("scales", ["subnormal", "mixed"])
def test_gemm_every_dequant_route(M, scales):
    """Weights of random codes and scale bytes, so that the fast path (LUT value times
    2^(S-127) in one bf16x2 multiply, S in 2..254) and the exact fp32 route (S = 0, 1:
    subnormal weights) meet in the same tile, for each token tiling."""
    K, N = 512, 256
    g = torch.Generator().manual_seed(M + (0 if scales == "subnormal" else 1))
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    wc = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8).numpy()
    if scales == "subnormal":   # 30% of the blocks at S = 0, 1 (subnormal weights), the rest normal
        tiny = torch.rand((N, K // 32), generator=g) < 0.3
        ws = torch.where(tiny, torch.randint(0, 2, (N, K // 32), generator=g),
                         torch.randint(120, 128, (N, K // 32), generator=g)).to(torch.uint8).numpy()
    else:
        ws = torch.randint(120, 160, (N, K // 32), generator=g, dtype=torch.uint8).numpy()  # both routes
    y = _run(x, wc, ws)
    assert_close_tol(y, oracle.gemm_w4a16(bits_of(x), wc, ws), what=f"gemm {M}x{K}x{N} scales {scales}")


def test_gemm_largest_k():
    # K = 7680, the largest contraction the W4A16 engine accepts (the tile's block
    # scales are staged whole in shared memory next to the rings)
    M, K, N = 40, 7680, 256
    g = torch.Generator().manual_seed(7680)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = torch.randn(N, K, generator=g) * 0.02
    wc, ws = oracle_quantize_weights(w)
    y = _run(x, wc, ws)
    assert_close_tol(y, oracle.gemm_w4a16(bits_of(x), wc, ws), what=f"gemm {M}x{K}x{N}")
