"""The Python binding refuses operands the C library cannot take, before it loads the
library or touches a GPU: wrong dtype, wrong shape, a strided view, or a host tensor.
The library takes raw device pointers, so each of these would otherwise reach a
kernel as a bad address.  All tensors here live on the CPU."""
import pytest
import torch

import moe_expert_gemm_mxfp4_b200 as mx

u8, bf16, f32 = torch.uint8, torch.bfloat16, torch.float32


def test_quantize_operands():
    with pytest.raises(ValueError, match="2-D"):
        mx.mxfp4_quantize(torch.zeros(2, 3, 64, dtype=bf16))
    with pytest.raises(ValueError, match="dtype"):
        mx.mxfp4_quantize(torch.zeros(4, 64, dtype=torch.float16))
    with pytest.raises(ValueError, match="contiguous"):
        mx.mxfp4_quantize(torch.zeros(64, 64, dtype=bf16).t())
    with pytest.raises(ValueError, match="CUDA"):
        mx.mxfp4_quantize(torch.zeros(4, 64, dtype=bf16))
    with pytest.raises(TypeError):
        mx.mxfp4_quantize([[0.0] * 64])


def test_quantize_outputs_must_match_the_input():
    x = torch.zeros(4, 64, dtype=bf16)
    with pytest.raises(ValueError, match="codes: expected shape"):
        mx.mxfp4_quantize(x, codes=torch.zeros(4, 64, dtype=u8))
    with pytest.raises(ValueError, match="scales: expected dtype"):
        mx.mxfp4_quantize(x, scales=torch.zeros(4, 2, dtype=torch.int32))


def test_dequantize_operands():
    with pytest.raises(ValueError, match="dtype"):
        mx.mxfp4_dequantize(torch.zeros(4, 32, dtype=torch.int8), torch.zeros(4, 2, dtype=u8))
    with pytest.raises(ValueError, match="scales: expected shape"):
        mx.mxfp4_dequantize(torch.zeros(4, 32, dtype=u8), torch.zeros(4, 4, dtype=u8))
    with pytest.raises(ValueError, match="out: expected shape"):
        mx.mxfp4_dequantize(torch.zeros(4, 32, dtype=u8), torch.zeros(4, 2, dtype=u8),
                            out=torch.zeros(4, 32, dtype=bf16))
    with pytest.raises(ValueError, match="CUDA"):
        mx.mxfp4_dequantize(torch.zeros(4, 32, dtype=u8), torch.zeros(4, 2, dtype=u8))


def test_gemm_operands():
    x = torch.zeros(8, 256, dtype=bf16)
    with pytest.raises(ValueError, match="dtype"):
        mx.mxfp4_gemm(x.float(), torch.zeros(512, 128, dtype=u8), torch.zeros(512, 8, dtype=u8))
    with pytest.raises(ValueError, match="w_codes: expected shape"):
        mx.mxfp4_gemm(x, torch.zeros(512, 256, dtype=u8), torch.zeros(512, 8, dtype=u8))
    with pytest.raises(ValueError, match="w_scales: expected shape"):
        mx.mxfp4_gemm(x, torch.zeros(512, 128, dtype=u8), torch.zeros(256, 8, dtype=u8))
    with pytest.raises(ValueError, match="CUDA"):
        mx.mxfp4_gemm(x, torch.zeros(512, 128, dtype=u8), torch.zeros(512, 8, dtype=u8))
    with pytest.raises(ValueError, match="2-D"):
        mx.mxfp4_gemm(x, torch.zeros(512 * 128, dtype=u8), torch.zeros(512, 8, dtype=u8))


def test_route_operands():
    with pytest.raises(ValueError, match="dtype"):
        mx.moe_mxfp4_route(torch.zeros(8, 32, dtype=torch.float64), 4)
    with pytest.raises(ValueError, match="CUDA"):
        mx.moe_mxfp4_route(torch.zeros(8, 32, dtype=f32), 4)


def _moe(T=8, H=128, I=64, E=4, **override):
    ops = dict(x=torch.zeros(T, H, dtype=bf16), logits=torch.zeros(T, E, dtype=f32),
               w13_codes=torch.zeros(E, 2 * I, H // 2, dtype=u8),
               w13_scales=torch.zeros(E, 2 * I, H // 32, dtype=u8),
               w2_codes=torch.zeros(E, H, I // 2, dtype=u8), w2_scales=torch.zeros(E, H, I // 32, dtype=u8))
    ops.update(override)
    return ops


@pytest.mark.parametrize("fn", [mx.moe_mxfp4_mlp, mx.moe_mxfp4_mlp_noalloc])
def test_moe_operands(fn):
    def call(**kw):
        o = _moe(**kw)
        return fn(o["x"], o["logits"], 2, o["w13_codes"], o["w13_scales"], o["w2_codes"], o["w2_scales"])

    with pytest.raises(ValueError, match="dtype"):
        call(x=torch.zeros(8, 128, dtype=f32))
    with pytest.raises(ValueError, match="3-D"):
        call(w13_codes=torch.zeros(4 * 128, 64, dtype=u8))
    with pytest.raises(ValueError, match="logits: expected shape"):
        call(logits=torch.zeros(7, 4, dtype=f32))
    with pytest.raises(ValueError, match="w13_scales: expected shape"):
        call(w13_scales=torch.zeros(4, 128, 8, dtype=u8))
    with pytest.raises(ValueError, match="w2_codes: expected shape"):
        call(w2_codes=torch.zeros(4, 64, 64, dtype=u8))
    with pytest.raises(ValueError, match="w2_scales: expected dtype"):
        call(w2_scales=torch.zeros(4, 128, 2, dtype=torch.int8))
    with pytest.raises(ValueError, match="contiguous"):
        call(w2_codes=torch.zeros(4, 32, 128, dtype=u8).transpose(1, 2))
    with pytest.raises(ValueError, match="x: expected a CUDA tensor"):   # consistent shapes
        call()


class _FakeLib:
    """Stands in for libmxfp4.so: records each entry point's arguments, returns OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return 64 if name.endswith("workspace_size") else 0
        return fn


@pytest.fixture
def fake(monkeypatch):
    lib = _FakeLib()
    monkeypatch.setattr(mx._lib, "load", lambda *a, **k: lib)
    monkeypatch.setattr(mx, "_on_current_device", lambda **k: None)
    monkeypatch.setattr(mx, "_stream", lambda stream=None: None)
    return lib


def test_operands_shaped_like_the_callers_reach_the_library(fake):
    # quantize / dequantize as the tests and the benchmark call them
    x = torch.zeros(64, 2880, dtype=bf16)
    c, s = mx.mxfp4_quantize(x)
    assert c.shape == (64, 1440) and s.shape == (64, 90)
    w13c = torch.zeros(4, 2 * 192, 256 // 2, dtype=u8)
    w13s = torch.zeros(4, 2 * 192, 256 // 32, dtype=u8)
    mx.mxfp4_quantize(torch.zeros(384, 256), codes=w13c[1], scales=w13s[1])   # per-expert slices
    out = mx.mxfp4_dequantize(c, s)
    mx.mxfp4_dequantize(c, s, out=out)
    mx.mxfp4_dequantize(torch.zeros(256, 16, dtype=u8), torch.zeros(256, 1, dtype=u8))
    # GEMM in both modes, with and without caller buffers
    xg = torch.zeros(8, 256, dtype=bf16)
    wc, ws = torch.zeros(512, 128, dtype=u8), torch.zeros(512, 8, dtype=u8)
    y = mx.mxfp4_gemm(xg, wc, ws)
    mx.mxfp4_gemm(xg, wc, ws, mx.W4A4, out=y, ws=torch.zeros(4096, dtype=u8))
    # routing, and the MoE layer with the smoke test's shapes
    mx.moe_mxfp4_route(torch.zeros(48, 8, dtype=f32), 2)
    T, H, I, E = 48, 256, 192, 8
    args = (torch.zeros(T, H, dtype=bf16), torch.zeros(T, E, dtype=f32), 2,
            torch.zeros(E, 2 * I, H // 2, dtype=u8), torch.zeros(E, 2 * I, H // 32, dtype=u8),
            torch.zeros(E, H, I // 2, dtype=u8), torch.zeros(E, H, I // 32, dtype=u8))
    o = mx.moe_mxfp4_mlp(*args)
    mx.moe_mxfp4_mlp(*args, mode=mx.W4A4, out=o, ws=torch.zeros(1 << 20, dtype=u8))
    mx.moe_mxfp4_mlp_noalloc(*args, out=o)
    for name in ("mxfp4_quantize", "mxfp4_dequantize", "mxfp4_gemm", "moe_mxfp4_route",
                 "moe_mxfp4_mlp", "moe_mxfp4_mlp_noalloc"):
        assert name in fake.calls
