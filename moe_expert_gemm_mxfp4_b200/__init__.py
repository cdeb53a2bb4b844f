"""MXFP4 quantization and the MXFP4-weight MoE expert MLP on NVIDIA B200 (sm_100a).

Python face of the C-ABI library ``libmxfp4.so`` (``include/mxfp4.h``).  The
functions below carry the C entry points' names and only marshal arguments:
torch tensors provide device memory and the current CUDA stream, and every step
runs in the library's CUDA kernels.  There is no CPU or fallback path: if the
library is missing, calls raise ``Mxfp4LibraryMissing``.

MXFP4 = E2M1 4-bit codes (1 sign, 2 exponent, 1 mantissa bit) with one E8M0
power-of-two scale per 32 consecutive elements (agentlenshq.com, "Transformers
4.40 performance upgrades for OpenAI GPT-OSS ...", section "What MXFP4 Is").
Packed layout: codes uint8 [rows, cols/2] (even element in the low nibble),
scales uint8 [rows, cols/32].
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (Mxfp4Error, Mxfp4LibraryMissing, SCALE_CEIL, SCALE_FLOOR, W4A4, W4A16)

__all__ = [
    "mxfp4_quantize", "mxfp4_dequantize", "mxfp4_gemm", "mxfp4_gemm_workspace_size",
    "mxfp4_token_tile_rows",
    "moe_mxfp4_route", "moe_mxfp4_route_workspace_size", "moe_mxfp4_mlp",
    "moe_mxfp4_workspace_size", "moe_mxfp4_mlp_noalloc", "mxfp4_get_device_status",
    "mxfp4_selftest_wait_timeout", "mxfp4_selftest_mma_rate", "mxfp4_set_trace_events",
    "moe_mxfp4_route_project", "mxfp4_gather_rows", "moe_mxfp4_experts",
    "moe_mxfp4_experts_workspace_size", "moe_mxfp4_combine", "moe_bf16_mlp", "moe_bf16_workspace_size",
    "Mxfp4Error", "Mxfp4LibraryMissing",
    "SCALE_FLOOR", "SCALE_CEIL", "W4A16", "W4A4", "library_path",
]


def library_path() -> str:
    return _lib.LIB_PATH


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, shape=None):
    """Raise unless `t` is a contiguous tensor of this dtype and shape.  The library
    takes raw pointers: a strided view or a wrongly sized operand has to stop here,
    not inside a kernel."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: expected dtype {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")


def _on_current_device(**tensors):
    """Raise unless every given tensor (None = absent) lives on the current CUDA device,
    the one the library launches on: a host tensor would reach a kernel as a bad
    address."""
    cur = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name}: expected a CUDA tensor, got one on {t.device}")
        cur = torch.cuda.current_device() if cur is None else cur
        if t.device.index != cur:
            raise ValueError(f"{name}: on {t.device}, but the library launches on the current "
                             f"device cuda:{cur}")


def _need_dims(t, name, ndim):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim}-D, got shape {tuple(t.shape)}")


def _empty(shape, dtype, like):
    return torch.empty(shape, dtype=dtype, device=like.device)


def mxfp4_quantize(x: torch.Tensor, rule: int = SCALE_FLOOR, codes=None, scales=None, stream=None):
    """x bf16/fp32 [rows, cols] -> (codes uint8 [rows, cols/2], scales uint8 [rows, cols/32])."""
    _need_dims(x, "x", 2)
    R, C = x.shape
    dt = {torch.bfloat16: _lib.IN_BF16, torch.float32: _lib.IN_F32}.get(x.dtype)
    if dt is None:
        raise ValueError(f"x: expected dtype bf16 or fp32, got {x.dtype}")
    _need(x, "x")
    if codes is not None:
        _need(codes, "codes", torch.uint8, (R, C // 2))
    if scales is not None:
        _need(scales, "scales", torch.uint8, (R, C // 32))
    _on_current_device(x=x, codes=codes, scales=scales)
    lib = _lib.load()
    codes = _empty((R, C // 2), torch.uint8, x) if codes is None else codes
    scales = _empty((R, C // 32), torch.uint8, x) if scales is None else scales
    _lib.check("mxfp4_quantize", lib.mxfp4_quantize(_p(x), dt, R, C, _p(codes), _p(scales),
                                                    int(rule), _stream(stream)))
    return codes, scales


def mxfp4_dequantize(codes: torch.Tensor, scales: torch.Tensor, out=None, stream=None):
    """codes uint8 [rows, cols/2] + scales uint8 [rows, cols/32] -> bf16 [rows, cols]."""
    _need_dims(codes, "codes", 2)
    R, half = codes.shape
    C = 2 * half
    _need(codes, "codes", torch.uint8)
    _need(scales, "scales", torch.uint8, (R, C // 32))
    if out is not None:
        _need(out, "out", torch.bfloat16, (R, C))
    _on_current_device(codes=codes, scales=scales, out=out)
    lib = _lib.load()
    out = _empty((R, C), torch.bfloat16, codes) if out is None else out
    _lib.check("mxfp4_dequantize", lib.mxfp4_dequantize(_p(codes), _p(scales), R, C, _p(out),
                                                        _stream(stream)))
    return out


def mxfp4_gemm_workspace_size(M, K, N, mode=W4A16) -> int:
    return int(_lib.load().mxfp4_gemm_workspace_size(M, K, N, int(mode)))


def mxfp4_token_tile_rows(rows, groups=1, mode=W4A16) -> int:
    """Token rows per work tile the grouped GEMMs take for `rows` rows over `groups` groups."""
    return int(_lib.load().mxfp4_token_tile_rows(rows, groups, int(mode)))


def mxfp4_gemm(x: torch.Tensor, w_codes: torch.Tensor, w_scales: torch.Tensor, mode: int = W4A16,
               out=None, ws=None, stream=None):
    """y bf16 [M, N] = x bf16 [M, K] . dequant(W)^T, W codes [N, K/2] + scales [N, K/32]."""
    _need_dims(x, "x", 2)
    _need_dims(w_codes, "w_codes", 2)
    M, K = x.shape
    N = w_codes.shape[0]
    _need(x, "x", torch.bfloat16)
    _need(w_codes, "w_codes", torch.uint8, (N, K // 2))
    _need(w_scales, "w_scales", torch.uint8, (N, K // 32))
    if out is not None:
        _need(out, "out", torch.bfloat16, (M, N))
    if ws is not None:
        _need(ws, "ws")
    _on_current_device(x=x, w_codes=w_codes, w_scales=w_scales, out=out, ws=ws)
    lib = _lib.load()
    out = _empty((M, N), torch.bfloat16, x) if out is None else out
    need = mxfp4_gemm_workspace_size(M, K, N, mode)
    if ws is None and need:
        ws = _empty((need,), torch.uint8, x)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _lib.check("mxfp4_gemm", lib.mxfp4_gemm(_p(x), M, K, _p(w_codes), _p(w_scales), N, _p(out),
                                            int(mode), _p(ws), nbytes, _stream(stream)))
    return out


def moe_mxfp4_route_workspace_size(T, E, top_k) -> int:
    return int(_lib.load().moe_mxfp4_route_workspace_size(T, E, top_k))


def moe_mxfp4_route(logits: torch.Tensor, top_k: int, ws=None, stream=None):
    """Top-k routing + expert-sorted permutation; returns a dict of device tensors
    ids [T, k] i32, weights [T, k] f32, counts [E] i32, offsets [E+1] i32,
    perm [T*k] i32, inv [T*k] i32."""
    _need_dims(logits, "logits", 2)
    _need(logits, "logits", torch.float32)
    if ws is not None:
        _need(ws, "ws")
    _on_current_device(logits=logits, ws=ws)
    lib = _lib.load()
    T, E = logits.shape
    P = T * top_k
    out = dict(ids=_empty((T, top_k), torch.int32, logits),
               weights=_empty((T, top_k), torch.float32, logits),
               counts=_empty((E,), torch.int32, logits),
               offsets=_empty((E + 1,), torch.int32, logits),
               perm=_empty((P,), torch.int32, logits),
               inv=_empty((P,), torch.int32, logits))
    need = moe_mxfp4_route_workspace_size(T, E, top_k)
    ws = _empty((need,), torch.uint8, logits) if ws is None else ws
    _lib.check("moe_mxfp4_route", lib.moe_mxfp4_route(
        _p(logits), T, E, top_k, _p(out["ids"]), _p(out["weights"]), _p(out["counts"]),
        _p(out["offsets"]), _p(out["perm"]), _p(out["inv"]), _p(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    return out


def moe_mxfp4_route_project(x: torch.Tensor, w_router: torch.Tensor, top_k: int, logits_out: bool = False,
                            ws=None, stream=None):
    """Router projection fused with top-k routing: logits = x . w_router^T (bf16
    x [T, H], bf16 w_router [E, H], fp32 accumulation), then the routing of
    ``moe_mxfp4_route``.  Returns the same dict, plus ``logits`` (fp32 [T, E]) when
    ``logits_out`` is set."""
    _need_dims(x, "x", 2)
    _need_dims(w_router, "w_router", 2)
    _need(x, "x", torch.bfloat16)
    T, H = x.shape
    _need(w_router, "w_router", torch.bfloat16, (w_router.shape[0], H))
    if ws is not None:
        _need(ws, "ws")
    _on_current_device(x=x, w_router=w_router, ws=ws)
    lib = _lib.load()
    E = w_router.shape[0]
    P = T * top_k
    out = dict(ids=_empty((T, top_k), torch.int32, x),
               weights=_empty((T, top_k), torch.float32, x),
               counts=_empty((E,), torch.int32, x),
               offsets=_empty((E + 1,), torch.int32, x),
               perm=_empty((P,), torch.int32, x),
               inv=_empty((P,), torch.int32, x))
    if logits_out:
        out["logits"] = _empty((T, E), torch.float32, x)
    need = moe_mxfp4_route_workspace_size(T, E, top_k)
    ws = _empty((need,), torch.uint8, x) if ws is None else ws
    _lib.check("moe_mxfp4_route_project", lib.moe_mxfp4_route_project(
        _p(x), T, H, _p(w_router), E, top_k, _p(out["ids"]), _p(out["weights"]), _p(out["counts"]),
        _p(out["offsets"]), _p(out["perm"]), _p(out["inv"]), _p(out["logits"]) if logits_out else None,
        _p(ws), ws.numel() * ws.element_size(), _stream(stream)))
    return out


def mxfp4_gather_rows(src: torch.Tensor, idx: torch.Tensor, div: int = 1, out=None, stream=None):
    """out[i] = src[idx[i] // div] (rows of a 2-D contiguous tensor; row bytes a
    multiple of 4); idx int32 [n]."""
    _need_dims(src, "src", 2)
    _need(src, "src")
    _need(idx, "idx", torch.int32)
    n = idx.numel()
    if out is None:
        out = _empty((n, src.shape[1]), src.dtype, src)
    else:
        _need(out, "out", src.dtype, (n, src.shape[1]))
    _on_current_device(src=src, idx=idx, out=out)
    _lib.check("mxfp4_gather_rows", _lib.load().mxfp4_gather_rows(
        _p(src), src.shape[0], src.shape[1] * src.element_size(), _p(idx), n, int(div), _p(out),
        _stream(stream)))
    return out


def moe_mxfp4_experts_workspace_size(P, H, I, E, mode=W4A16) -> int:
    return int(_lib.load().moe_mxfp4_experts_workspace_size(P, H, I, E, int(mode)))


def moe_mxfp4_experts(x_sorted: torch.Tensor, offsets: torch.Tensor, row_w: torch.Tensor, w13_codes,
                      w13_scales, w2_codes, w2_scales, mode: int = W4A16, out=None, ws=None, stream=None):
    """The experts on expert-grouped rows: x_sorted bf16 [P, H], offsets int32 [E+1],
    row_w fp32 [P] -> y_sorted fp32 [P, H] = row_w * down(SwiGLU(gate_up(x)))."""
    _need_dims(x_sorted, "x_sorted", 2)
    _need(x_sorted, "x_sorted", torch.bfloat16)
    P, H = x_sorted.shape
    _need_dims(w13_codes, "w13_codes", 3)
    E, twoI, _ = w13_codes.shape
    I = twoI // 2
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need(row_w, "row_w", torch.float32, (P,))
    _need(w13_codes, "w13_codes", torch.uint8, (E, 2 * I, H // 2))
    _need(w13_scales, "w13_scales", torch.uint8, (E, 2 * I, H // 32))
    _need(w2_codes, "w2_codes", torch.uint8, (E, H, I // 2))
    _need(w2_scales, "w2_scales", torch.uint8, (E, H, I // 32))
    if out is None:
        out = _empty((P, H), torch.float32, x_sorted)
    else:
        _need(out, "out", torch.float32, (P, H))
    need = moe_mxfp4_experts_workspace_size(P, H, I, E, mode)
    if ws is None:
        ws = _empty((max(need, 16),), torch.uint8, x_sorted)
    else:
        _need(ws, "ws")
    _on_current_device(x_sorted=x_sorted, offsets=offsets, row_w=row_w, w13_codes=w13_codes,
                       w13_scales=w13_scales, w2_codes=w2_codes, w2_scales=w2_scales, out=out, ws=ws)
    _lib.check("moe_mxfp4_experts", _lib.load().moe_mxfp4_experts(
        _p(x_sorted), P, H, _p(offsets), E, _p(w13_codes), _p(w13_scales), I, _p(w2_codes), _p(w2_scales),
        _p(row_w), _p(out), int(mode), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))
    return out


def moe_mxfp4_combine(y_sorted: torch.Tensor, inv: torch.Tensor, top_k: int, out=None, stream=None):
    """out[t] = bf16(sum_j y_sorted[inv[t*k + j]]) in slot order; y_sorted fp32 [*, H]."""
    _need_dims(y_sorted, "y_sorted", 2)
    _need(y_sorted, "y_sorted", torch.float32)
    _need(inv, "inv", torch.int32)
    H = y_sorted.shape[1]
    T = inv.numel() // top_k
    if out is None:
        out = _empty((T, H), torch.bfloat16, y_sorted)
    else:
        _need(out, "out", torch.bfloat16, (T, H))
    _on_current_device(y_sorted=y_sorted, inv=inv, out=out)
    _lib.check("moe_mxfp4_combine", _lib.load().moe_mxfp4_combine(
        _p(y_sorted), _p(inv), T, top_k, H, _p(out), _stream(stream)))
    return out


def moe_bf16_workspace_size(T, H, I, E, top_k) -> int:
    return int(_lib.load().moe_bf16_workspace_size(T, H, I, E, top_k))


def moe_bf16_mlp(x: torch.Tensor, logits: torch.Tensor, top_k: int, w13: torch.Tensor, w2: torch.Tensor,
                 out=None, ws=None, stream=None):
    """The MoE layer with bf16 expert weights (the comparison for moe_mxfp4_mlp):
    w13 bf16 [E, 2I, H], w2 bf16 [E, H, I]."""
    _need_dims(x, "x", 2)
    _need_dims(logits, "logits", 2)
    _need_dims(w13, "w13", 3)
    T, H = x.shape
    E, twoI, _ = w13.shape
    I = twoI // 2
    _need(x, "x", torch.bfloat16)
    _need(logits, "logits", torch.float32, (T, E))
    _need(w13, "w13", torch.bfloat16, (E, 2 * I, H))
    _need(w2, "w2", torch.bfloat16, (E, H, I))
    if out is None:
        out = _empty((T, H), torch.bfloat16, x)
    else:
        _need(out, "out", torch.bfloat16, (T, H))
    need = moe_bf16_workspace_size(T, H, I, E, top_k)
    if ws is None:
        ws = _empty((need,), torch.uint8, x)
    else:
        _need(ws, "ws")
    _on_current_device(x=x, logits=logits, w13=w13, w2=w2, out=out, ws=ws)
    _lib.check("moe_bf16_mlp", _lib.load().moe_bf16_mlp(
        _p(x), T, H, _p(logits), E, top_k, _p(w13), I, _p(w2), _p(out), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    return out


def _check_moe_operands(x, logits, w13_codes, w13_scales, w2_codes, w2_scales, out):
    """Shapes of one MoE layer's operands, from x [T, H], logits [T, E] and the
    gate/up codes [E, 2I, H/2]; returns (T, H, E, I)."""
    _need_dims(x, "x", 2)
    _need_dims(logits, "logits", 2)
    _need_dims(w13_codes, "w13_codes", 3)
    T, H = x.shape
    E = logits.shape[1]
    if w13_codes.shape[1] % 2:
        raise ValueError(f"w13_codes: expected [E, 2I, H/2], got {tuple(w13_codes.shape)}")
    I = w13_codes.shape[1] // 2
    _need(x, "x", torch.bfloat16)
    _need(logits, "logits", torch.float32, (T, E))
    _need(w13_codes, "w13_codes", torch.uint8, (E, 2 * I, H // 2))
    _need(w13_scales, "w13_scales", torch.uint8, (E, 2 * I, H // 32))
    _need(w2_codes, "w2_codes", torch.uint8, (E, H, I // 2))
    _need(w2_scales, "w2_scales", torch.uint8, (E, H, I // 32))
    if out is not None:
        _need(out, "out", torch.bfloat16, (T, H))
    _on_current_device(x=x, logits=logits, w13_codes=w13_codes, w13_scales=w13_scales,
                       w2_codes=w2_codes, w2_scales=w2_scales, out=out)
    return T, H, E, I


def moe_mxfp4_workspace_size(T, H, I, E, top_k, mode=W4A16) -> int:
    return int(_lib.load().moe_mxfp4_workspace_size(T, H, I, E, top_k, int(mode)))


def moe_mxfp4_mlp(x: torch.Tensor, logits: torch.Tensor, top_k: int, w13_codes, w13_scales,
                  w2_codes, w2_scales, mode: int = W4A16, out=None, ws=None, stream=None):
    """One MoE expert-MLP layer with MXFP4 expert weights (see include/mxfp4.h).
    x bf16 [T, H]; logits f32 [T, E]; w13 codes [E, 2I, H/2] + scales [E, 2I, H/32];
    w2 codes [E, H, I/2] + scales [E, H, I/32] -> out bf16 [T, H]."""
    T, H, E, I = _check_moe_operands(x, logits, w13_codes, w13_scales, w2_codes, w2_scales, out)
    if ws is not None:
        _need(ws, "ws")
        _on_current_device(ws=ws)
    lib = _lib.load()
    out = _empty((T, H), torch.bfloat16, x) if out is None else out
    need = moe_mxfp4_workspace_size(T, H, I, E, top_k, mode)
    ws = _empty((need,), torch.uint8, x) if ws is None else ws
    _lib.check("moe_mxfp4_mlp", lib.moe_mxfp4_mlp(
        _p(x), T, H, _p(logits), E, top_k, _p(w13_codes), _p(w13_scales), I, _p(w2_codes),
        _p(w2_scales), _p(out), int(mode), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    return out


def moe_mxfp4_mlp_noalloc(x: torch.Tensor, logits: torch.Tensor, top_k: int, w13_codes, w13_scales,
                          w2_codes, w2_scales, mode: int = W4A16, out=None, stream=None):
    """The MoE layer of ``moe_mxfp4_mlp`` without a workspace, for callers that must not
    allocate device memory per call (cudaMalloc synchronizes the device and can fail
    under memory pressure).  Its scratch is a fixed 16 MiB array inside the library,
    shared by all calls: calls that overlap on the GPU race on it.  ``out`` is the
    caller's; pass it to keep this call allocation-free on the Python side too."""
    T, H, E, I = _check_moe_operands(x, logits, w13_codes, w13_scales, w2_codes, w2_scales, out)
    lib = _lib.load()
    out = _empty((T, H), torch.bfloat16, x) if out is None else out
    _lib.check("moe_mxfp4_mlp_noalloc", lib.moe_mxfp4_mlp_noalloc(
        _p(x), T, H, _p(logits), E, top_k, _p(w13_codes), _p(w13_scales), I, _p(w2_codes),
        _p(w2_scales), _p(out), int(mode), _stream(stream)))
    return out


def mxfp4_get_device_status(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device status word."""
    return int(_lib.load().mxfp4_get_device_status(_stream(stream)))


def mxfp4_selftest_wait_timeout(stream=None):
    """Launch the failure-detection self-test: one wait that nothing satisfies, which
    gives up after the library's wait limit and records MXFP4_ERR_TIMEOUT."""
    _lib.check("mxfp4_selftest_wait_timeout",
               _lib.load().mxfp4_selftest_wait_timeout(_stream(stream)))


def mxfp4_selftest_mma_rate(kind: int, iters: int, stream=None) -> float:
    """Launch the tensor-pipe rate probe (kind 0: kind::f16 bf16 MMAs, 1: block-scaled
    kind::mxf4 MMAs; one CTA per SM, iters x 4 MMAs of M = 128, N = 256 each) on the
    stream and return the launch's flop count.  Time it with CUDA events."""
    flops = ctypes.c_double(0.0)
    _lib.check("mxfp4_selftest_mma_rate",
               _lib.load().mxfp4_selftest_mma_rate(int(kind), int(iters), ctypes.byref(flops),
                                                   _stream(stream)))
    return flops.value


_trace_keepalive = None


def mxfp4_set_trace_events(events=None):
    """Record the given torch.cuda.Event objects (already created: recorded once)
    at the stage boundaries of subsequent moe_mxfp4_mlp calls on this thread
    (0 start, 1 routed + gathered, 2 gate/up done, 3 down done, 4 combined).
    ``None`` turns tracing off."""
    global _trace_keepalive
    lib = _lib.load()
    if not events:
        _trace_keepalive = None
        lib.mxfp4_set_trace_events(None, 0)
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _trace_keepalive = arr
    lib.mxfp4_set_trace_events(ctypes.cast(arr, ctypes.c_void_p), len(events))
