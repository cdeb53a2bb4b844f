"""CPU oracle for MXFP4 quantization and the MXFP4-weight MoE expert MLP.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously-correct
definition of what the CUDA library computes.  Only ``tests/``, the smoke check
and the benchmark's CPU-baseline leg may import it; the library never does, and
it imports nothing from the library.  It shares no code with the CUDA path.

Floating point is fp64 throughout.  Quantize / dequantize / bf16 rounding live in
plain C (``mxfp4_ref.c``, compiled by ``build.py``); routing and the matrix
products are numpy (fp64 ``@`` is used as the matmul primitive).

Sources (web pages on one subject; cited by page title and section):
  [P4] agentlenshq.com (en), "Transformers 4.40 performance upgrades for OpenAI
       GPT-OSS: zero-build kernels, MXFP4 quantization, parallelism, and faster
       loading" -- sections "What MXFP4 Is", "Native Support in transformers",
       "Memory Savings", "Expert Parallelism (EP)".
  [P2] the zh-CN version of the same summary (same sections).
  [P1] blog.feedonlabs.com, "gpt-oss-transformers-opt" -- its table of numbers.
The pages fix the E2M1 bit split (1 sign, 2 exponent, 1 mantissa) and that 32
consecutive elements share one scale ([P4] "What MXFP4 Is"), and that the MoE
expert MLP runs on MXFP4 weights ([P4] "Zero-Build Kernels from the Hub",
MegaBlocks MoE).  Everything else (scale encoding, rounding, nibble order,
routing rule, gated-SiLU expert MLP) is a reading, stated at the function that
takes it.

Parity pins: every function here is pinned by ``tests/test_oracle.py`` against
values the pages fix, closed forms, invariants or brute force.  The one part
left unpinned beyond the tolerance is the numerical precision of SiLU/exp on
the GPU side ("parity unpinned" for the GPU's transcendental precision only).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

__all__ = [
    "E2M1_GRID", "FLOOR", "CEIL", "e2m1_magnitude", "bf16_to_f64", "f64_to_bf16",
    "quantize", "dequantize_bf16", "dequantize_f64", "route", "gemm_w4a16",
    "gemm_w4a4", "moe_mlp", "moe_down", "silu", "router_logits", "moe_mlp_dense",
]

FLOOR = 0
CEIL = 1
BLOCK = 32

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, vp, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        lib.oracle_e2m1_magnitude.restype = ctypes.c_double
        lib.oracle_e2m1_magnitude.argtypes = [ci]
        lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
        lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_bf16_array.argtypes = [vp, i64, vp]
        for name in ("oracle_quantize_bf16", "oracle_quantize_f32"):
            getattr(lib, name).argtypes = [vp, i64, i64, vp, vp, ci]
        for name in ("oracle_dequantize_f64", "oracle_dequantize_bf16"):
            getattr(lib, name).argtypes = [vp, vp, i64, i64, vp]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def e2m1_magnitude(code: int) -> float:
    """Magnitude of a 3-bit E2M1 magnitude code (2 exponent bits, 1 mantissa bit,
    bias 1) -- [P4] "What MXFP4 Is" fixes the 1/2/1 split; bias 1 is the reading."""
    return float(_load().oracle_e2m1_magnitude(int(code)))


def _grid():
    return np.array([e2m1_magnitude(c) for c in range(8)], dtype=np.float64)


E2M1_GRID = None  # filled lazily by grid()


def grid() -> np.ndarray:
    global E2M1_GRID
    if E2M1_GRID is None:
        E2M1_GRID = _grid()
    return E2M1_GRID


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact fp64 values of bf16 bit patterns (uint16 array)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 to bf16 (round-to-nearest-even, subnormals kept, overflow to
    Inf); returns uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_f64_to_bf16_array(_ptr(x), x.size, _ptr(out))
    return out


def quantize(x: np.ndarray, rule: int = FLOOR, dtype: str | None = None):
    """MXFP4-quantize a 2-D array along its last dimension.

    ``x`` is either float32 values or uint16 bf16 bit patterns (``dtype='bf16'``
    or inferred from a uint16 array).  Returns ``(codes uint8 [R, C/2],
    scales uint8 [R, C/32])``.  Blocks of 32 consecutive elements share one E8M0
    scale ([P4] "What MXFP4 Is"); see ``mxfp4_ref.c`` for the readings taken.
    """
    x = np.ascontiguousarray(x)
    if x.ndim != 2 or x.shape[1] % BLOCK:
        raise ValueError("quantize expects a 2-D array with cols % 32 == 0")
    R, C = x.shape
    codes = np.empty((R, C // 2), dtype=np.uint8)
    scales = np.empty((R, C // BLOCK), dtype=np.uint8)
    lib = _load()
    if dtype == "bf16" or x.dtype == np.uint16:
        x = x.astype(np.uint16, copy=False)
        lib.oracle_quantize_bf16(_ptr(x), R, C, _ptr(codes), _ptr(scales), int(rule))
    elif x.dtype == np.float32:
        lib.oracle_quantize_f32(_ptr(x), R, C, _ptr(codes), _ptr(scales), int(rule))
    else:
        raise TypeError(f"unsupported input dtype {x.dtype}")
    return codes, scales


def _check_packed(codes: np.ndarray, scales: np.ndarray):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    R, half = codes.shape[-2], codes.shape[-1]
    C = 2 * half
    lead = codes.shape[:-2]
    if scales.shape != lead + (R, C // BLOCK):
        raise ValueError("scales shape does not match codes")
    return codes, scales, int(np.prod(lead + (R,))), C, lead + (R, C)


def dequantize_f64(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Exact values code * 2^(S-127) in fp64 (NaN where S = 0xFF)."""
    codes, scales, rows, C, shape = _check_packed(codes, scales)
    out = np.empty(shape, dtype=np.float64)
    _load().oracle_dequantize_f64(_ptr(codes), _ptr(scales), rows, C, _ptr(out))
    return out


def dequantize_bf16(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Dequantize to bf16 bit patterns: the exact product rounded once to bf16."""
    codes, scales, rows, C, shape = _check_packed(codes, scales)
    out = np.empty(shape, dtype=np.uint16)
    _load().oracle_dequantize_bf16(_ptr(codes), _ptr(scales), rows, C, _ptr(out))
    return out


# --------------------------------------------------------------------------- routing

def router_logits(x_bits: np.ndarray, w_router_bits: np.ndarray) -> np.ndarray:
    """Router projection: logits[t, e] = sum_h x[t, h] * W_r[e, h] with bf16 x [T, H]
    and bf16 router weights W_r [E, H], in fp64 (returned unrounded).

    Reading: the pages route each token through the MoE kernel's top-k ([P4]
    "Zero-Build Kernels from the Hub", MegaBlocks MoE) without printing the router;
    the plainest router is a bias-free linear map of the token to one logit per
    expert, its operands in the layer's bf16.
    """
    x = bf16_to_f64(_as_bf16_bits(x_bits))
    w = bf16_to_f64(_as_bf16_bits(w_router_bits))
    return x @ w.T



def route(logits: np.ndarray, top_k: int):
    """Top-k routing, softmax over the k selected logits, and the expert-sorted
    permutation of the (token, slot) pairs.

    Readings (the pages only say the MoE layer routes tokens to experts):
      * experts ordered by (logit descending, expert id ascending), exact fp32
        comparison -- ties go to the lower expert id; a NaN logit ranks below
        every number (-inf included), NaNs among themselves by id (numpy's sort
        places NaN last, and the stable sort keeps ids ascending);
      * w_tj = exp(l_tj - l_t0) / sum_i exp(l_ti - l_t0) over the k selected
        logits, in fp64;
      * pair p = t * k + j; counts[e] = #pairs routed to e; offsets = exclusive
        prefix sum; inside an expert pairs keep ascending p;
        perm[offsets[e] + r] = p, inv[p] = position of p.
    Returns dict(ids int32 [T,k], w f64 [T,k], counts int64 [E],
    offsets int64 [E+1], perm int64 [P], inv int64 [P]).
    """
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    if not (1 <= top_k <= E):
        raise ValueError("top_k out of range")
    # stable sort of -logit keeps the lower expert id first among equal logits
    order = np.argsort(-logits, axis=1, kind="stable")
    ids = order[:, :top_k].astype(np.int32)
    sel = np.take_along_axis(logits, ids.astype(np.int64), axis=1).astype(np.float64)
    z = np.exp(sel - sel[:, :1])
    w = z / z.sum(axis=1, keepdims=True)
    flat = ids.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int64)
    return dict(ids=ids, w=w, counts=counts, offsets=offsets, perm=perm, inv=inv)


# --------------------------------------------------------------------------- GEMM

def _as_bf16_bits(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype != np.uint16:
        raise TypeError("expected bf16 bit patterns (uint16)")
    return np.ascontiguousarray(x)


def _deq_weights(codes, scales) -> np.ndarray:
    """W4A16 weight operand: dequantized to bf16, as exact fp64 values."""
    return bf16_to_f64(dequantize_bf16(codes, scales))


def gemm_w4a16(x_bits: np.ndarray, w_codes: np.ndarray, w_scales: np.ndarray) -> np.ndarray:
    """y = x . dequant(W)^T with bf16 x [M, K] and MXFP4 W [N, K] (blocks along K),
    accumulated in fp64.  Returns the unrounded fp64 result [M, N]."""
    x = bf16_to_f64(_as_bf16_bits(x_bits))
    return x @ _deq_weights(w_codes, w_scales).T


def _fake_quant_bf16(x_bits: np.ndarray) -> np.ndarray:
    """Quantize bf16 values to MXFP4 (floor rule) and dequantize back to fp64."""
    c, s = quantize(x_bits, FLOOR, dtype="bf16")
    return bf16_to_f64(dequantize_bf16(c, s))


def gemm_w4a4(x_bits: np.ndarray, w_codes: np.ndarray, w_scales: np.ndarray) -> np.ndarray:
    """W4A4: x is MXFP4-quantized along K (floor rule) before the product."""
    return _fake_quant_bf16(_as_bf16_bits(x_bits)) @ _deq_weights(w_codes, w_scales).T


# --------------------------------------------------------------------------- MoE MLP

def silu(g: np.ndarray) -> np.ndarray:
    """SiLU(g) = g * sigmoid(g) = g / (1 + exp(-g)), fp64."""
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def moe_mlp(x_bits, logits, top_k, w13_codes, w13_scales, w2_codes, w2_scales,
            mode: str = "w4a16", tokens=None, return_h: bool = False):
    """gpt-oss-style MoE expert MLP with MXFP4 expert weights.

    For each token t and each of its k routed experts e (``route``):
        g = x_t . Wg[e]^T,  u = x_t . Wu[e]^T          (Wg = rows [0, I) of W13,
                                                       Wu = rows [I, 2I))
        h = bf16( SiLU(g) * u )                        (the down GEMM's A16 operand)
        y = h . W2[e]^T
    out_t = sum_j w_tj * y_j, all in fp64 (returned unrounded).
    ``mode='w4a4'`` additionally MXFP4-quantizes x_t and h (blocks along K) before
    each product.  ``tokens`` restricts the computation to a subset of tokens
    (routing is per token, so those rows are exact).
    Shapes: x bf16 bits [T, H]; logits f32 [T, E]; w13 codes [E, 2I, H/2],
    scales [E, 2I, H/32]; w2 codes [E, H, I/2], scales [E, H, I/32].
    Returns out f64 [n_tokens, H] (and h f64 [n_tokens, k, I] if return_h).
    """
    x_bits = _as_bf16_bits(x_bits)
    T, H = x_bits.shape
    E, twoI, _ = w13_codes.shape
    I = twoI // 2
    r = route(logits, top_k)
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    n = tok.size
    xs = x_bits[tok]
    xf = _fake_quant_bf16(xs) if mode == "w4a4" else bf16_to_f64(xs)
    ids = r["ids"][tok]
    w = r["w"][tok]
    out = np.zeros((n, H), dtype=np.float64)
    h_all = np.zeros((n, top_k, I), dtype=np.float64) if return_h else None
    for e in np.unique(ids):
        rows, slots = np.nonzero(ids == e)
        W13 = _deq_weights(w13_codes[e], w13_scales[e])
        g = xf[rows] @ W13[:I].T
        u = xf[rows] @ W13[I:].T
        h_bits = f64_to_bf16(silu(g) * u)
        h = _fake_quant_bf16(h_bits) if mode == "w4a4" else bf16_to_f64(h_bits)
        if return_h:
            h_all[rows, slots] = bf16_to_f64(h_bits)
        W2 = _deq_weights(w2_codes[e], w2_scales[e])
        y = h @ W2.T
        np.add.at(out, rows, w[rows, slots][:, None] * y)
    if return_h:
        return out, h_all
    return out


def moe_down(h_bits, logits, top_k, w2_codes, w2_scales, mode: str = "w4a16", tokens=None):
    """The second half of ``moe_mlp`` from a given h: for each token t and slot j
    with expert e (``route``),
        y = h_tj . W2[e]^T          (``mode='w4a4'``: h_tj MXFP4-quantized first)
    and out_t = sum_j w_tj * y_j in fp64 (returned unrounded).

    h_bits: bf16 bit patterns [n_tokens, top_k, I] of the h rows of ``tokens`` (all
    tokens if None), slot-major per token like ``moe_mlp(..., return_h=True)``.
    This is the staged check's reference: fed with another implementation's h, it
    isolates that implementation's down projection and combine from the rounding
    of h (in W4A4 a last-bit difference in h can flip one of its MXFP4 codes).
    """
    h_bits = _as_bf16_bits(h_bits)
    r = route(logits, top_k)
    T = r["ids"].shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    n, H = tok.size, w2_codes.shape[1]
    ids, w = r["ids"][tok], r["w"][tok]
    out = np.zeros((n, H), dtype=np.float64)
    for e in np.unique(ids):
        rows, slots = np.nonzero(ids == e)
        hb = h_bits[rows, slots]
        h = _fake_quant_bf16(hb) if mode == "w4a4" else bf16_to_f64(hb)
        y = h @ _deq_weights(w2_codes[e], w2_scales[e]).T
        np.add.at(out, rows, w[rows, slots][:, None] * y)
    return out


def moe_mlp_dense(x_bits, logits, top_k, w13_bits, w2_bits, tokens=None):
    """The expert MLP of ``moe_mlp`` with bf16 expert weights instead of MXFP4 ones
    (the pages' bf16 fallback, [P4] "Native Support in transformers"): w13 bf16 bits
    [E, 2I, H] (rows [0, I) gate, [I, 2I) up), w2 bf16 bits [E, H, I]; for each token
    t and slot j with expert e (``route``): g, u = x_t W13[e]^T split, h =
    bf16(SiLU(g) * u), y = h W2[e]^T; out_t = sum_j w_tj * y_j, fp64, unrounded."""
    x_bits = _as_bf16_bits(x_bits)
    T, H = x_bits.shape
    E, twoI, _ = w13_bits.shape
    I = twoI // 2
    r = route(logits, top_k)
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    xf = bf16_to_f64(x_bits[tok])
    ids, w = r["ids"][tok], r["w"][tok]
    out = np.zeros((tok.size, H), dtype=np.float64)
    for e in np.unique(ids):
        rows, slots = np.nonzero(ids == e)
        W13 = bf16_to_f64(_as_bf16_bits(w13_bits[e]))
        g = xf[rows] @ W13[:I].T
        u = xf[rows] @ W13[I:].T
        h = bf16_to_f64(f64_to_bf16(silu(g) * u))
        y = h @ bf16_to_f64(_as_bf16_bits(w2_bits[e])).T
        np.add.at(out, rows, w[rows, slots][:, None] * y)
    return out
