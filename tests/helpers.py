"""Shared test helpers: bf16 <-> bit-pattern conversion and the GEMM tolerance."""
import numpy as np
import torch

import oracle

# Per-element acceptance of a floating-point result: |gpu - ref| <= TOL * max(|ref|, rms(ref)),
# rms over the whole output tensor, ref = the fp64 oracle.
TOL = 8e-3


def bits_of(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def from_bits(b: np.ndarray, device="cpu") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(device)


def f64_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def assert_close_tol(gpu: np.ndarray, ref: np.ndarray, tol: float = TOL, what: str = ""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    rms = float(np.sqrt(np.mean(ref * ref)))
    bound = tol * np.maximum(np.abs(ref), rms)
    err = np.abs(gpu - ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err / bound), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} / {bad.size} elements out of tolerance; worst at {i}: "
            f"gpu={gpu[i]!r} ref={ref[i]!r} bound={bound[i]!r} (rms {rms:.4g})")
    return float((err / np.maximum(np.abs(ref), rms)).max())


def oracle_quantize_weights(w_f32: torch.Tensor):
    """fp32 [rows, K] -> oracle codes/scales (numpy)."""
    return oracle.quantize(w_f32.contiguous().numpy(), oracle.FLOOR)


def _align(v, a=256):
    return (v + a - 1) // a * a


def moe_ws_layout(T, H, I, E, k, w4a4):
    """Byte offsets of the pieces of moe_mxfp4_mlp's workspace, in the order the
    library carves them (256-byte aligned), and the total.  Tests read h (the
    expert-sorted bf16 [T*k, I] output of the gate/up GEMM) from it for the staged
    check; a CPU test keeps the total equal to moe_mxfp4_workspace_size."""
    P = T * k
    off, lay = 0, {}

    def take(name, n):
        nonlocal off
        lay[name] = off
        off = _align(off + n)

    for name, n in (("ids", P * 4), ("weights", P * 4), ("counts", E * 4), ("offsets", (E + 1) * 4),
                    ("perm", P * 4), ("inv", P * 4), ("w_sorted", P * 4),
                    ("route_tmp", ((T + 7) // 8 * E + P) * 4)):
        take(name, n)
    if w4a4:
        take("xq_codes", T * H // 2)
        take("xq_scales", T * H // 32 + 16)
        take("xs_codes", P * H // 2)
        take("xs_scales", P * H // 32 + 16)
    else:
        take("x_sorted", P * H * 2)
    take("h", P * I * 2)
    if w4a4:
        take("hq_codes", P * I // 2)
        take("hq_scales", P * I // 32 + 16)
    take("y_sorted", P * H * 4)
    lay["total"] = off
    return lay


def gpu_h_from_ws(ws, T, H, I, E, k, w4a4, perm):
    """h of every (token, slot) as bf16 bits [T, k, I], read from a workspace that a
    moe_mxfp4_mlp call just used (rows are in expert-sorted order; perm maps sorted
    position -> pair t*k + j)."""
    lay = moe_ws_layout(T, H, I, E, k, w4a4)
    P = T * k
    raw = ws[lay["h"]:lay["h"] + P * I * 2].cpu().numpy().view(np.uint16).reshape(P, I)
    h = np.empty((P, I), dtype=np.uint16)
    h[np.asarray(perm)] = raw
    return h.reshape(T, k, I)
