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
