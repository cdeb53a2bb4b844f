"""The allocation-free MoE entry point (moe_mxfp4_mlp_noalloc) against the regular one.

moe_mxfp4_mlp_noalloc serves callers that must not allocate device memory per call
(cudaMalloc / cudaFree synchronize the device and can fail under memory pressure): it
runs the same layer on a fixed scratch array inside the library instead of a caller
workspace.  Its output must match moe_mxfp4_mlp's within the layer tolerance, on
consecutive calls that reuse the same scratch, and calls too large for the scratch
must be refused.  This file is collected last so a failure here cannot hide others.
"""
import numpy as np
import pytest
import torch

import moe_expert_gemm_mxfp4_b200 as mx
from moe_expert_gemm_mxfp4_b200 import _lib
from helpers import assert_close_tol, f64_of

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _layer(seed, T, H, I, E, k):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16).to(DEV)
    logits = torch.randn(T, E, generator=g).to(DEV)
    w13c = torch.randint(0, 256, (E, 2 * I, H // 2), generator=g, dtype=torch.uint8).to(DEV)
    w13s = torch.randint(118, 124, (E, 2 * I, H // 32), generator=g, dtype=torch.uint8).to(DEV)
    w2c = torch.randint(0, 256, (E, H, I // 2), generator=g, dtype=torch.uint8).to(DEV)
    w2s = torch.randint(118, 124, (E, H, I // 32), generator=g, dtype=torch.uint8).to(DEV)
    return x, logits, k, w13c, w13s, w2c, w2s


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # decode-shaped layer first, then a different shape that reuses the scratch the
    # first call left behind
    # (the third case takes the 32-row token tile: its experts average 20 routed rows)
    cases = [(1, 64, 2880, 2880, 32, 4), (2, 40, 512, 256, 6, 3), (4, 160, 384, 320, 32, 4)]
    for mode in (mx.W4A16, mx.W4A4):
        for seed, T, H, I, E, k in cases:
            args = _layer(seed, T, H, I, E, k)
            ref = mx.moe_mxfp4_mlp(*args, mode=mode)
            out = torch.empty_like(ref)
            got = mx.moe_mxfp4_mlp_noalloc(*args, mode=mode, out=out)
            torch.cuda.synchronize()
            assert mx.mxfp4_get_device_status() == 0
            assert_close_tol(f64_of(got), f64_of(ref), what=f"noalloc T={T} H={H} I={I} E={E} k={k}")


def test_noalloc_refuses_layers_larger_than_its_scratch():
    T, H, I, E, k = 200, 2880, 2880, 32, 4   # ~18.5 MB of scratch needed
    assert mx.moe_mxfp4_workspace_size(T, H, I, E, k) > _lib.NOALLOC_SCRATCH_BYTES
    args = _layer(3, T, H, I, E, k)
    with pytest.raises(mx.Mxfp4Error) as ei:
        mx.moe_mxfp4_mlp_noalloc(*args)
    assert ei.value.status == _lib.ERR_WORKSPACE
