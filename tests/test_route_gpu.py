"""GPU parity of moe_mxfp4_route against the oracle: ids, counts, offsets, perm
and inv bit-exact; softmax weights within 1e-6 relative of the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import moe_expert_gemm_mxfp4_b200 as mx
from moe_expert_gemm_mxfp4_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _check(logits, k):
    r = mx.moe_mxfp4_route(logits.to(DEV), k)
    torch.cuda.synchronize()
    ref = oracle.route(logits.numpy(), k)
    assert np.array_equal(r["ids"].cpu().numpy(), ref["ids"])
    assert np.array_equal(r["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(r["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(r["perm"].cpu().numpy(), ref["perm"])
    assert np.array_equal(r["inv"].cpu().numpy(), ref["inv"])
    w = r["weights"].cpu().numpy().astype(np.float64)
    nan = np.isnan(ref["w"])
    assert np.array_equal(np.isnan(w), nan)
    assert np.all(np.abs(w - ref["w"])[~nan] <= 1e-6 * np.abs(ref["w"][~nan]) + 1e-7)


# Shapes at the routing's limits (top-8 of 256 experts, top-1 of a few) and a token
# count off the 8-token chunk boundary on either side of 256 pairs.
@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (5, 4, 2), (63, 8, 3), (64, 32, 4), (65, 33, 4),
                                   (200, 256, 8), (1000, 128, 4), (130, 7, 7), (32, 256, 8),
                                   (256, 32, 1), (1, 256, 8), (257, 4, 1), (33, 256, 8)])
def test_route_small(T, E, k):
    g = torch.Generator().manual_seed(T * 1000 + E)
    logits = torch.randn(T, E, generator=g)
    _check(logits, k)


@pytest.mark.parametrize("T", [70, 60])
def test_route_ties_and_infinities(T):
    E, k = 16, 4
    logits = torch.zeros(T, E)
    logits[1::3, 5] = 1.0
    logits[2::5, [3, 9, 12]] = 2.0
    logits[4, :] = float("-inf")
    logits[4, 7] = 0.0
    logits[6, 2] = 3.0
    _check(logits, k)


@pytest.mark.parametrize("name", ["moe_decode", "moe_prefill", "moe_120b"])
def test_route_workloads(name):
    cfg = inputs.MOE_CONFIGS[name]
    _, logits = inputs.moe_activations(cfg)
    _check(logits, cfg.top_k)


def test_route_nan_logits():
    # NaN logits rank below every number (-inf included), NaNs among themselves by id;
    # a token that has to select a NaN gets NaN weights on every slot
    T, E, k = 45, 40, 4
    g = torch.Generator().manual_seed(7)
    logits = torch.randn(T, E, generator=g)
    logits[0, [1, 4, 33]] = float("nan")
    logits[1, :] = float("nan")
    logits[2, :] = float("nan")
    logits[2, [5, 39]] = 1.0
    logits[3, 10:] = float("-inf")
    logits[3, :10] = float("nan")
    logits[9::4, 0] = float("nan")
    _check(logits, k)
