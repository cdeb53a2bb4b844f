"""GPU parity of moe_mxfp4_route against the oracle: ids, counts, offsets, perm
and inv bit-exact; softmax weights within 1e-6 relative of the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import moe_expert_gemm_mxfp4_b200 as mx
from moe_expert_gemm_mxfp4_b200 import inputs
from helpers import bits_of

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


def _check_project(x, w, k, what):
    """moe_mxfp4_route_project against the oracle: (1) its fp32 logits within fp32
    accumulation error of the fp64 router projection; (2) the routing of those
    logits bit-exact (oracle.route on the GPU's own logits); (3) the ids equal the
    fp64 router's wherever the k-th and (k+1)-th logits are further apart than the
    error bound (elsewhere both choices are correct roundings)."""
    r = mx.moe_mxfp4_route_project(x.to(DEV), w.to(DEV), k, logits_out=True)
    torch.cuda.synchronize()
    assert mx.mxfp4_get_device_status() == 0
    T, H = x.shape
    gl = r["logits"].cpu().numpy()
    xb, wb = bits_of(x), bits_of(w)
    ref = oracle.router_logits(xb, wb)
    absdot = np.abs(x.double().numpy()) @ np.abs(w.double().numpy()).T
    bound = H * 2.0 ** -24 * absdot + 1e-30
    err = np.abs(gl.astype(np.float64) - ref)
    assert np.all(err <= bound), f"{what}: logits off by {float((err / bound).max()):.2f} x the fp32 bound"
    ro = oracle.route(gl, k)
    for key in ("ids", "counts", "offsets", "perm", "inv"):
        assert np.array_equal(r[key].cpu().numpy(), ro[key]), (what, key)
    w_gpu = r["weights"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(w_gpu - ro["w"]) <= 1e-6 * np.abs(ro["w"]) + 1e-7), what
    r64 = oracle.route(ref, k)
    srt = np.sort(ref, axis=1)[:, ::-1]
    E = ref.shape[1]
    gap = srt[:, k - 1] - srt[:, k] if k < E else np.full(T, np.inf)
    clear = gap > 2 * bound.max(axis=1)
    same = (np.sort(r["ids"].cpu().numpy(), axis=1) == np.sort(r64["ids"], axis=1)).all(axis=1)
    assert same[clear].all(), f"{what}: ids differ from the fp64 router on a clear-cut token"
    return clear.mean()


# the K split runs over clusters of 1 (H = 64, or T large enough to fill the SMs with
# tiles: T = 10000), 2, 4 (E > 64) and 8 CTAs
@pytest.mark.parametrize("T,H,E,k", [(1, 64, 1, 1), (37, 128, 8, 2), (50, 192, 20, 3), (130, 256, 256, 8),
                                     (200, 2880, 32, 4), (300, 2880, 128, 4), (1000, 2880, 32, 4),
                                     (129, 640, 48, 6), (10000, 256, 16, 2)])
def test_route_project_shapes(T, H, E, k):
    g = torch.Generator().manual_seed(T + H + E)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    w = (torch.randn(E, H, generator=g) * H ** -0.5).to(torch.bfloat16)
    _check_project(x, w, k, f"route_project T={T} H={H} E={E} k={k}")


@pytest.mark.parametrize("name", ["moe_decode", "moe_prefill", "moe_120b"])
def test_route_project_workloads(name):
    cfg = inputs.MOE_CONFIGS[name]
    x, _ = inputs.moe_activations(cfg)
    clear = _check_project(x, inputs.router_weights(cfg), cfg.top_k, f"route_project {name}")
    assert clear > 0.8     # the bound is worst-case; most tokens are still clear-cut


def test_route_project_ties_resolve_to_lower_ids():
    # identical router rows give exactly equal logits: ids must be the lower ones
    T, H, E, k = 20, 128, 16, 4
    g = torch.Generator().manual_seed(5)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    w = (torch.randn(E, H, generator=g) * 0.1).to(torch.bfloat16)
    w[9] = w[2]
    w[12] = w[2]
    w[7] = w[3]
    r = mx.moe_mxfp4_route_project(x.to(DEV), w.to(DEV), k, logits_out=True)
    torch.cuda.synchronize()
    ro = oracle.route(r["logits"].cpu().numpy(), k)
    assert np.array_equal(r["ids"].cpu().numpy(), ro["ids"])


def test_route_project_zero_tokens_tie_across_signed_zeros():
    # a zero token's logits are all zeros, some of them -0 (negative weights): +0 and
    # -0 are equal logits, so the lowest ids win and the weights are uniform
    T, H, E, k = 40, 256, 32, 4
    g = torch.Generator().manual_seed(11)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    x[::3] = 0.0
    w = (torch.randn(E, H, generator=g) * H ** -0.5).to(torch.bfloat16)
    r = mx.moe_mxfp4_route_project(x.to(DEV), w.to(DEV), k, logits_out=True)
    torch.cuda.synchronize()
    assert mx.mxfp4_get_device_status() == 0
    ids, wts = r["ids"].cpu().numpy(), r["weights"].cpu().numpy()
    for t in range(0, T, 3):
        assert np.all(r["logits"].cpu().numpy()[t] == 0.0)
        assert list(ids[t]) == list(range(k)), (t, ids[t])
        assert np.allclose(wts[t], 1.0 / k, rtol=1e-6)
    ro = oracle.route(r["logits"].cpu().numpy(), k)
    assert np.array_equal(ids, ro["ids"])
