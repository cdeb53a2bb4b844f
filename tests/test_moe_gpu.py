"""GPU parity of moe_mxfp4_mlp (the whole MoE expert-MLP layer) against the fp64
oracle: every token for small layers and the decode workload, a seeded sample of
tokens (computed one by one by the oracle) for the prefill and 120b-shaped
workloads at full size, in the launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import oracle
import moe_expert_gemm_mxfp4_b200 as mx
from moe_expert_gemm_mxfp4_b200 import inputs
from helpers import assert_close_tol, bits_of, f64_of, gpu_h_from_ws, oracle_quantize_weights

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


class Layer:
    """MoE layer inputs: fp32 weights quantized by the oracle, kept on host and device."""

    def __init__(self, cfg, T=None):
        self.cfg = cfg
        self.x, self.logits = inputs.moe_activations(cfg, T)
        E, I, H = cfg.E, cfg.I, cfg.H
        self.w13c = np.empty((E, 2 * I, H // 2), np.uint8)
        self.w13s = np.empty((E, 2 * I, H // 32), np.uint8)
        self.w2c = np.empty((E, H, I // 2), np.uint8)
        self.w2s = np.empty((E, H, I // 32), np.uint8)
        for e in range(E):
            w13, w2 = inputs.expert_weights(cfg, e)
            self.w13c[e], self.w13s[e] = oracle_quantize_weights(w13)
            self.w2c[e], self.w2s[e] = oracle_quantize_weights(w2)
        self.dev = [torch.from_numpy(a).to(DEV) for a in (self.w13c, self.w13s, self.w2c, self.w2s)]

    def gpu(self, mode=mx.W4A16):
        return self.gpu_ws(mode)[0]

    def gpu_ws(self, mode=mx.W4A16):
        """The layer's output (fp64 view) and the workspace the call used."""
        c = self.cfg
        T = self.x.shape[0]
        ws = torch.empty((mx.moe_mxfp4_workspace_size(T, c.H, c.I, c.E, c.top_k, mode),),
                         dtype=torch.uint8, device=DEV)
        out = mx.moe_mxfp4_mlp(self.x.to(DEV), self.logits.to(DEV), c.top_k, *self.dev, mode=mode, ws=ws)
        torch.cuda.synchronize()
        assert mx.mxfp4_get_device_status() == 0
        return f64_of(out), ws

    def check_w4a4(self, tokens=None, what=""):
        """W4A4 parity with the staged check.  h is rounded to bf16 and then quantized
        to MXFP4 on both sides; the GPU's h comes from fp32 accumulation, the oracle's
        from fp64, so a rare last-bit difference in h can move one element across an
        E2M1 rounding boundary (or a block across a scale boundary).  Both results are
        correct roundings; they differ by one grid step of one h element.  So:
          (1) staged: the oracle's down projection and combine fed with the GPU's h
              must match the GPU's output everywhere;
          (2) the GPU's h must equal the oracle's h on all but a tiny fraction of
              elements (last-bit differences only);
          (3) end to end: every token whose quantized h matches the oracle's is within
              tolerance of the oracle; tokens with a flipped code or scale are few and
              covered by (1)."""
        c = self.cfg
        T = self.x.shape[0]
        out, ws = self.gpu_ws(mx.W4A4)
        r = oracle.route(self.logits.numpy(), c.top_k)
        tok = np.arange(T) if tokens is None else np.asarray(tokens)
        h_gpu = gpu_h_from_ws(ws, T, c.H, c.I, c.E, c.top_k, True, r["perm"])[tok]
        staged = oracle.moe_down(h_gpu, self.logits.numpy(), c.top_k, self.w2c, self.w2s, mode="w4a4",
                                 tokens=tok)
        assert_close_tol(out[tok], staged, what=f"{what} staged (oracle down fed with the GPU's h)")
        ref, h_ref = oracle.moe_mlp(bits_of(self.x), self.logits.numpy(), c.top_k, self.w13c, self.w13s,
                                    self.w2c, self.w2s, mode="w4a4", tokens=tok, return_h=True)
        h_ref = oracle.f64_to_bf16(h_ref)
        diff = h_gpu != h_ref
        assert diff.mean() < 1e-3, f"{what}: GPU h differs from the oracle's in {diff.mean():.2e} of elements"
        n, k, I = h_gpu.shape
        cg, sg = oracle.quantize(h_gpu.reshape(n * k, I), oracle.FLOOR, dtype="bf16")
        cr, sr = oracle.quantize(h_ref.reshape(n * k, I), oracle.FLOOR, dtype="bf16")
        flip = ((cg != cr).any(axis=1) | (sg != sr).any(axis=1)).reshape(n, k).any(axis=1)
        assert flip.mean() <= 0.05, f"{what}: {int(flip.sum())} of {n} tokens with a flipped h code"
        assert_close_tol(out[tok][~flip], ref[~flip], what=f"{what} end to end ({int(flip.sum())} flipped tokens excluded)")
        return out

    def ref(self, mode="w4a16", tokens=None):
        return oracle.moe_mlp(bits_of(self.x), self.logits.numpy(), self.cfg.top_k, self.w13c,
                              self.w13s, self.w2c, self.w2s, mode=mode, tokens=tokens)


def _small(T, H, I, E, k, seed, hot=()):
    return inputs.MoEConfig("small", seed=seed, T=T, E=E, top_k=k, H=H, I=I,
                            hot_experts=hot, hot_bias=2.0 if hot else 0.0, w_std=0.05)


@pytest.mark.parametrize("T,H,I,E,k", [(1, 64, 64, 1, 1), (5, 128, 64, 4, 2), (37, 192, 128, 8, 2),
                                       (64, 256, 320, 16, 4), (300, 128, 192, 5, 3),
                                       (513, 64, 128, 3, 1)])
def test_moe_small_all_tokens(T, H, I, E, k):
    L = Layer(_small(T, H, I, E, k, seed=T + H + I + E + k))
    assert_close_tol(L.gpu(), L.ref(), what=f"moe T={T} H={H} I={I} E={E} k={k}")


def test_moe_small_imbalanced_and_empty_experts():
    L = Layer(_small(200, 128, 128, 12, 2, seed=99, hot=(0, 1)))
    assert_close_tol(L.gpu(), L.ref(), what="imbalanced")


@pytest.fixture(scope="module")
def decode_layer():
    return Layer(inputs.MOE_CONFIGS["moe_decode"])


def test_moe_decode_workload_all_tokens(decode_layer):
    L = decode_layer
    assert_close_tol(L.gpu(), L.ref(), what="decode T=64 E=32")


def _sample(T, n, seed):
    g = torch.Generator().manual_seed(seed)
    return np.sort(torch.randperm(T, generator=g)[:n].numpy())


def test_moe_prefill_workload_sampled():
    L = Layer(inputs.MOE_CONFIGS["moe_prefill"])
    out = L.gpu()
    tok = _sample(L.cfg.T, 96, 1)
    assert_close_tol(out[tok], L.ref(tokens=tok), what="prefill T=8192 (sampled)")
    assert np.all(np.isfinite(out))


@pytest.fixture(scope="module")
def l120():
    return Layer(inputs.MOE_CONFIGS["moe_120b"])


def test_moe_120b_w4a16_sampled(l120):
    out = l120.gpu(mx.W4A16)
    tok = _sample(l120.cfg.T, 64, 2)
    assert_close_tol(out[tok], l120.ref(tokens=tok), what="120b W4A16 (sampled)")


def test_moe_120b_w4a4_sampled(l120):
    l120.check_w4a4(tokens=_sample(l120.cfg.T, 64, 3), what="120b W4A4 (sampled)")


def test_moe_small_w4a4_all_tokens():
    L = Layer(_small(64, 256, 192, 8, 2, seed=5))
    L.check_w4a4(what="small W4A4")


# Token tiles of 32, 64 and 128 rows with both fused epilogues (SwiGLU, weighted), in
# W4A16 and W4A4, every token compared.  The sizes land on the same tile in both engines
# (the library's own tiling query says which).
@pytest.mark.parametrize("mode", [mx.W4A16, mx.W4A4])
@pytest.mark.parametrize("T,H,I,nt", [(160, 384, 320, 32), (208, 256, 192, 32),
                                      (400, 320, 256, 64), (448, 256, 384, 64),
                                      (640, 256, 192, 128)])
def test_moe_mid_token_tiles_all_tokens(mode, T, H, I, nt):
    E, k = 32, 4
    assert mx.mxfp4_token_tile_rows(T * k, E, mode) == nt
    L = Layer(_small(T, H, I, E, k, seed=T + H))
    if mode == mx.W4A16:
        assert_close_tol(L.gpu(mode), L.ref(), what=f"moe T={T} E={E} (NT={nt}) W4A16")
    else:
        L.check_w4a4(what=f"moe T={T} E={E} (NT={nt}) W4A4")


def test_moe_decode_batch_256_tokens_full_size():
    """A 256-token decode batch of the gpt-oss-20b-shaped layer (experts average 32
    routed rows: 64-row token tiles in W4A16, 32-row ones in W4A4), every token
    compared."""
    cfg = inputs.MOE_CONFIGS["moe_decode"]
    L = Layer(cfg, T=256)
    assert mx.mxfp4_token_tile_rows(256 * cfg.top_k, cfg.E, mx.W4A16) == 64
    assert mx.mxfp4_token_tile_rows(256 * cfg.top_k, cfg.E, mx.W4A4) == 32
    assert_close_tol(L.gpu(mx.W4A16), L.ref(), what="decode T=256 W4A16")
    L.check_w4a4(what="decode T=256 W4A4")


# The large token tiles with every token compared at small H, I: 192-row tiles (W4A16)
# and 128-row tiles (W4A4), ragged tails included.
@pytest.mark.parametrize("mode,T,E,k", [(mx.W4A16, 1300, 4, 2), (mx.W4A16, 1000, 3, 1),
                                        (mx.W4A4, 600, 4, 2), (mx.W4A4, 700, 5, 3)])
def test_moe_large_token_tiles_all_tokens(mode, T, E, k):
    L = Layer(_small(T, 128, 192, E, k, seed=T + E + k))
    if mode == mx.W4A16:
        assert mx.mxfp4_token_tile_rows(T * k, E, mode) == 192
        assert_close_tol(L.gpu(mode), L.ref(), what=f"moe T={T} E={E} k={k} W4A16 (192-row tiles)")
    else:
        assert mx.mxfp4_token_tile_rows(T * k, E, mode) == 128
        L.check_w4a4(what=f"moe T={T} E={E} k={k} W4A4 (128-row tiles)")


def test_moe_all_tokens_to_one_expert():
    # a router bias so large that every token's top-1 is expert 0: one group holds all
    # T rows (many token tiles), every other group is empty
    cfg = inputs.MoEConfig("one_expert", seed=3, T=300, E=16, top_k=1, H=128, I=128,
                           hot_experts=(0,), hot_bias=100.0, w_std=0.05)
    L = Layer(cfg)
    assert_close_tol(L.gpu(), L.ref(), what="all tokens to expert 0")


def test_moe_widest_routing():
    # the largest router the kernels take: 256 experts, top-8 (most experts hold a row
    # or two, many none)
    L = Layer(_small(96, 128, 64, 256, 8, seed=256))
    assert_close_tol(L.gpu(), L.ref(), what="E=256 top-8")
    L.check_w4a4(what="E=256 top-8 W4A4")
