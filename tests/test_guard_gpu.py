"""Out-of-bounds evidence for the library's kernels: every output (and the MoE
workspace) is a view into a larger device buffer whose bytes before and after it
hold a canary pattern.  After each call, on ragged shapes (partial tiles in every
dimension), the results must still match the oracle and every canary byte must be
untouched, so a stray store past an output's end or into a neighbour shows up even
where the result itself is right."""
import numpy as np
import pytest
import torch

import oracle
import moe_expert_gemm_mxfp4_b200 as mx
from moe_expert_gemm_mxfp4_b200 import inputs
from helpers import assert_close_tol, bits_of, f64_of, oracle_quantize_weights

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
GUARD = 4096          # canary bytes on each side
CANARY = 0xA5


class Guarded:
    """A device tensor of `shape`/`dtype` placed GUARD bytes into a canary-filled buffer."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.buf = torch.full((GUARD + n + GUARD,), CANARY, dtype=torch.uint8, device=DEV)
        self.t = self.buf[GUARD:GUARD + n].view(dtype).view(shape)

    def check(self, what):
        torch.cuda.synchronize()
        b = self.buf.cpu().numpy()
        head, tail = b[:GUARD], b[GUARD + self.n:]
        bad_head = np.nonzero(head != CANARY)[0]
        bad_tail = np.nonzero(tail != CANARY)[0]
        assert bad_head.size == 0, f"{what}: {bad_head.size} canary bytes overwritten before the output (first at -{GUARD - bad_head[0]})"
        assert bad_tail.size == 0, f"{what}: {bad_tail.size} canary bytes overwritten past the output (first at +{bad_tail[0]})"


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 96), (129, 64), (77, 2880)])
def test_quantize_dequantize_stay_inside_outputs(rows, cols):
    x = inputs.seeded_bf16((rows, cols), seed=rows + cols) * 2
    codes, scales = Guarded((rows, cols // 2), torch.uint8), Guarded((rows, cols // 32), torch.uint8)
    mx.mxfp4_quantize(x.to(DEV), codes=codes.t, scales=scales.t)
    codes.check("quantize codes")
    scales.check("quantize scales")
    rc, rs = oracle.quantize(bits_of(x), oracle.FLOOR, dtype="bf16")
    assert np.array_equal(codes.t.cpu().numpy(), rc) and np.array_equal(scales.t.cpu().numpy(), rs)
    out = Guarded((rows, cols), torch.bfloat16)
    mx.mxfp4_dequantize(codes.t, scales.t, out=out.t)
    out.check("dequantize out")
    assert np.array_equal(bits_of(out.t), oracle.dequantize_bf16(rc, rs))


@pytest.mark.parametrize("mode", [mx.W4A16, mx.W4A4])
@pytest.mark.parametrize("M,K,N", [(1, 64, 1), (17, 192, 200), (100, 512, 129), (257, 704, 331)])
def test_gemm_stays_inside_output_and_workspace(mode, M, K, N):
    g = torch.Generator().manual_seed(M + K + N)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    wc, ws = oracle_quantize_weights(torch.randn(N, K, generator=g) * 0.05)
    y = Guarded((M, N), torch.bfloat16)
    nws = mx.mxfp4_gemm_workspace_size(M, K, N, mode)
    w = Guarded((max(nws, 16),), torch.uint8)
    mx.mxfp4_gemm(x.to(DEV), torch.from_numpy(wc).to(DEV), torch.from_numpy(ws).to(DEV), mode,
                  out=y.t, ws=w.t if nws else None)
    y.check("gemm y")
    w.check("gemm workspace")
    assert mx.mxfp4_get_device_status() == 0
    ref = oracle.gemm_w4a16(bits_of(x), wc, ws) if mode == mx.W4A16 else oracle.gemm_w4a4(bits_of(x), wc, ws)
    assert_close_tol(f64_of(y.t), ref, what=f"gemm {M}x{K}x{N}")


def _moe_layer(T, H, I, E, k, seed):
    cfg = inputs.MoEConfig("guard", seed=seed, T=T, E=E, top_k=k, H=H, I=I, w_std=0.05)
    x, logits = inputs.moe_activations(cfg)
    q13 = [oracle.quantize(inputs.expert_weights(cfg, e)[0].numpy()) for e in range(E)]
    q2 = [oracle.quantize(inputs.expert_weights(cfg, e)[1].numpy()) for e in range(E)]
    w = [np.stack([a for a, _ in q13]), np.stack([b for _, b in q13]),
         np.stack([a for a, _ in q2]), np.stack([b for _, b in q2])]
    return x, logits, w


@pytest.mark.parametrize("mode", [mx.W4A16, mx.W4A4])
@pytest.mark.parametrize("T,H,I,E,k", [(37, 192, 128, 8, 2), (150, 320, 192, 32, 4)])
def test_moe_stays_inside_output_and_workspace(mode, T, H, I, E, k):
    x, logits, w = _moe_layer(T, H, I, E, k, seed=T + E)
    out = Guarded((T, H), torch.bfloat16)
    ws = Guarded((mx.moe_mxfp4_workspace_size(T, H, I, E, k, mode),), torch.uint8)
    mx.moe_mxfp4_mlp(x.to(DEV), logits.to(DEV), k, *(torch.from_numpy(a).to(DEV) for a in w),
                     mode=mode, out=out.t, ws=ws.t)
    out.check("moe out")
    ws.check("moe workspace")
    assert mx.mxfp4_get_device_status() == 0
    ref = oracle.moe_mlp(bits_of(x), logits.numpy(), k, *w, mode="w4a16" if mode == mx.W4A16 else "w4a4")
    assert_close_tol(f64_of(out.t), ref, what=f"moe T={T}")
