"""GPU tests of the layer's composable parts (mxfp4_gather_rows, moe_mxfp4_experts,
moe_mxfp4_combine) and of the expert-parallel module on them.

The parts run the same kernels in the same order as moe_mxfp4_mlp, so route ->
gather -> experts -> combine must reproduce the whole-layer entry point bit for bit
(both modes); the layer itself is checked against the oracle in test_moe_gpu.py.
The expert-parallel layer runs here over a one-rank NCCL group (this pool gives one
GPU), so its exchanges are trivial but its data path is the library's; the
multi-rank bookkeeping is checked on CPU with gloo ranks in test_ep_dist.py."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import moe_expert_gemm_mxfp4_b200 as mx
from moe_expert_gemm_mxfp4_b200 import inputs
from helpers import bits_of

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("n_src,n,row,dtype,div", [(10, 37, 64, torch.bfloat16, 1), (50, 200, 2880, torch.bfloat16, 4),
                                                   (33, 33, 1, torch.float32, 1), (7, 100, 3, torch.float32, 3)])
def test_gather_rows_bit_exact(n_src, n, row, dtype, div):
    g = torch.Generator().manual_seed(n + row)
    src = torch.randn(n_src, row, generator=g).to(dtype).to(DEV)
    idx = torch.randint(0, n_src * div, (n,), generator=g, dtype=torch.int32).to(DEV)
    out = mx.mxfp4_gather_rows(src, idx, div)
    torch.cuda.synchronize()
    assert mx.mxfp4_get_device_status() == 0
    assert torch.equal(out.cpu(), src.cpu()[idx.cpu().long() // div])


def test_gather_rows_reports_an_index_outside_the_source():
    src = torch.ones(4, 8, dtype=torch.float32, device=DEV)
    out = torch.zeros(3, 8, dtype=torch.float32, device=DEV)
    mx.mxfp4_gather_rows(src, torch.tensor([0, 9, 2], dtype=torch.int32, device=DEV), out=out)
    assert mx.mxfp4_get_device_status() == mx._lib.ERR_INVALID_ARG
    o = out.cpu()
    assert torch.equal(o[0], torch.ones(8)) and torch.equal(o[1], torch.zeros(8))   # row left unwritten
    assert mx.mxfp4_get_device_status() == 0                                        # reading cleared it


def _layer(T, H, I, E, k, seed):
    cfg = inputs.MoEConfig("parts", seed=seed, T=T, E=E, top_k=k, H=H, I=I, w_std=0.05)
    x, logits = inputs.moe_activations(cfg)
    q13 = [oracle.quantize(inputs.expert_weights(cfg, e)[0].numpy()) for e in range(E)]
    q2 = [oracle.quantize(inputs.expert_weights(cfg, e)[1].numpy()) for e in range(E)]
    w = [torch.from_numpy(np.stack([a for a, _ in q13])).to(DEV), torch.from_numpy(np.stack([b for _, b in q13])).to(DEV),
         torch.from_numpy(np.stack([a for a, _ in q2])).to(DEV), torch.from_numpy(np.stack([b for _, b in q2])).to(DEV)]
    return x.to(DEV), logits.to(DEV), w


@pytest.mark.parametrize("mode", [mx.W4A16, mx.W4A4])
@pytest.mark.parametrize("T,H,I,E,k", [(37, 192, 128, 8, 2), (300, 256, 320, 32, 4), (64, 2880, 2880, 32, 4)])
def test_parts_reproduce_the_layer(mode, T, H, I, E, k):
    x, logits, w = _layer(T, H, I, E, k, seed=T + I)
    ref = mx.moe_mxfp4_mlp(x, logits, k, *w, mode=mode)
    r = mx.moe_mxfp4_route(logits, k)
    xs = mx.mxfp4_gather_rows(x, r["perm"], k)
    ws = mx.mxfp4_gather_rows(r["weights"].reshape(-1, 1), r["perm"], 1).reshape(-1)
    y = mx.moe_mxfp4_experts(xs, r["offsets"], ws, *w, mode=mode)
    out = mx.moe_mxfp4_combine(y, r["inv"], k)
    torch.cuda.synchronize()
    assert mx.mxfp4_get_device_status() == 0
    assert np.array_equal(bits_of(out), bits_of(ref))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("mode", [mx.W4A16, mx.W4A4])
def test_expert_parallel_layer_on_one_nccl_rank(mode):
    import torch.distributed as dist
    from moe_expert_gemm_mxfp4_b200 import ep
    T, H, I, E, k = 96, 256, 192, 8, 2
    x, logits, w = _layer(T, H, I, E, k, seed=77)
    ref = mx.moe_mxfp4_mlp(x, logits, k, *w, mode=mode)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device(DEV))
    try:
        trace = {}
        out = ep.moe_mlp_ep(x, logits, k, w, ep.ExpertPartition(E, 1), 0, ops=ep.LibraryOps(mode), trace=trace)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert mx.mxfp4_get_device_status() == 0
    assert trace["send_rows"] == [T * k] and trace["recv_rows"] == [T * k]
    assert np.array_equal(bits_of(out), bits_of(ref))


# ---------------------------------------------------------------- bf16-weight comparison layer

def _bf16_layer(T, H, I, E, k, seed):
    cfg = inputs.MoEConfig("bf16w", seed=seed, T=T, E=E, top_k=k, H=H, I=I, w_std=0.05)
    x, logits = inputs.moe_activations(cfg)
    w13 = torch.stack([inputs.expert_weights(cfg, e)[0] for e in range(E)]).to(torch.bfloat16)
    w2 = torch.stack([inputs.expert_weights(cfg, e)[1] for e in range(E)]).to(torch.bfloat16)
    return x, logits, w13, w2


@pytest.mark.parametrize("T,H,I,E,k", [(5, 128, 64, 4, 2), (37, 192, 128, 8, 2), (300, 256, 320, 32, 4),
                                       (64, 2880, 2880, 32, 4), (400, 320, 256, 8, 2), (700, 512, 384, 8, 3),
                                       (2048, 256, 192, 4, 2)])
def test_bf16_weight_layer_against_oracle(T, H, I, E, k):
    x, logits, w13, w2 = _bf16_layer(T, H, I, E, k, seed=T + H)
    out = mx.moe_bf16_mlp(x.to(DEV), logits.to(DEV), k, w13.to(DEV), w2.to(DEV))
    torch.cuda.synchronize()
    assert mx.mxfp4_get_device_status() == 0
    ref = oracle.moe_mlp_dense(bits_of(x), logits.numpy(), k, bits_of(w13), bits_of(w2))
    from helpers import assert_close_tol, f64_of
    assert_close_tol(f64_of(out), ref, what=f"bf16-weight layer T={T} H={H} I={I} E={E} k={k}")
