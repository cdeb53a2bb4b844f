"""Expert parallelism on CPU: two (and three) gloo ranks run moe_mlp_ep, each holding a
contiguous range of the experts and its own tokens, with the oracle as the compute
(routing, the experts' products, the combine).  The exchange bookkeeping of the
ep module must reproduce the single-process oracle layer: routing tables bit for
bit for every rank's tokens, exchange sizes equal to the global routing's per-rank
pair counts, and the output equal up to fp64 summation order.  No GPU is used; on
GPUs the same module runs over NCCL with the CUDA library's ops."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(T, H, I, E, k, seed):
    import oracle
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    logits = torch.randn(T, E, generator=g)
    q13 = [oracle.quantize((torch.randn(2 * I, H, generator=g) * 0.1).numpy()) for _ in range(E)]
    q2 = [oracle.quantize((torch.randn(H, I, generator=g) * 0.1).numpy()) for _ in range(E)]
    w = [np.stack([a for a, _ in q13]), np.stack([b for _, b in q13]),
         np.stack([a for a, _ in q2]), np.stack([b for _, b in q2])]
    return x, logits, w


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class OracleOps:
    """CPU reference of the compute steps (test infrastructure; fp64)."""

    def route(self, logits, top_k):
        import oracle
        r = oracle.route(logits.numpy(), top_k)
        i32 = lambda a: torch.from_numpy(np.asarray(a, dtype=np.int32))
        return dict(ids=i32(r["ids"]), weights=torch.from_numpy(r["w"]),
                    counts=i32(r["counts"]), offsets=i32(r["offsets"]), perm=i32(r["perm"]), inv=i32(r["inv"]))

    def gather_rows(self, src, idx, div=1):
        return src[idx.long() // div]

    def experts(self, x_sorted, offsets, row_w, w):
        import oracle
        w13c, w13s, w2c, w2s = w
        I = w13c.shape[1] // 2
        off = offsets.numpy()
        xb = _bits(x_sorted)
        y = np.zeros((x_sorted.shape[0], w2c.shape[1]), np.float64)
        for e in range(w13c.shape[0]):
            a, b = off[e], off[e + 1]
            if a == b:
                continue
            gg = oracle.gemm_w4a16(xb[a:b], w13c[e][:I], w13s[e][:I])
            uu = oracle.gemm_w4a16(xb[a:b], w13c[e][I:], w13s[e][I:])
            h = oracle.f64_to_bf16(oracle.silu(gg) * uu)
            y[a:b] = row_w.numpy()[a:b, None].astype(np.float64) * oracle.gemm_w4a16(h, w2c[e], w2s[e])
        return torch.from_numpy(y)

    def combine(self, y_sorted, inv, top_k):
        y = y_sorted.numpy()
        iv = inv.numpy().reshape(-1, top_k)
        out = np.zeros((iv.shape[0], y.shape[1]), np.float64)
        for j in range(top_k):
            out += y[iv[:, j]]
        return torch.from_numpy(out)


def _worker(rank, world, port, q, shape):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from moe_expert_gemm_mxfp4_b200 import ep
        T, H, I, E, k, seed = shape
        x, logits, w = _layer(T, H, I, E, k, seed)
        part = ep.ExpertPartition(E, world)
        lo, hi = part.range(rank)
        t0, t1 = (rank * T) // world, ((rank + 1) * T) // world     # this rank's tokens
        trace = {}
        out = ep.moe_mlp_ep(x[t0:t1], logits[t0:t1], k, [a[lo:hi] for a in w], part, rank,
                            ops=OracleOps(), trace=trace)
        q.put((rank, t0, t1, out.numpy(), trace["route"]["ids"].numpy(), trace["recv_rows"],
               trace["send_rows"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape", [(2, (48, 64, 64, 6, 2, 1)), (2, (40, 96, 64, 5, 3, 2)),
                                         (3, (50, 64, 96, 7, 2, 3))])
def test_expert_parallel_layer_matches_single_process_oracle(world, shape):
    sys.path.insert(0, ROOT)
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, shape)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = sorted((q.get() for _ in range(world)), key=lambda g: g[0])
    T, H, I, E, k, seed = shape
    x, logits, w = _layer(T, H, I, E, k, seed)
    ref = oracle.moe_mlp(_bits(x), logits.numpy(), k, *w)
    r = oracle.route(logits.numpy(), k)
    flat = r["ids"].reshape(-1)
    from moe_expert_gemm_mxfp4_b200 import ep
    part = ep.ExpertPartition(E, world)
    total_recv = [0] * world
    for rank, t0, t1, out, ids, recv_rows, send_rows in got:
        assert np.array_equal(ids, r["ids"][t0:t1])                       # routing, bit for bit
        assert np.allclose(out, ref[t0:t1], rtol=1e-12, atol=1e-14)       # fp64, order only
        mine = r["ids"][t0:t1].reshape(-1)
        assert send_rows == [int(np.isin(mine, range(*part.range(d))).sum()) for d in range(world)]
        total_recv[rank] = sum(recv_rows)
    for d in range(world):    # every pair routed to rank d's experts arrived there
        assert total_recv[d] == int(np.isin(flat, range(*part.range(d))).sum())


def test_receive_plan_orders_rows_expert_major():
    sys.path.insert(0, ROOT)
    from moe_expert_gemm_mxfp4_b200 import ep
    # 2 sources x 3 local experts; arrivals: source 0 [e0 x2, e1 x0, e2 x1], source 1 [e0 x1, e1 x2, e2 x0]
    rc = np.array([[2, 0, 1], [1, 2, 0]])
    idx, off = ep.receive_plan(rc)
    assert off.tolist() == [0, 3, 5, 6]
    assert idx.tolist() == [0, 1, 3, 4, 5, 2]
    part = ep.ExpertPartition(7, 3)
    assert [part.range(r) for r in range(3)] == [(0, 2), (2, 4), (4, 7)]
    assert [part.owner(e) for e in range(7)] == [0, 0, 1, 1, 2, 2, 2]
