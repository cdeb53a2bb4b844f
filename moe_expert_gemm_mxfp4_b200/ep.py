"""Expert parallelism (EP) for the MXFP4 MoE layer over ``torch.distributed``.

The pages distribute a mixture-of-experts model's experts across GPUs
(agentlenshq.com, "Transformers 4.40 performance upgrades for OpenAI GPT-OSS ...",
section "Expert Parallelism (EP)").  Here each of the G ranks of a process group
holds a contiguous range of the E experts (rank r: experts [r*E/G, (r+1)*E/G),
their MXFP4 weights only) and its own tokens.  One layer is:

  1. route the local tokens (top-k, softmax, expert-sorted permutation);
  2. counts all-to-all: every rank sends each peer the per-expert pair counts of
     that peer's experts, so every rank knows how many rows it will receive from
     whom, and for which of its experts;
  3. rows all-to-all: the local token rows in expert-sorted order (contiguous per
     destination, since each rank's experts are a contiguous range) and their
     routing weights go to the ranks that hold their experts;
  4. the receiver reorders what arrived (source-major) into expert-major order and
     runs its experts (gate/up + SwiGLU, down x routing weight, fp32 out);
  5. the results go back in source-major order (reverse all-to-all) and land in the
     sender's expert-sorted positions;
  6. the sender combines each token's k results in slot order (bf16 out).

Split sizes of an all-to-all must be host integers, so the per-expert counts make
one device -> host trip per layer (step 2); everything else stays on the device.
The collectives are ``all_to_all_single`` on byte views of the rows, so the same
code runs over NCCL (GPU tensors) and gloo (CPU tensors, as the tests do).  No
collective here uses TMA or any multicast load.

The compute steps come from an ``ops`` object, so that the bookkeeping is the same
whatever computes: ``LibraryOps`` (the CUDA library; the product path) or a test's
CPU reference.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

__all__ = ["ExpertPartition", "LibraryOps", "moe_mlp_ep", "receive_plan"]


@dataclass(frozen=True)
class ExpertPartition:
    """E experts over `world` ranks in contiguous ranges (the first E % world ranks
    hold one expert more than the rest)."""

    E: int
    world: int

    def range(self, r: int) -> tuple[int, int]:
        return (r * self.E) // self.world, ((r + 1) * self.E) // self.world

    def owner(self, e: int) -> int:
        for r in range(self.world):
            lo, hi = self.range(r)
            if lo <= e < hi:
                return r
        raise ValueError(f"expert {e} out of range")

    def sizes(self) -> list[int]:
        return [self.range(r)[1] - self.range(r)[0] for r in range(self.world)]


def receive_plan(recv_counts: np.ndarray):
    """From recv_counts[s, e] (rows from source s for local expert e, arriving
    source-major and, within a source, expert-sorted) -> (idx, offsets): idx[i] is
    the arrival position of the i-th row in expert-major order (expert, then source,
    then arrival order), offsets [E_local + 1] the expert-major group offsets."""
    G, El = recv_counts.shape
    src_start = np.concatenate([[0], np.cumsum(recv_counts.sum(axis=1))])
    exp_start = np.concatenate([np.zeros((G, 1), np.int64), np.cumsum(recv_counts, axis=1)], axis=1)
    idx = [np.arange(src_start[s] + exp_start[s, e], src_start[s] + exp_start[s, e] + recv_counts[s, e])
           for e in range(El) for s in range(G)]
    idx = np.concatenate(idx).astype(np.int32) if idx else np.zeros(0, np.int32)
    offsets = np.concatenate([[0], np.cumsum(recv_counts.sum(axis=0))]).astype(np.int32)
    return idx, offsets


def _a2a_rows(t: torch.Tensor, out_rows: list[int], in_rows: list[int], group) -> torch.Tensor:
    """all_to_all_single of the rows of a 2-D tensor, on its bytes."""
    import torch.distributed as dist
    rb = t.shape[1] * t.element_size()
    src = t.contiguous().view(torch.uint8).reshape(t.shape[0], rb)
    dst = torch.empty((sum(out_rows), rb), dtype=torch.uint8, device=t.device)
    dist.all_to_all_single(dst, src, [r for r in out_rows], [r for r in in_rows], group=group)
    return dst.view(t.dtype).reshape(sum(out_rows), t.shape[1])


class LibraryOps:
    """The compute steps on the CUDA library (the product path)."""

    def __init__(self, mode: int = 0):
        self.mode = mode

    def route(self, logits, top_k):
        from . import moe_mxfp4_route
        return moe_mxfp4_route(logits, top_k)

    def gather_rows(self, src, idx, div=1):
        from . import mxfp4_gather_rows
        return mxfp4_gather_rows(src, idx, div)

    def experts(self, x_sorted, offsets, row_w, w):
        from . import moe_mxfp4_experts
        return moe_mxfp4_experts(x_sorted, offsets, row_w, *w, mode=self.mode)

    def combine(self, y_sorted, inv, top_k):
        from . import moe_mxfp4_combine
        return moe_mxfp4_combine(y_sorted, inv, top_k)


def moe_mlp_ep(x: torch.Tensor, logits: torch.Tensor, top_k: int, local_w, part: ExpertPartition,
               rank: int, ops=None, group=None, trace: dict | None = None):
    """One MoE layer under expert parallelism (see the module docstring).

    x [T_r, H] (bf16) and logits [T_r, E] are this rank's tokens; local_w = (w13
    codes, w13 scales, w2 codes, w2 scales) of this rank's experts part.range(rank)
    only, shaped [E_r, ...].  Returns out [T_r, H].  Every rank must call it, with
    the same partition, in the same order.  `trace`, if given, receives this rank's
    routing tables and exchange sizes (for tests)."""
    ops = LibraryOps() if ops is None else ops
    G = part.world
    lo, hi = part.range(rank)
    El = hi - lo
    sizes = part.sizes()
    r = ops.route(logits, top_k)
    offsets = r["offsets"].cpu().numpy().astype(np.int64)          # the one device -> host trip
    send_rows = [int(offsets[part.range(d)[1]] - offsets[part.range(d)[0]]) for d in range(G)]
    # counts of each destination's experts -> (source, local expert) counts here
    recv = _a2a_rows(r["counts"].reshape(-1, 1).to(torch.int32), [El] * G, sizes, group)
    recv_counts = recv.reshape(G, El).cpu().numpy().astype(np.int64)
    recv_rows = [int(c) for c in recv_counts.sum(axis=1)]
    # local rows and routing weights in expert-sorted order -> their experts' ranks
    x_sorted = ops.gather_rows(x, r["perm"], top_k)
    w_sorted = ops.gather_rows(r["weights"].reshape(-1, 1), r["perm"], 1)
    rows_in = _a2a_rows(x_sorted, recv_rows, send_rows, group)
    w_in = _a2a_rows(w_sorted, recv_rows, send_rows, group)
    # source-major arrivals -> expert-major groups, run the local experts, and back
    idx, loc_off = receive_plan(recv_counts)
    R = int(idx.size)
    H = x.shape[1]
    if R:
        dev = x.device
        idx_t = torch.from_numpy(idx).to(dev)
        y_em = ops.experts(ops.gather_rows(rows_in, idx_t, 1), torch.from_numpy(loc_off).to(dev),
                           ops.gather_rows(w_in, idx_t, 1).reshape(-1), local_w)
        back = torch.from_numpy(np.argsort(idx, kind="stable").astype(np.int32)).to(dev)
        y_sm = ops.gather_rows(y_em, back, 1)
    else:
        y_sm = torch.zeros((0, H), dtype=torch.float32, device=x.device)
    y_sorted = _a2a_rows(y_sm, send_rows, recv_rows, group)
    out = ops.combine(y_sorted, r["inv"], top_k)
    if trace is not None:
        trace.update(route=r, send_rows=send_rows, recv_rows=recv_rows, recv_counts=recv_counts,
                     local_offsets=loc_off)
    return out
