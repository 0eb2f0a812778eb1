"""Ring attention (context parallelism) over torch.distributed.

"long-context-models", section "Context parallelism distributes exact attention", and
"Long context (engineering 100k+ tokens)", sec. 3: the sequence is split into one
contiguous slice per worker; key/value blocks travel around a ring of workers, each
worker attends its own queries to the block it holds, folds the partial result into a
running one with the online-softmax (log-sum-exp) weights, and passes the block on while
it receives the next.  After `world` steps every worker has seen every block, and its
slice of the output equals exact attention over the whole sequence.

Layout: rank r holds tokens [r*C, (r+1)*C) of q [B, Hq, C, d] and k, v [B, Hkv, C, d]
(bf16, C = T / world).  The circulating block is the fp16 rotated-key/value workspace of
`api.prefill_prepare_kv_at` (keys rotated once, by their owner, at absolute positions).
Causal attention skips blocks wholly in a worker's future; a window skips blocks wholly
behind it (the sink block stays visible).  Blocks are exchanged with `batch_isend_irecv`
(NCCL on GPUs), double-buffered so that the transfer of the next block overlaps the
attention to the current one.

The compute goes through `BlockOps`: by default the CUDA kernels of this package (no
fallback).  Tests of the schedule and exchange on CPU ranks pass their own ops.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import api


def ring_schedule(rank: int, world: int):
    """(step, block) pairs: at step i rank r holds the block that started on rank r - i."""
    return [(i, (rank - i) % world) for i in range(world)]


def block_visible(q_block: int, k_block: int, C: int, causal: bool, window: int,
                  n_sink: int) -> bool:
    """Does any query of slice q_block see any key of slice k_block (slices of C tokens)?"""
    if not causal:
        return True
    if k_block > q_block:
        return False
    if window <= 0:
        return True
    nearest = max(0, q_block * C - ((k_block + 1) * C - 1))  # closest query-key distance
    return nearest < window or k_block * C < n_sink


class BlockOps:
    """The three block operations of a ring step, on this package's CUDA kernels."""

    def prepare(self, k, v, table, k_pos0: int):
        B, Hkv, C, d = k.shape
        ws = torch.empty(api.attn_prefill_workspace_bytes(B, Hkv, C, d), dtype=torch.uint8,
                         device=k.device)
        return api.prefill_prepare_kv_at(k, v, table, ws, k_pos0)

    def attend(self, q, block, Hkv: int, Tk: int, table, q_pos0: int, k_pos0: int,
               causal: bool, window: int, n_sink: int):
        return api.prefill_attend_block(q, Hkv, Tk, table, block, q_pos0, k_pos0, causal,
                                        window, n_sink)

    def new_acc(self, q):
        B, Hq, C, d = q.shape
        return (torch.empty((B, Hq, C, d), dtype=torch.float32, device=q.device),
                torch.empty((B, Hq, C), dtype=torch.float32, device=q.device),
                torch.empty((B, Hq, C, d), dtype=torch.bfloat16, device=q.device))

    def merge(self, o_part, lse_part, acc, first: bool, last: bool):
        o_acc, lse_acc, out = acc
        api.attn_merge(o_part, lse_part, o_acc, lse_acc, out=out if last else None, init=first)

    def result(self, acc):
        return acc[2], acc[1]


def ring_prefill(q, k, v, table, group=None, causal: bool = True, window: int = 0,
                 n_sink: int = 0, ops: BlockOps | None = None):
    """This rank's slice of ring attention.  Returns (o bf16 [B,Hq,C,d], lse fp32 [B,Hq,C])."""
    ops = ops or BlockOps()
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, Hq, C, d = q.shape
    Hkv = k.shape[1]
    if k.shape[2] != C or v.shape != k.shape:
        raise ValueError("ring_prefill: q, k and v must hold the same C tokens per rank")
    peer_next = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    peer_prev = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    steps = ring_schedule(rank, world)
    visible = [block_visible(rank, src, C, causal, window, n_sink) for _, src in steps]
    last_visible = max(i for i, vis in enumerate(visible) if vis)  # own block: always visible
    block = ops.prepare(k, v, table, rank * C)
    spare = torch.empty_like(block)
    acc = ops.new_acc(q)
    first = True
    for (step, src), vis in zip(steps, visible):
        reqs = []
        if step < world - 1:
            reqs = dist.batch_isend_irecv([
                dist.P2POp(dist.isend, block, peer_next, group),
                dist.P2POp(dist.irecv, spare, peer_prev, group)])
        if vis:
            o_p, lse_p = ops.attend(q, block, Hkv, C, table, rank * C, src * C, causal, window,
                                    n_sink)
            ops.merge(o_p, lse_p, acc, first, step == last_visible)
            first = False
        for r in reqs:
            r.wait()
        block, spare = spare, block
    return ops.result(acc)


def ring_prefill_emulated(q, k, v, table, world: int, causal: bool = True, window: int = 0,
                          n_sink: int = 0, ops: BlockOps | None = None):
    """Every virtual rank's ring schedule run in turn in one process: the same block
    kernels with the same positions and the same merge order as `ring_prefill`, without
    the exchange.  q [B,Hq,T,d], k, v [B,Hkv,T,d] with T divisible by `world`.  Returns
    the per-rank (o, lse) slices in rank order."""
    ops = ops or BlockOps()
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if T % world:
        raise ValueError("ring_prefill_emulated: T must be divisible by world")
    C = T // world
    blocks = [ops.prepare(k[:, :, r * C:(r + 1) * C], v[:, :, r * C:(r + 1) * C], table, r * C)
              for r in range(world)]
    outs = []
    for rank in range(world):
        q_r = q[:, :, rank * C:(rank + 1) * C]
        steps = [(i, src) for i, src in ring_schedule(rank, world)
                 if block_visible(rank, src, C, causal, window, n_sink)]
        acc = ops.new_acc(q_r)
        for n, (_, src) in enumerate(steps):
            o_p, lse_p = ops.attend(q_r, blocks[src], Hkv, C, table, rank * C, src * C, causal,
                                    window, n_sink)
            ops.merge(o_p, lse_p, acc, n == 0, n == len(steps) - 1)
        outs.append(ops.result(acc))
    return outs
