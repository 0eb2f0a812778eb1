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

Causal attention gives the contiguous layout uneven work: rank r attends r + 1 of the
`world` blocks.  The zigzag layout ("long-context-models", context parallelism: load
balancing of causal work) cuts the sequence into 2 * world chunks and gives rank r
chunks r and 2 * world - 1 - r, so every rank attends 2 * world + 1 (query chunk, key
chunk) pairs under a causal mask.  Its blocks are the two chunks' workspaces, exchanged
together.

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


def zigzag_chunks(rank: int, world: int):
    """The two of 2 * world equal chunks rank r holds in the zigzag layout."""
    return (rank, 2 * world - 1 - rank)


def rank_pairs(rank: int, world: int, layout: str, causal: bool = True, window: int = 0,
               n_sink: int = 0, C: int = 1):
    """(query chunk, key chunk) pairs rank r attends over a whole ring pass, in chunk
    indices of the layout (chunks of C tokens: T / world contiguous, T / (2 world) zigzag)."""
    mine = [rank] if layout == "contiguous" else list(zigzag_chunks(rank, world))
    n = world if layout == "contiguous" else 2 * world
    return [(a, b) for a in mine for b in range(n)
            if block_visible(a, b, C, causal, window, n_sink)]


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
                 n_sink: int = 0, ops: BlockOps | None = None, layout: str = "contiguous"):
    """This rank's slice of ring attention.  Returns (o bf16 [B,Hq,C,d], lse fp32 [B,Hq,C]).
    layout "contiguous": the rank's C tokens are slice r of the sequence; "zigzag": they are
    chunks r and 2 world - 1 - r of C / 2 tokens each, in that order."""
    ops = ops or BlockOps()
    if layout == "zigzag":
        return _ring_prefill_zigzag(q, k, v, table, group, causal, window, n_sink, ops)
    if layout != "contiguous":
        raise ValueError(f"ring_prefill: unknown layout {layout!r}")
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


def _zigzag_plan(rank, world, c, causal, window, n_sink):
    """Per ring step: (step, source rank, its chunks, visible (own chunk, its chunk) index
    pairs); and per own query chunk the (step, key index) of its last visible pair."""
    mine = zigzag_chunks(rank, world)
    plan, last = [], {}
    for step, src in ring_schedule(rank, world):
        theirs = zigzag_chunks(src, world)
        pairs = [(a, b) for a in (0, 1) for b in (0, 1)
                 if block_visible(mine[a], theirs[b], c, causal, window, n_sink)]
        for a, b in pairs:
            last[a] = (step, b)
        plan.append((step, src, theirs, pairs))
    return mine, plan, last


def _ring_prefill_zigzag(q, k, v, table, group, causal, window, n_sink, ops):
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, Hq, C, d = q.shape
    Hkv = k.shape[1]
    if k.shape[2] != C or v.shape != k.shape or C % 2:
        raise ValueError("ring_prefill: q, k and v must hold the same even number of tokens")
    c = C // 2
    peer_next = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    peer_prev = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    mine, plan, last = _zigzag_plan(rank, world, c, causal, window, n_sink)
    q_ch = [q[:, :, a * c:(a + 1) * c] for a in (0, 1)]
    blocks = [ops.prepare(k[:, :, a * c:(a + 1) * c], v[:, :, a * c:(a + 1) * c], table,
                          mine[a] * c) for a in (0, 1)]
    spares = [torch.empty_like(b) for b in blocks]
    accs = [ops.new_acc(q_ch[a]) for a in (0, 1)]
    first = [True, True]
    for step, src, theirs, pairs in plan:
        reqs = []
        if step < world - 1:
            ops_p2p = []
            for b in (0, 1):
                ops_p2p += [dist.P2POp(dist.isend, blocks[b], peer_next, group),
                            dist.P2POp(dist.irecv, spares[b], peer_prev, group)]
            reqs = dist.batch_isend_irecv(ops_p2p)
        for a, b in pairs:
            o_p, lse_p = ops.attend(q_ch[a], blocks[b], Hkv, c, table, mine[a] * c,
                                    theirs[b] * c, causal, window, n_sink)
            ops.merge(o_p, lse_p, accs[a], first[a], last.get(a) == (step, b))
            first[a] = False
        for r in reqs:
            r.wait()
        blocks, spares = spares, blocks
    res = [ops.result(accs[a]) for a in (0, 1)]
    return torch.cat([res[0][0], res[1][0]], dim=2), torch.cat([res[0][1], res[1][1]], dim=2)


def zigzag_gather(x, world: int, rank: int):
    """Rank r's zigzag share of a sequence tensor [B, H, T, ...]: chunks r and
    2 world - 1 - r of T / (2 world) tokens, concatenated."""
    c = x.shape[2] // (2 * world)
    a, b = zigzag_chunks(rank, world)
    return torch.cat([x[:, :, a * c:(a + 1) * c], x[:, :, b * c:(b + 1) * c]], dim=2)


def ring_prefill_emulated(q, k, v, table, world: int, causal: bool = True, window: int = 0,
                          n_sink: int = 0, ops: BlockOps | None = None,
                          layout: str = "contiguous"):
    """Every virtual rank's ring schedule run in turn in one process: the same block
    kernels with the same positions and the same merge order as `ring_prefill`, without
    the exchange.  q [B,Hq,T,d], k, v [B,Hkv,T,d] with T divisible by `world`.  Returns
    the per-rank (o, lse) slices in rank order."""
    ops = ops or BlockOps()
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if layout == "zigzag":
        if T % (2 * world):
            raise ValueError("ring_prefill_emulated: T must be divisible by 2 world")
        c = T // (2 * world)
        chunk_blocks = [ops.prepare(k[:, :, i * c:(i + 1) * c], v[:, :, i * c:(i + 1) * c],
                                    table, i * c) for i in range(2 * world)]
        outs = []
        for rank in range(world):
            mine, plan, last = _zigzag_plan(rank, world, c, causal, window, n_sink)
            q_ch = [q[:, :, m * c:(m + 1) * c] for m in mine]
            accs = [ops.new_acc(q_ch[a]) for a in (0, 1)]
            first = [True, True]
            for step, src, theirs, pairs in plan:
                for a, b in pairs:
                    o_p, lse_p = ops.attend(q_ch[a], chunk_blocks[theirs[b]], Hkv, c, table,
                                            mine[a] * c, theirs[b] * c, causal, window, n_sink)
                    ops.merge(o_p, lse_p, accs[a], first[a], last.get(a) == (step, b))
                    first[a] = False
            res = [ops.result(accs[a]) for a in (0, 1)]
            outs.append((torch.cat([res[0][0], res[1][0]], dim=2),
                         torch.cat([res[0][1], res[1][1]], dim=2)))
        return outs
    if layout != "contiguous":
        raise ValueError(f"ring_prefill_emulated: unknown layout {layout!r}")
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
