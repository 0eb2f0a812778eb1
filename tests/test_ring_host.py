"""Ring attention host logic on CPU ranks over gloo: the schedule, the block visibility
rule, the positions each block is rotated and masked at, the exchange and the
log-sum-exp merge.  The block operations are plain fp64 numpy here (built on the
oracle's rotation); the result must equal the oracle's exact attention over the whole
sequence.  The CUDA block kernels are checked against the oracle in test_gpu_ring.py.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from tests._util import to_bits
from yarn_position_scaling_b200 import ring

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _visible_pairs(qb, kb, C, causal, window, n_sink):
    qp = np.arange(qb * C, (qb + 1) * C)[:, None]
    kp = np.arange(kb * C, (kb + 1) * C)[None, :]
    if not causal:
        return True
    vis = kp <= qp
    if window > 0:
        vis &= (qp - kp < window) | (kp < n_sink)
    return bool(vis.any())


@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_schedule_visits_every_block_once(world):
    for r in range(world):
        steps = ring.ring_schedule(r, world)
        assert [s for s, _ in steps] == list(range(world))
        assert sorted(b for _, b in steps) == list(range(world))
        assert steps[0] == (0, r)
        # the block a rank holds at step i+1 is the one its predecessor held at step i
        prev = ring.ring_schedule((r - 1) % world, world)
        for i in range(world - 1):
            assert steps[i + 1][1] == prev[i][1]


@pytest.mark.parametrize("causal,window,n_sink", [(True, 0, 0), (False, 0, 0), (True, 20, 0),
                                                  (True, 20, 2), (True, 33, 0), (True, 1, 0),
                                                  (True, 64, 40)])
def test_block_visibility_matches_brute_force(causal, window, n_sink):
    C = 32
    for qb in range(5):
        for kb in range(5):
            want = _visible_pairs(qb, kb, C, causal, window, n_sink)
            assert ring.block_visible(qb, kb, C, causal, window, n_sink) == want, (qb, kb)


class CpuBlockOps:
    """fp64 numpy stand-ins for the three block kernels (test only)."""

    def __init__(self, theta, scale):
        self.theta, self.scale = theta, scale

    def _rot(self, x, pos0):
        B, H, C, d = x.shape
        pos = np.tile(np.arange(pos0, pos0 + C, dtype=np.float64), B * H)
        return oracle.rotate(to_bits(x).reshape(-1, d), pos, self.theta).reshape(B, H, C, d)

    def prepare(self, k, v, table, k_pos0):
        kr = self._rot(k, k_pos0)
        vv = v.to(torch.float64).numpy()
        return torch.from_numpy(np.stack([kr, vv]))

    def attend(self, q, block, Hkv, Tk, table, q_pos0, k_pos0, causal, window, n_sink):
        qr = self._rot(q, q_pos0)
        kr, vv = block[0].numpy(), block[1].numpy()
        B, Hq, C, d = qr.shape
        g = Hq // Hkv
        kr = np.repeat(kr, g, axis=1)
        vv = np.repeat(vv, g, axis=1)
        s = self.scale * np.einsum("bhqd,bhkd->bhqk", qr, kr)
        qp = (q_pos0 + np.arange(C))[:, None]
        kp = (k_pos0 + np.arange(Tk))[None, :]
        vis = np.ones((C, Tk), bool)
        if causal:
            vis = kp <= qp
            if window > 0:
                vis &= (qp - kp < window) | (kp < n_sink)
        s = np.where(vis, s, -np.inf)
        m = s.max(axis=-1, keepdims=True)
        live = np.isfinite(m)
        p = np.where(live, np.exp(s - np.where(live, m, 0.0)), 0.0)
        l = p.sum(axis=-1, keepdims=True)
        o = np.where(live, np.einsum("bhqk,bhkd->bhqd", p, vv) / np.where(live, l, 1.0), 0.0)
        lse = np.where(live[..., 0], m[..., 0] + np.log(np.where(live, l, 1.0))[..., 0], -np.inf)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def new_acc(self, q):
        return [None, None]

    def merge(self, o_p, lse_p, acc, first, last):
        if first:
            acc[0], acc[1] = o_p.clone(), lse_p.clone()
            return
        la, lp = acc[1].numpy(), lse_p.numpy()
        m = np.maximum(la, lp)
        live = np.isfinite(m)
        mm = np.where(live, m, 0.0)
        wa, wp = np.exp(la - mm), np.exp(lp - mm)
        tot = np.where(live, wa + wp, 1.0)
        o = (wa[..., None] * acc[0].numpy() + wp[..., None] * o_p.numpy()) / tot[..., None]
        acc[0] = torch.from_numpy(np.where(live[..., None], o, acc[0].numpy()))
        acc[1] = torch.from_numpy(np.where(live, mm + np.log(tot), -np.inf))

    def result(self, acc):
        return acc[0], acc[1]


CASE = dict(B=1, Hq=4, Hkv=2, d=16, C=24, base=10000.0, L_train=32, s=4.0, method="yarn")


def _inputs(world, B, Hq, Hkv, d, C, **_):
    g = torch.Generator().manual_seed(1234)
    T = world * C
    q = torch.randn((B, Hq, T, d), generator=g).to(torch.bfloat16)
    k = torch.randn((B, Hkv, T, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, Hkv, T, d), generator=g).to(torch.bfloat16)
    return q, k, v


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, causal, window, n_sink, out, layout="contiguous"):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _inputs(world, **CASE)
        C = CASE["C"]
        th, _, ss = oracle.rope_theta(CASE["d"], CASE["base"], CASE["L_train"], CASE["s"],
                                      CASE["method"])
        if layout == "zigzag":
            share = [ring.zigzag_gather(x, world, rank) for x in (q, k, v)]
        else:
            sl = slice(rank * C, (rank + 1) * C)
            share = [x[:, :, sl] for x in (q, k, v)]
        o, lse = ring.ring_prefill(*share, None, causal=causal, window=window, n_sink=n_sink,
                                   ops=CpuBlockOps(th, ss), layout=layout)
        out.put((rank, o.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal,window,n_sink", [
    (2, True, 0, 0), (3, True, 0, 0), (3, False, 0, 0),
    (3, True, 20, 0),   # rank 2 skips block 0
    (3, True, 20, 2),   # ... unless block 0 holds the sinks
    (4, True, 30, 3)])
def test_ring_over_gloo_equals_exact_attention(world, causal, window, n_sink):
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, window, n_sink, qu))
             for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((qu.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v = _inputs(world, **CASE)
    th, _, ss = oracle.rope_theta(CASE["d"], CASE["base"], CASE["L_train"], CASE["s"],
                                  CASE["method"])
    ro, rl, _ = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss, causal, window,
                                 n_sink)
    B, Hq, d, C = CASE["B"], CASE["Hq"], CASE["d"], CASE["C"]
    T = world * C
    ro = ro.reshape(B, Hq, T, d)
    rl = rl.reshape(B, Hq, T)
    for rank, o, lse in got:
        sl = slice(rank * C, (rank + 1) * C)
        np.testing.assert_allclose(o, ro[:, :, sl], atol=1e-10)
        np.testing.assert_allclose(lse, rl[:, :, sl], atol=1e-10)


def test_ring_rejects_unequal_slices():
    q = torch.zeros((1, 2, 8, 16), dtype=torch.bfloat16)
    k = torch.zeros((1, 1, 4, 16), dtype=torch.bfloat16)
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group is already initialised")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        with pytest.raises(ValueError):
            ring.ring_prefill(q, k, k, None, ops=CpuBlockOps(np.zeros(8), 1.0))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal,window,n_sink", [
    (2, True, 0, 0), (3, True, 0, 0), (3, False, 0, 0), (4, True, 30, 3)])
def test_zigzag_ring_over_gloo_equals_exact_attention(world, causal, window, n_sink):
    # zigzag layout: rank r holds chunks r and 2 world - 1 - r of C / 2 tokens each
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, window, n_sink, qu,
                                               "zigzag"))
             for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((qu.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v = _inputs(world, **CASE)
    th, _, ss = oracle.rope_theta(CASE["d"], CASE["base"], CASE["L_train"], CASE["s"],
                                  CASE["method"])
    ro, rl, _ = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss, causal, window,
                                 n_sink)
    B, Hq, d, C = CASE["B"], CASE["Hq"], CASE["d"], CASE["C"]
    T = world * C
    ro = torch.from_numpy(ro.reshape(B, Hq, T, d))
    rl = torch.from_numpy(rl.reshape(B, Hq, T, 1))
    for rank, o, lse in got:
        np.testing.assert_allclose(o, ring.zigzag_gather(ro, world, rank).numpy(), atol=1e-10)
        np.testing.assert_allclose(lse, ring.zigzag_gather(rl, world, rank).numpy()[..., 0],
                                   atol=1e-10)


@pytest.mark.parametrize("world", [2, 4, 8])
def test_zigzag_balances_causal_work(world):
    # contiguous slices: rank r attends r + 1 of world blocks; zigzag: every rank attends
    # 2 world + 1 (query chunk, key chunk) pairs, i.e. the same share of the causal work
    zz = [len(ring.rank_pairs(r, world, "zigzag")) for r in range(world)]
    assert zz == [2 * world + 1] * world
    assert sum(zz) == (2 * world) * (2 * world + 1) // 2   # every causal chunk pair once
    co = [len(ring.rank_pairs(r, world, "contiguous")) for r in range(world)]
    assert co == list(range(1, world + 1))

