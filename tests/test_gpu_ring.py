"""Ring attention building blocks on the GPU, through the C ABI, against the fp64 oracle.

The block kernels (keys prepared at an absolute position, queries attending to one
block) and the log-sum-exp merge are run exactly as a ring worker runs them, for every
virtual rank in turn on one device (`ring_prefill_emulated`: no kernel waits on another,
no exchange).  Each rank's slice of the output and of the log-sum-exp must match the
oracle's exact attention over the whole sequence.  The exchange itself is covered on CPU
ranks in test_ring_host.py.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from tests._util import O_MAX_ABS, O_MEAN_ABS, err_stats, to_bits, to_f64
from yarn_position_scaling_b200 import api, build, ring, synth

pytestmark = pytest.mark.gpu

LSE_ABS = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    api.load()
    assert torch.cuda.is_available()


def _tables(w):
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    th, _, ss = oracle.rope_theta(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    return tab, th, ss


def _ring_vs_oracle(w, T, world, causal=True, window=0, n_sink=0, rows_per_slice=None):
    q, k, v = synth.prefill_inputs(w, "cuda", T=T)
    tab, th, ss = _tables(w)
    outs = ring.ring_prefill_emulated(q, k, v, tab, world, causal, window, n_sink)
    api.device_status()
    C = T // world
    B, Hq, d = q.shape[0], q.shape[1], q.shape[3]
    o = torch.cat([o_r for o_r, _ in outs], dim=2)
    lse = torch.cat([l_r for _, l_r in outs], dim=2)
    if rows_per_slice is None:
        rows = None
    else:
        rng = np.random.default_rng(7)
        ms = []
        for r in range(world):
            edge = [r * C, r * C + 1, r * C + 127, r * C + 128, (r + 1) * C - 1]
            ms += edge + rng.integers(r * C, (r + 1) * C, rows_per_slice).tolist()
        ms = sorted(set(m for m in ms if 0 <= m < T))
        heads = sorted(set([0, Hq - 1, Hq // 2]))
        rows = np.array([(b * Hq + h) * T + m for b in range(B) for h in heads for m in ms],
                        dtype=np.int64)
    ro, rl, _ = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss, causal, window,
                                 n_sink, rows=rows)
    got_o = to_f64(o).reshape(-1, d)
    got_l = to_f64(lse).reshape(-1)
    if rows is not None:
        got_o, got_l = got_o[rows], got_l[rows]
    emax, emean = err_stats(got_o, ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(got_l, rl)[0] <= LSE_ABS
    return q, k, v, tab, o, lse


@pytest.mark.parametrize("world,T", [(2, 512), (4, 600), (3, 384), (5, 640)])
def test_ring_causal_slices_match_oracle(world, T):
    # T = 600 over 4 ranks: 150-token slices, so block edges fall inside key tiles
    _ring_vs_oracle(synth.TINY, T, world)


@pytest.mark.parametrize("world,T,window,n_sink", [(4, 1024, 200, 4), (4, 1024, 200, 0),
                                                   (3, 900, 64, 1), (2, 700, 300, 130)])
def test_ring_window_and_sinks(world, T, window, n_sink):
    # the 200-token window over 256-token slices skips blocks; sinks keep block 0 visible
    _ring_vs_oracle(synth.TINY, T, world, window=window, n_sink=n_sink)


def test_ring_non_causal():
    _ring_vs_oracle(synth.TINY, 384, 3, causal=False)


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 2, 128), (4, 4, 64), (8, 1, 128)])
def test_ring_heads_and_head_dims(Hq, Hkv, d):
    w = dataclasses.replace(synth.LLAMA3_128K, Hq=Hq, Hkv=Hkv, d=d)
    _ring_vs_oracle(w, 768, 3)


def test_ring_of_one_rank_is_the_prefill_bit_for_bit():
    w = synth.TINY
    q, k, v = synth.prefill_inputs(w, "cuda", T=700)
    tab, _, _ = _tables(w)
    (o, lse), = ring.ring_prefill_emulated(q, k, v, tab, 1, window=300, n_sink=4)
    lse_ref = torch.empty(q.shape[:3], device="cuda")
    ref = api.attn_prefill(q, k, v, tab, True, 300, 4, lse=lse_ref)
    api.device_status()
    assert torch.equal(o, ref)
    assert torch.equal(lse, lse_ref)


def test_ring_llama2_16k_four_ranks_sampled():
    # the 16K workload split over four 4096-token ranks
    _ring_vs_oracle(synth.LLAMA2_16K, synth.LLAMA2_16K.T, 4, rows_per_slice=12)


def test_block_rejects_future_block_and_bad_positions():
    w = synth.TINY
    q, k, v = synth.prefill_inputs(w, "cuda", T=256)
    tab, _, _ = _tables(w)
    ws = torch.empty(api.attn_prefill_workspace_bytes(1, w.Hkv, 128, w.d), dtype=torch.uint8,
                     device="cuda")
    api.prefill_prepare_kv_at(k[:, :, 128:], v[:, :, 128:], tab, ws, 128)
    with pytest.raises(api.YarnAttnError):
        api.prefill_attend_block(q[:, :, :128], w.Hkv, 128, tab, ws, q_pos0=0, k_pos0=128)
    with pytest.raises(api.YarnAttnError):
        api.prefill_attend_block(q[:, :, :128], w.Hkv, 128, tab, ws, q_pos0=-1, k_pos0=0)
    with pytest.raises(api.YarnAttnError):
        api.prefill_prepare_kv_at(k[:, :, 128:], v[:, :, 128:], tab, ws, -5)
    # a workspace sized for 128 keys cannot serve a 256-key block
    with pytest.raises(api.YarnAttnError):
        api.prefill_attend_block(q[:, :, :128], w.Hkv, 256, tab, ws, q_pos0=256, k_pos0=0)
    api.device_status()


def test_block_with_no_visible_key_writes_zero_and_minus_inf():
    # queries at 1000.. with a 64-token window see none of the keys 0..255
    w = synth.TINY
    q, k, v = synth.prefill_inputs(w, "cuda", T=256)
    tab, _, _ = _tables(w)
    ws = torch.empty(api.attn_prefill_workspace_bytes(1, w.Hkv, 256, w.d), dtype=torch.uint8,
                     device="cuda")
    api.prefill_prepare_kv_at(k, v, tab, ws, 0)
    o = torch.full(q.shape, float("nan"), device="cuda")
    lse = torch.full(q.shape[:3], 7.0, device="cuda")
    api.prefill_attend_block(q, w.Hkv, 256, tab, ws, q_pos0=1000, k_pos0=0, window=64,
                             out=o, lse=lse)
    api.device_status()
    assert torch.count_nonzero(o) == 0 and not torch.isnan(o).any()
    assert torch.isneginf(lse).all()


def _merge_ref(o_acc, lse_acc, o_part, lse_part, init):
    la = np.full_like(lse_part, -np.inf) if init else lse_acc
    m = np.maximum(la, lse_part)
    live = np.isfinite(m)
    mm = np.where(live, m, 0.0)
    wa, wp = np.exp(la - mm), np.exp(lse_part - mm)
    tot = np.where(live, wa + wp, 1.0)
    acc = np.zeros_like(o_part) if init else np.where(np.isfinite(la)[:, None], o_acc, 0.0)
    part = np.where(np.isfinite(lse_part)[:, None], o_part, 0.0)
    o = (wa[:, None] * acc + wp[:, None] * part) / tot[:, None]
    o = np.where(live[:, None], o, o_acc if not init else 0.0)
    return o, np.where(live, mm + np.log(tot), -np.inf)


@pytest.mark.parametrize("d,init", [(128, False), (64, False), (128, True)])
def test_merge_kernel_against_numpy(d, init):
    g = torch.Generator(device="cuda").manual_seed(3)
    rows = 1000
    o_part = torch.randn((rows, d), generator=g, device="cuda")
    lse_part = torch.randn((rows,), generator=g, device="cuda") * 4
    o_acc = torch.randn((rows, d), generator=g, device="cuda")
    lse_acc = torch.randn((rows,), generator=g, device="cuda") * 4
    lse_part[::7] = -float("inf")           # no visible key in this block
    o_part[::7] = float("nan")              # ... whose o_part must not be read
    lse_acc[::5] = -float("inf")            # empty accumulator rows
    o_acc[::5] = float("nan")               # ... whose o_acc must not be read
    want_o, want_l = _merge_ref(to_f64(o_acc), to_f64(lse_acc), to_f64(o_part), to_f64(lse_part),
                                init)
    out = torch.empty((rows, d), dtype=torch.bfloat16, device="cuda")
    api.attn_merge(o_part, lse_part, o_acc, lse_acc, out=out, init=init)
    api.device_status()
    got_o, got_l = to_f64(o_acc), to_f64(lse_acc)
    both_empty = ~np.isfinite(want_l)
    assert np.array_equal(both_empty, ~np.isfinite(got_l))
    np.testing.assert_allclose(got_l[~both_empty], want_l[~both_empty], rtol=1e-6, atol=1e-6)
    live = ~both_empty
    np.testing.assert_allclose(got_o[live], want_o[live], rtol=1e-5, atol=1e-5)
    ob = to_f64(out)
    np.testing.assert_allclose(ob[live], got_o[live], rtol=2.0 ** -8, atol=1e-6)
    assert np.all(ob[both_empty] == 0.0)


@pytest.mark.parametrize("world,T,window,n_sink", [(2, 512, 0, 0), (4, 1024, 0, 0),
                                                   (4, 1024, 300, 4)])
def test_zigzag_ring_matches_oracle(world, T, window, n_sink):
    # zigzag layout: rank r's queries are chunks r and 2 world - 1 - r of T / (2 world)
    w = dataclasses.replace(synth.LLAMA3_128K, Hq=8, Hkv=2)
    q, k, v = synth.prefill_inputs(w, "cuda", T=T)
    tab, th, ss = _tables(w)
    outs = ring.ring_prefill_emulated(q, k, v, tab, world, True, window, n_sink,
                                      layout="zigzag")
    api.device_status()
    ro, rl, _ = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss, True, window,
                                 n_sink)
    B, Hq, d = q.shape[0], q.shape[1], q.shape[3]
    ro = torch.from_numpy(ro.reshape(B, Hq, T, d))
    rl = torch.from_numpy(rl.reshape(B, Hq, T, 1))
    for rank, (o_r, lse_r) in enumerate(outs):
        want = ring.zigzag_gather(ro, world, rank).numpy()
        emax, emean = err_stats(to_f64(o_r), want)
        assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (rank, emax, emean)
        wl = ring.zigzag_gather(rl, world, rank).numpy()[..., 0]
        assert err_stats(to_f64(lse_r), wl)[0] <= LSE_ABS
