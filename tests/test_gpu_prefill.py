"""Prefill parity: the CUDA path through the C ABI against the fp64 oracle.

Small shapes compare every output element; the full-size workloads (launched
exactly as bench.py launches them) compare sampled query rows, always including
the tile edges and the window edges.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from tests._util import O_MAX_ABS, O_MEAN_ABS, ROT_ABS, err_stats, to_bits, to_f64
from yarn_position_scaling_b200 import api, build, synth

pytestmark = pytest.mark.gpu

LSE_ABS = 5e-3  # natural-log units; fp16 operands move logits by ~1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    api.load()
    assert torch.cuda.is_available()


def _table(w, d=None, **kw):
    return api.rope_freq_table(d or w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta,
                               **kw)


def _oracle_table(w, d=None, **kw):
    return oracle.rope_theta(d or w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta,
                             **kw)


def run_full(w, T, B=1, causal=True, window=0, n_sink=0, d=None, Hq=None, Hkv=None,
             table_kw=None):
    w = dataclasses.replace(w, d=d or w.d, Hq=Hq or w.Hq, Hkv=Hkv or w.Hkv)
    table_kw = table_kw or {}
    q, k, v = synth.prefill_inputs(w, "cuda", T=T, B=B)
    tab = _table(w, **table_kw)
    lse = torch.empty(q.shape[:3], device="cuda")
    qd = torch.empty(q.shape, device="cuda")
    kd = torch.empty(k.shape, device="cuda")
    o = api.attn_prefill(q, k, v, tab, causal, window, n_sink, lse=lse, q_rot_dbg=qd,
                         k_rot_dbg=kd)
    api.device_status()
    th, _, ss = _oracle_table(w, **table_kw)
    ro, rl, rq = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss, causal, window,
                                  n_sink, want_qrot=True)
    emax, emean = err_stats(to_f64(o).reshape(ro.shape), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(to_f64(lse).reshape(-1), rl)[0] <= LSE_ABS
    assert err_stats(to_f64(qd).reshape(rq.shape), rq)[0] <= ROT_ABS
    pos = np.tile(np.arange(T, dtype=np.float64), B * w.Hkv)
    rk = oracle.rotate(to_bits(k).reshape(-1, w.d), pos, th)
    assert err_stats(to_f64(kd).reshape(rk.shape), rk)[0] <= ROT_ABS
    return emax, emean


def test_tiny_workload_every_element():
    run_full(synth.TINY, synth.TINY.T)


@pytest.mark.parametrize("B,Hq,Hkv,T,d", [
    (1, 4, 2, 1, 64),       # a single token
    (1, 4, 2, 127, 64),     # one partial tile
    (1, 2, 1, 129, 128),    # one key past a tile boundary, MQA
    (2, 4, 4, 300, 128),    # MHA, batch 2, ragged tail
    (1, 8, 1, 513, 64),     # 8 query heads on one KV head
    (1, 4, 4, 255, 128),
    (1, 4, 2, 257, 64),     # one row past a CTA's two tiles
    (1, 6, 2, 640, 128),    # several CTAs per head, group of 3
])
def test_shapes_and_ragged_tails(B, Hq, Hkv, T, d):
    run_full(synth.TINY, T, B=B, d=d, Hq=Hq, Hkv=Hkv)


@pytest.mark.parametrize("T,window,n_sink", [(700, 200, 4), (700, 128, 0), (900, 77, 130),
                                             (520, 1, 0), (400, 1000, 3), (1000, 256, 256)])
def test_window_and_sinks(T, window, n_sink):
    run_full(synth.LLAMA3_128K, T, window=window, n_sink=n_sink)


@pytest.mark.parametrize("B,Hq,Hkv,T,d,window,n_sink", [
    (1, 4, 2, 129, 128, 64, 0),      # two heads per CTA, one row past a tile
    (2, 8, 1, 1000, 64, 300, 4),     # eight query heads on one KV head, batch 2
    (1, 16, 2, 777, 128, 128, 130),  # sinks reaching past the first key tile
    (1, 6, 2, 700, 128, 200, 4),     # a group of three: one head per CTA
])
def test_window_head_pairs(B, Hq, Hkv, T, d, window, n_sink):
    """Windowed calls with an even number of query heads per KV head run two heads of one
    group at the same 128 rows in a CTA (odd groups keep 256 rows of one head)."""
    run_full(synth.LLAMA3_128K, T, B=B, d=d, Hq=Hq, Hkv=Hkv, window=window, n_sink=n_sink)


@pytest.mark.parametrize("T,d", [(200, 64), (300, 128)])
def test_non_causal(T, d):
    run_full(synth.TINY, T, causal=False, d=d)


@pytest.mark.parametrize("method", ["rope", "pi", "ntk", "yarn"])
def test_position_methods(method):
    run_full(synth.sweep(method, False), 600)


# Table variants (dynamic NTK, dimension-ramp YaRN, per-dimension factors): the kernels
# consume the table as given, so one small shape per variant checks that it arrives.
TABLE_VARIANTS = [
    ("ntk_dynamic", {"L_cur": 3000}),     # below L_train: plain RoPE
    ("ntk_dynamic", {"L_cur": 40000}),    # s = 40000 / 4096
    ("yarn_dimramp", {}),
    ("factors", {"factors": np.geomspace(1.0, 16.0, 64), "attn_factor": 1.2}),
]


@pytest.mark.parametrize("method,kw", TABLE_VARIANTS)
def test_table_variants(method, kw):
    run_full(dataclasses.replace(synth.sweep("yarn", False), method=method), 600, table_kw=kw)


@pytest.mark.parametrize("Hq,Hkv,T,window,n_sink", [(8, 2, 600, 0, 0), (8, 2, 700, 256, 4),
                                                    (32, 8, 1000, 0, 0), (4, 4, 300, 0, 0)])
def test_alibi(Hq, Hkv, T, window, n_sink):
    # ALiBi: no rotation, the bias -m_h (i - j) on the logits (slopes 2^(-8(h+1)/Hq))
    w = dataclasses.replace(synth.LLAMA3_128K, Hq=Hq, Hkv=Hkv, method="alibi")
    q, k, v = synth.prefill_inputs(w, "cuda", T=T)
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, "alibi")
    lse = torch.empty(q.shape[:3], device="cuda")
    o = api.attn_prefill(q, k, v, tab, True, window, n_sink, lse=lse)
    api.device_status()
    ro, rl, _ = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), np.zeros(w.d // 2),
                                 1.0 / np.sqrt(w.d), True, window, n_sink,
                                 slopes=oracle.alibi_slopes(Hq))
    emax, emean = err_stats(to_f64(o).reshape(ro.shape), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(to_f64(lse).reshape(-1), rl)[0] <= LSE_ABS


def test_strided_inputs_and_outputs_match_contiguous():
    w = synth.LLAMA3_128K
    T = 333
    q, k, v = synth.prefill_inputs(w, "cuda", T=T)
    tab = _table(w)
    ref = api.attn_prefill(q, k, v, tab)
    # [B, T, H, d] storage seen as [B, H, T, d]
    qt = q.transpose(1, 2).contiguous().transpose(1, 2)
    kt = k.transpose(1, 2).contiguous().transpose(1, 2)
    vt = v.transpose(1, 2).contiguous().transpose(1, 2)
    out = torch.empty((1, T, w.Hq, w.d), dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    api.attn_prefill(qt, kt, vt, tab, out=out)
    api.device_status()
    assert torch.equal(out, ref)


def test_rotated_key_cache_output():
    w = synth.LLAMA2_16K
    T = 260
    q, k, v = synth.prefill_inputs(w, "cuda", T=T)
    tab = _table(w)
    T_max = 300
    cache = torch.zeros((1, w.Hkv, T_max, w.d), dtype=torch.bfloat16, device="cuda")
    api.attn_prefill(q, k, v, tab, k_cache=cache[:, :, :T])
    api.device_status()
    th, _, _ = _oracle_table(w)
    pos = np.tile(np.arange(T, dtype=np.float64), w.Hkv)
    rk = oracle.rotate(to_bits(k).reshape(-1, w.d), pos, th).reshape(1, w.Hkv, T, w.d)
    got = to_f64(cache[:, :, :T])
    assert np.all(np.abs(got - rk) <= 1e-3 + np.abs(rk) * 2.0 ** -8)
    assert torch.count_nonzero(cache[:, :, T:]) == 0


def test_repeated_calls_are_bitwise_deterministic():
    w = synth.LLAMA3_128K
    q, k, v = synth.prefill_inputs(w, "cuda", T=1000)
    tab = _table(w)
    a = api.attn_prefill(q, k, v, tab, window=300, n_sink=4)
    b = api.attn_prefill(q, k, v, tab, window=300, n_sink=4)
    api.device_status()
    assert torch.equal(a, b)


# ---------------------------------------------------------- full-size workloads

def sample_rows(w, T, n_heads=8, per_head=36, seed=0):
    rng = np.random.default_rng(seed)
    heads = sorted(set([0, w.Hq - 1] + rng.choice(w.Hq, n_heads - 2, replace=False).tolist()))
    fixed = [0, 1, 2, 127, 128, 129, 255, 256, T // 2, T - 2, T - 1]
    if w.window:
        W = w.window
        fixed += [W - 1, W, W + 1, W + 3, W + 4, W + 127, W + 128]
    rows = []
    for b in range(w.B):
        for h in heads:
            ms = sorted(set(fixed + rng.integers(0, T, per_head - len(fixed)).tolist()))
            rows += [(b * w.Hq + h) * T + m for m in ms if 0 <= m < T]
    return np.array(rows, dtype=np.int64)


def check_sampled(w):
    q, k, v = synth.prefill_inputs(w, "cuda")
    tab = _table(w)
    ws = torch.empty(api.attn_prefill_workspace_bytes(w.B, w.Hkv, w.T, w.d), dtype=torch.uint8,
                     device="cuda")
    lse = torch.empty(q.shape[:3], device="cuda")
    o = api.attn_prefill(q, k, v, tab, w.causal, w.window, w.n_sink, lse=lse, workspace=ws)
    api.device_status()
    rows = sample_rows(w, w.T)
    th, _, ss = _oracle_table(w)
    ro, rl, _ = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss, w.causal, w.window,
                                 w.n_sink, rows=rows)
    got = to_f64(o).reshape(-1, w.d)[rows]
    emax, emean = err_stats(got, ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (w.name, emax, emean)
    assert err_stats(to_f64(lse).reshape(-1)[rows], rl)[0] <= LSE_ABS
    assert torch.isfinite(o).all()


def test_llama2_16k_sampled_rows():
    check_sampled(synth.LLAMA2_16K)


def test_llama3_128k_sampled_rows():
    check_sampled(synth.LLAMA3_128K)


@pytest.mark.parametrize("w", synth.SWEEP, ids=[w.name for w in synth.SWEEP])
def test_sweep_sampled_rows(w):
    check_sampled(w)


def test_host_prefill_pipeline_matches_device_call():
    # pinned host in, pinned host out, transfers overlapped per (batch, KV-head group)
    for w, T, B in [(synth.TINY, 700, 2), (synth.LLAMA3_128K, 1000, 1)]:
        q, k, v = synth.prefill_inputs(w, "cpu", T=T, B=B)
        qh, kh, vh = [t.pin_memory() for t in (q, k, v)]
        tab = _table(w)
        hp = api.HostPrefill(B, w.Hq, w.Hkv, T, w.d, units_per_batch=3)
        got = hp(qh, kh, vh, tab, True, 300, 4)
        torch.cuda.synchronize()
        again = hp(qh, kh, vh, tab, True, 300, 4)
        torch.cuda.synchronize()
        ref = api.attn_prefill(q.cuda(), k.cuda(), v.cuda(), tab, True, 300, 4)
        api.device_status()
        assert torch.equal(got, ref.cpu()) and torch.equal(again, ref.cpu())
