"""Decode parity: split-KV decode through the C ABI against the fp64 oracle, plus
the cross-path check that decode at position L equals prefill row L."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from tests._util import O_MAX_ABS, O_MEAN_ABS, ROT_ABS, err_stats, to_bits, to_f64
from yarn_position_scaling_b200 import api, build, synth

pytestmark = pytest.mark.gpu

# The new key enters the score as the bf16 value written to the cache: one rounding of
# k~ (2^-9 relative) moves its logit by up to scale * |q~| |k~| 2^-9 (~0.036 at d=128 for
# N(0,1) data, ~0.003 typically); with one visible key the LSE is that logit.
LSE_ABS = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    api.load()


def run_decode(w, lens, T_max, window=0, n_sink=0, table_kw=None):
    B = len(lens)
    qn, kn, vn, kc, vc, _ = synth.decode_inputs(w, "cuda", T_max=T_max, B=B)
    cl = torch.tensor(lens, dtype=torch.int32)
    kc0, vc0 = to_bits(kc), to_bits(vc)
    table_kw = table_kw or {}
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta,
                              **table_kw)
    lse = torch.empty(qn.shape[:2], device="cuda")
    qd = torch.empty(qn.shape, device="cuda")
    o = api.attn_decode(qn, kn, vn, kc, vc, cl.cuda(), tab, window, n_sink, lse=lse,
                        q_rot_dbg=qd)
    api.device_status()
    th, _, ss = oracle.rope_theta(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta,
                                  **table_kw)
    ro, rl, rk, rq = oracle.decode(to_bits(qn), to_bits(kn), to_bits(vn), kc0, vc0, cl.numpy(),
                                   th, ss, window, n_sink)
    emax, emean = err_stats(to_f64(o), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(to_f64(lse), rl)[0] <= LSE_ABS
    assert err_stats(to_f64(qd), rq)[0] <= ROT_ABS
    # slot L of each sequence now holds the rotated new key (bf16) and the new value
    kslot = np.stack([to_f64(kc)[b, :, lens[b]] for b in range(B)])
    assert np.all(np.abs(kslot - rk) <= 1e-3 + np.abs(rk) * 2.0 ** -8)
    vslot = torch.stack([vc[b, :, lens[b]] for b in range(B)])
    assert torch.equal(vslot, vn)
    # every other slot is untouched
    for b in range(B):
        before = kc0[b].copy()
        after = to_bits(kc)[b]
        before[:, lens[b]] = after[:, lens[b]]
        assert np.array_equal(before, after)
    return emax, emean


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 8, 128), (8, 8, 128), (16, 1, 64), (8, 1, 128),
                                      (12, 4, 64)])
def test_decode_lengths_across_chunk_edges(Hq, Hkv, d):
    w = dataclasses.replace(synth.DECODE, Hq=Hq, Hkv=Hkv, d=d)
    run_decode(w, [0, 1, 63, 64, 2047, 2048, 2049, 4999], T_max=5000)


@pytest.mark.parametrize("window,n_sink", [(300, 4), (64, 0), (2048, 1), (5000, 8), (1, 0)])
def test_decode_window_and_sinks(window, n_sink):
    run_decode(synth.DECODE, [0, 5, 299, 300, 2100, 4500, 4999], T_max=5000, window=window,
               n_sink=n_sink)


def test_decode_full_workload():
    w = synth.DECODE
    lens = synth.cache_lengths(w).tolist()
    run_decode(w, lens, T_max=w.T)


def test_decode_reports_bad_cache_length():
    w = dataclasses.replace(synth.DECODE, Hq=8, Hkv=2)
    qn, kn, vn, kc, vc, _ = synth.decode_inputs(w, "cuda", T_max=64, B=2)
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method)
    cl = torch.tensor([10, 64], dtype=torch.int32, device="cuda")  # 64 == T_max: no free slot
    o = api.attn_decode(qn, kn, vn, kc, vc, cl, tab)
    with pytest.raises(api.YarnAttnError) as ei:
        api.device_status()
    assert ei.value.code == api.YR_EINVAL
    assert torch.isnan(o[1].float()).all() and torch.isfinite(o[0].float()).all()
    api.device_status()  # cleared


@pytest.mark.parametrize("L", [1, 130, 2500])
def test_decode_at_L_equals_prefill_row_L(L):
    w = synth.LLAMA3_128K
    T = L + 1
    q, k, v = synth.prefill_inputs(w, "cuda", T=T)
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method)
    T_max = T + 5
    kcache = torch.zeros((1, w.Hkv, T_max, w.d), dtype=torch.bfloat16, device="cuda")
    vcache = torch.zeros_like(kcache)
    pre = api.attn_prefill(q, k, v, tab, k_cache=kcache[:, :, :T])
    vcache[:, :, :T] = v
    kcache[:, :, L] = 0  # the decode writes slot L itself
    cl = torch.tensor([L], dtype=torch.int32, device="cuda")
    dec = api.attn_decode(q[:, :, L].contiguous(), k[:, :, L].contiguous(),
                          v[:, :, L].contiguous(), kcache, vcache, cl, tab)
    api.device_status()
    th, _, ss = oracle.rope_theta(w.d, w.base, w.L_train, w.scale, w.method)
    rows = np.array([h * T + L for h in range(w.Hq)], dtype=np.int64)
    ro, _, _ = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss, rows=rows)
    assert err_stats(to_f64(pre[0, :, L]), ro)[0] <= O_MAX_ABS
    assert err_stats(to_f64(dec[0]), ro)[0] <= O_MAX_ABS
    assert err_stats(to_f64(dec[0]), to_f64(pre[0, :, L]))[0] <= 2 * O_MAX_ABS


@pytest.mark.parametrize("method,kw", [
    ("ntk_dynamic", {"L_cur": 9001}),  # one table per call: the longest sequence's length
    ("yarn_dimramp", {}),
    ("factors", {"factors": np.geomspace(1.0, 16.0, 64), "attn_factor": 1.2}),
])
def test_decode_table_variants(method, kw):
    w = dataclasses.replace(synth.DECODE, method=method, B=2)
    run_decode(w, [4000, 9000], 9001, table_kw=kw)


@pytest.mark.parametrize("Hq,Hkv,window,n_sink", [(32, 8, 0, 0), (8, 2, 3000, 4)])
def test_decode_alibi(Hq, Hkv, window, n_sink):
    w = dataclasses.replace(synth.DECODE, Hq=Hq, Hkv=Hkv, B=2, method="alibi")
    lens = [4000, 9000]
    qn, kn, vn, kc, vc, _ = synth.decode_inputs(w, "cuda", T_max=9001, B=2)
    cl = torch.tensor(lens, dtype=torch.int32)
    kc0, vc0 = to_bits(kc), to_bits(vc)
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, "alibi")
    lse = torch.empty(qn.shape[:2], device="cuda")
    o = api.attn_decode(qn, kn, vn, kc, vc, cl.cuda(), tab, window, n_sink, lse=lse)
    api.device_status()
    ro, rl, _, _ = oracle.decode(to_bits(qn), to_bits(kn), to_bits(vn), kc0, vc0, cl.numpy(),
                                 np.zeros(w.d // 2), 1.0 / np.sqrt(w.d), window, n_sink,
                                 slopes=oracle.alibi_slopes(Hq))
    emax, emean = err_stats(to_f64(o), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(to_f64(lse), rl)[0] <= LSE_ABS
