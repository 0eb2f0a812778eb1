"""The largest sizes of the path on one GPU: a prefill of 2^20 tokens and a decode over a
cache of 2^20 keys (the Llama-3-8B-shaped heads of the 128K workload, YaRN with the
128K table).

Positions up to 2^20 test the angle reduction far from 0 (the fp64 reduction of the
first row of each warp, the fp32 lane offset) and grids of 131,072 CTAs.  The full
prefill output is 8 GB, so the check gathers sampled rows of two query heads on the
GPU and compares them, and the log-sum-exp, with the oracle run on those heads only.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from tests._util import O_MAX_ABS, O_MEAN_ABS, err_stats, to_bits, to_f64
from yarn_position_scaling_b200 import api, build, synth

pytestmark = pytest.mark.gpu

T_MILLION = 1 << 20
LSE_ABS = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    api.load()


def _tables(w):
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    th, _, ss = oracle.rope_theta(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    return tab, th, ss


def test_million_token_prefill_sampled_rows():
    w = synth.LLAMA3_1M
    assert w.T == T_MILLION
    q, k, v = synth.prefill_inputs(w, "cuda")
    tab, th, ss = _tables(w)
    lse = torch.empty(q.shape[:3], device="cuda")
    o = api.attn_prefill(q, k, v, tab, lse=lse)
    api.device_status()
    rng = np.random.default_rng(11)
    T, g = w.T, w.Hq // w.Hkv
    ms = np.array(sorted(set([0, 1, 127, 128, 255, 256, T // 2, T - 257, T - 256, T - 2, T - 1] +
                             rng.integers(0, T, 13).tolist())), dtype=np.int64)
    for h in (0, w.Hq - 1):
        kvh = h // g
        # the oracle on this head alone: q [1,1,T,d] against its KV head's k, v
        qh = to_bits(q[:, h:h + 1])
        kh, vh = to_bits(k[:, kvh:kvh + 1]), to_bits(v[:, kvh:kvh + 1])
        ro, rl, _ = oracle.attn_rows(qh, kh, vh, th, ss, True, 0, 0, rows=ms)
        idx = torch.from_numpy(ms).cuda()
        got = to_f64(o[0, h].index_select(0, idx))
        emax, emean = err_stats(got, ro)
        assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (h, emax, emean)
        assert err_stats(to_f64(lse[0, h].index_select(0, idx)), rl)[0] <= LSE_ABS
        assert torch.isfinite(o[0, h]).all()
    del q, k, v, o, lse
    torch.cuda.empty_cache()


def test_decode_over_a_million_token_cache():
    w = dataclasses.replace(synth.DECODE, B=2)
    T_max = T_MILLION + 1
    qn, kn, vn, kc, vc, _ = synth.decode_inputs(w, "cuda", T_max=T_max, B=2)
    lens = np.array([T_MILLION, 777_777], dtype=np.int32)
    kc0, vc0 = to_bits(kc), to_bits(vc)
    tab, th, ss = _tables(w)
    lse = torch.empty((2, w.Hq), device="cuda")
    o = api.attn_decode(qn, kn, vn, kc, vc, torch.from_numpy(lens).cuda(), tab, lse=lse)
    api.device_status()
    ro, rl, _, _ = oracle.decode(to_bits(qn), to_bits(kn), to_bits(vn), kc0, vc0, lens, th, ss)
    emax, emean = err_stats(to_f64(o), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(to_f64(lse), rl)[0] <= LSE_ABS
    # the new key and value land in slot L_b of each sequence
    for b in range(2):
        assert torch.equal(vc[b, :, int(lens[b])], vn[b])
    del kc, vc
    torch.cuda.empty_cache()
