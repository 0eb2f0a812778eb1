"""The half-split pair layout (i, i + d/2) through every rotating kernel, against the
oracle's half-split rotation: prefill (queries in the attention prologue, keys in the
rotated-key pass, the rotated-key cache copy), chunked prefill and decode."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from tests._util import O_MAX_ABS, O_MEAN_ABS, ROT_ABS, err_stats, to_bits, to_f64
from yarn_position_scaling_b200 import api, build, synth

pytestmark = pytest.mark.gpu

LSE_ABS = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    api.load()


def _tables(w, pairs):
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta,
                              pairs=pairs)
    th, _, ss = oracle.rope_theta(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    return tab, th, ss


@pytest.mark.parametrize("w,T,d,Hq,Hkv,window,n_sink", [
    (synth.TINY, 256, 64, 4, 2, 0, 0),
    (synth.LLAMA3_128K, 700, 128, 8, 2, 0, 0),
    (synth.LLAMA3_128K, 900, 128, 4, 4, 200, 4),
    (synth.LLAMA2_16K, 333, 64, 6, 3, 0, 0),
])
def test_prefill_half_pairs(w, T, d, Hq, Hkv, window, n_sink):
    w = dataclasses.replace(w, d=d, Hq=Hq, Hkv=Hkv)
    q, k, v = synth.prefill_inputs(w, "cuda", T=T)
    tab, th, ss = _tables(w, "half")
    assert tab.pairs == api.PAIR_HALF
    lse = torch.empty(q.shape[:3], device="cuda")
    qd = torch.empty(q.shape, device="cuda")
    kd = torch.empty(k.shape, device="cuda")
    cache = torch.zeros(k.shape, dtype=torch.bfloat16, device="cuda")
    o = api.attn_prefill(q, k, v, tab, True, window, n_sink, lse=lse, q_rot_dbg=qd,
                         k_rot_dbg=kd, k_cache=cache)
    api.device_status()
    ro, rl, rq = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss, True, window,
                                  n_sink, want_qrot=True, pairs="half")
    emax, emean = err_stats(to_f64(o).reshape(ro.shape), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(to_f64(lse).reshape(-1), rl)[0] <= LSE_ABS
    assert err_stats(to_f64(qd).reshape(rq.shape), rq)[0] <= ROT_ABS
    pos = np.tile(np.arange(T, dtype=np.float64), Hkv)
    rk = oracle.rotate(to_bits(k).reshape(-1, d), pos, th, pairs="half")
    assert err_stats(to_f64(kd).reshape(rk.shape), rk)[0] <= ROT_ABS
    got = to_f64(cache).reshape(rk.shape)
    assert np.all(np.abs(got - rk) <= 1e-3 + np.abs(rk) * 2.0 ** -8)
    # and it is not the interleaved result
    o_int = api.attn_prefill(q, k, v, _tables(w, "interleaved")[0], True, window, n_sink)
    assert (o_int.float() - o.float()).abs().max().item() > 0.05


@pytest.mark.parametrize("d", [64, 128])
def test_decode_half_pairs(d):
    w = dataclasses.replace(synth.DECODE, d=d, Hq=8, Hkv=2)
    lens = [0, 5, 2047, 2048, 2999]
    qn, kn, vn, kc, vc, _ = synth.decode_inputs(w, "cuda", T_max=3000, B=len(lens))
    cl = torch.tensor(lens, dtype=torch.int32)
    kc0, vc0 = to_bits(kc), to_bits(vc)
    tab, th, ss = _tables(w, "half")
    qd = torch.empty(qn.shape, device="cuda")
    o = api.attn_decode(qn, kn, vn, kc, vc, cl.cuda(), tab, 300, 4, q_rot_dbg=qd)
    api.device_status()
    ro, _, rk, rq = oracle.decode(to_bits(qn), to_bits(kn), to_bits(vn), kc0, vc0, cl.numpy(),
                                  th, ss, 300, 4, pairs="half")
    emax, emean = err_stats(to_f64(o), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(to_f64(qd), rq)[0] <= ROT_ABS
    kslot = np.stack([to_f64(kc)[b, :, lens[b]] for b in range(len(lens))])
    assert np.all(np.abs(kslot - rk) <= 1e-3 + np.abs(rk) * 2.0 ** -8)


@pytest.mark.parametrize("fp16cache", [False, True])
def test_chunk_half_pairs(fp16cache):
    w = dataclasses.replace(synth.CHUNK, Hq=8, Hkv=2)
    P0, Tq, T_max = 600, 300, 1000
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=P0, Tq=Tq, T_max=T_max)
    kc0, vc0 = to_bits(kc), to_bits(vc)
    tab, th, ss = _tables(w, "half")
    if fp16cache:
        k16 = torch.zeros(kc.shape, dtype=torch.float16, device="cuda")
        v16 = torch.zeros(vc.shape, dtype=torch.float16, device="cuda")
        o = api.attn_prefill_chunk_fp16cache(q, kn, vn, kc, vc, k16, v16, 0, P0, tab)
    else:
        o = api.attn_prefill_chunk(q, kn, vn, kc, vc, P0, tab)
    api.device_status()
    ro, _, rk = oracle.prefill_chunk(to_bits(q), to_bits(kn), to_bits(vn), kc0, vc0, P0, th, ss,
                                     pairs="half")
    emax, emean = err_stats(to_f64(o), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    kslot = to_f64(kc)[:, :, P0:P0 + Tq]
    assert np.all(np.abs(kslot - rk) <= 1e-3 + np.abs(rk) * 2.0 ** -8)

