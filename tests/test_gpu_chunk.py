"""Chunked prefill after a cached prefix: the CUDA path through the C ABI against the
fp64 oracle, plus cross-path checks (P0 = 0 is a causal prefill, Tq = 1 is decode)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from tests._util import O_MAX_ABS, O_MEAN_ABS, err_stats, to_bits, to_f64
from yarn_position_scaling_b200 import api, build, synth

pytestmark = pytest.mark.gpu

LSE_ABS = 5e-3  # as prefill: fp16 operands move logits by ~1e-3; cached keys are used as given


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    api.load()


def _tables(w):
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    th, _, ss = oracle.rope_theta(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    return tab, th, ss


def run_chunk(w, P0, Tq, T_max, B=1, window=0, n_sink=0, rows=None):
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=P0, Tq=Tq, T_max=T_max, B=B)
    kc0, vc0 = to_bits(kc), to_bits(vc)
    tab, th, ss = _tables(w)
    lse = torch.empty(q.shape[:3], device="cuda")
    o = api.attn_prefill_chunk(q, kn, vn, kc, vc, P0, tab, window, n_sink, lse=lse)
    api.device_status()
    ro, rl, rk = oracle.prefill_chunk(to_bits(q), to_bits(kn), to_bits(vn), kc0, vc0, P0, th, ss,
                                      window, n_sink)
    emax, emean = err_stats(to_f64(o), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(to_f64(lse), rl)[0] <= LSE_ABS
    # slots P0 .. P0+Tq-1 hold the rotated new keys (bf16) and the new values; the rest is
    # untouched
    kslot = to_f64(kc)[:, :, P0:P0 + Tq]
    assert np.all(np.abs(kslot - rk) <= 1e-3 + np.abs(rk) * 2.0 ** -8)
    assert torch.equal(vc[:, :, P0:P0 + Tq], vn)
    after_k, after_v = to_bits(kc), to_bits(vc)
    for arr0, arr1 in ((kc0, after_k), (vc0, after_v)):
        assert np.array_equal(arr0[:, :, :P0], arr1[:, :, :P0])
        assert np.array_equal(arr0[:, :, P0 + Tq:], arr1[:, :, P0 + Tq:])
    return emax, emean


SMALL = dataclasses.replace(synth.CHUNK, Hq=8, Hkv=2)


@pytest.mark.parametrize("P0,Tq", [(0, 300), (128, 256), (200, 77), (1000, 1), (777, 513),
                                   (4096, 129)])
def test_chunk_offsets_and_ragged_sizes(P0, Tq):
    run_chunk(SMALL, P0, Tq, P0 + Tq + 50)


@pytest.mark.parametrize("window,n_sink", [(256, 0), (300, 4), (64, 1)])
def test_chunk_window_and_sinks(window, n_sink):
    run_chunk(SMALL, 900, 400, 1400, window=window, n_sink=n_sink)


@pytest.mark.parametrize("Hq,Hkv,d", [(4, 4, 64), (8, 1, 128), (12, 4, 64)])
def test_chunk_heads_and_head_dims(Hq, Hkv, d):
    run_chunk(dataclasses.replace(synth.CHUNK, Hq=Hq, Hkv=Hkv, d=d), 333, 200, 600, B=2)


def test_chunk_at_zero_matches_causal_prefill():
    w = SMALL
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=0, Tq=500, T_max=500)
    tab, _, _ = _tables(w)
    o_chunk = api.attn_prefill_chunk(q, kn, vn, kc, vc, 0, tab)
    o_full = api.attn_prefill(q, kn, vn, tab)
    assert torch.equal(o_chunk, o_full)


def test_chunk_of_one_token_matches_decode():
    w = SMALL
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=5000, Tq=1, T_max=5001)
    kc2, vc2 = kc.clone(), vc.clone()
    tab, _, _ = _tables(w)
    o_chunk = api.attn_prefill_chunk(q, kn, vn, kc, vc, 5000, tab)
    o_dec = api.attn_decode(q[:, :, 0].contiguous(), kn[:, :, 0].contiguous(),
                            vn[:, :, 0].contiguous(), kc2, vc2,
                            torch.tensor([5000], dtype=torch.int32, device="cuda"), tab)
    # two different kernels (fp16 tensor-core tiles against fp32 split-KV): both within the
    # tolerance of the oracle, and of each other
    err = (o_chunk[:, :, 0].float() - o_dec.float()).abs()
    assert err.max().item() <= 2 * O_MAX_ABS and err.mean().item() <= O_MEAN_ABS
    assert torch.equal(vc[:, :, 5000], vc2[:, :, 5000])


def test_chunk_workload_sampled():
    # the bench's workload shape (124K cached prefix + 4K chunk), all heads, every query row
    # of the chunk's first and last tiles compared in full against the oracle
    w = synth.CHUNK
    P0, Tq = w.P0, 256
    run_chunk(dataclasses.replace(w, Hq=8, Hkv=2), P0, Tq, P0 + Tq)


def test_chunk_rejects_bad_arguments():
    w = SMALL
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=10, Tq=20, T_max=25)
    tab, _, _ = _tables(w)
    with pytest.raises(api.YarnAttnError):
        api.attn_prefill_chunk(q, kn, vn, kc, vc, 10, tab)  # P0 + Tq > T_max
    with pytest.raises(api.YarnAttnError):
        api.attn_prefill_chunk(q, kn, vn, kc, vc, 0, tab, 0, 4)  # sinks without a window


def test_chunk_alibi():
    w = dataclasses.replace(SMALL, method="alibi")
    P0, Tq, T_max = 700, 300, 1000
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=P0, Tq=Tq, T_max=T_max)
    kc0, vc0 = to_bits(kc), to_bits(vc)
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, "alibi")
    o = api.attn_prefill_chunk(q, kn, vn, kc, vc, P0, tab)
    api.device_status()
    ro, _, _ = oracle.prefill_chunk(to_bits(q), to_bits(kn), to_bits(vn), kc0, vc0, P0,
                                    np.zeros(w.d // 2), 1.0 / np.sqrt(w.d),
                                    slopes=oracle.alibi_slopes(w.Hq))
    emax, emean = err_stats(to_f64(o), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    # no rotation: the appended keys are the new keys as given
    assert torch.equal(kc[:, :, P0:P0 + Tq], kn)
