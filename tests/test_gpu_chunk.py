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


# ------------------------------------------------- chunks with a kept fp16 cache copy

def test_fp16cache_matches_the_workspace_form_bit_for_bit():
    w = SMALL
    P0, Tq, T_max = 777, 513, 1400
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=P0, Tq=Tq, T_max=T_max)
    tab, _, _ = _tables(w)
    kc2, vc2 = kc.clone(), vc.clone()
    lse1 = torch.empty(q.shape[:3], device="cuda")
    lse2 = torch.empty(q.shape[:3], device="cuda")
    ref = api.attn_prefill_chunk(q, kn, vn, kc, vc, P0, tab, 300, 4, lse=lse1)
    k16 = torch.full(kc.shape, float("nan"), dtype=torch.float16, device="cuda")
    v16 = torch.full(vc.shape, float("nan"), dtype=torch.float16, device="cuda")
    got = api.attn_prefill_chunk_fp16cache(q, kn, vn, kc2, vc2, k16, v16, 0, P0, tab, 300, 4,
                                           lse=lse2)
    api.device_status()
    assert torch.equal(got, ref) and torch.equal(lse2, lse1)
    assert torch.equal(kc2, kc) and torch.equal(vc2, vc)
    # the converted prefix is the fp16 value of the bf16 cache; the chunk's keys are its fp32
    # rotation rounded once to fp16 (the bf16 cache holds the same rotation rounded to bf16);
    # values are copied; slots past the chunk are untouched
    assert torch.equal(k16[:, :, :P0], kc[:, :, :P0].to(torch.float16))
    _same_rotation(k16[:, :, P0:P0 + Tq], kc[:, :, P0:P0 + Tq])
    assert torch.equal(v16[:, :, :P0 + Tq], vc[:, :, :P0 + Tq].to(torch.float16))
    assert torch.isnan(k16[:, :, P0 + Tq:]).all() and torch.isnan(v16[:, :, P0 + Tq:]).all()


def _same_rotation(k16, kbf16):
    """An fp16 and a bf16 rounding of the same fp32 rotated keys: within one bf16 rounding."""
    a, b = k16.float(), kbf16.float()
    assert torch.all((a - b).abs() <= b.abs() * 2.0 ** -8 + 1e-6)


def test_fp16cache_chunk_sequence_against_the_oracle():
    # a prompt fed in chunks of 300, 257, 1 and 700 tokens; each call converts only what
    # the copy lacks (nothing after the first), and two decode-appended slots are picked
    # up by passing the last valid length
    w = SMALL
    T_max = 1400
    tab, th, ss = _tables(w)
    _, _, _, kc, vc = synth.chunk_inputs(w, "cuda", P0=0, Tq=1, T_max=T_max)
    k16 = torch.zeros(kc.shape, dtype=torch.float16, device="cuda")
    v16 = torch.zeros(vc.shape, dtype=torch.float16, device="cuda")
    P0, valid = 0, 0
    for i, Tq in enumerate([300, 257, 1, 700]):
        if i == 3:
            P0 += 2      # two slots appended to the bf16 cache by someone else
        qq, kn, vn, _, _ = synth.chunk_inputs(dataclasses.replace(w, seed=w.seed + 10 + i),
                                              "cuda", P0=P0, Tq=Tq, T_max=T_max)
        kc0, vc0 = to_bits(kc), to_bits(vc)
        o = api.attn_prefill_chunk_fp16cache(qq, kn, vn, kc, vc, k16, v16, valid, P0, tab,
                                             256, 4)
        api.device_status()
        ro, _, _ = oracle.prefill_chunk(to_bits(qq), to_bits(kn), to_bits(vn), kc0, vc0, P0, th,
                                        ss, 256, 4)
        emax, emean = err_stats(to_f64(o), ro)
        assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (i, emax, emean)
        _same_rotation(k16[:, :, P0:P0 + Tq], kc[:, :, P0:P0 + Tq])
        P0 += Tq
        valid = P0
        assert torch.equal(v16[:, :, :P0], vc[:, :, :P0].to(torch.float16))


def test_fp16cache_small_chunk_after_a_long_prefix():
    # 256 new tokens after a 124K prefix that is already in the fp16 copy: only the
    # chunk's rows are written; sampled rows against the oracle
    w = dataclasses.replace(synth.CHUNK, Hq=8, Hkv=2)
    P0, Tq = w.P0, 256
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=P0, Tq=Tq, T_max=P0 + Tq)
    kc0, vc0 = to_bits(kc), to_bits(vc)
    k16, v16 = kc.to(torch.float16), vc.to(torch.float16)
    tab, th, ss = _tables(w)
    o = api.attn_prefill_chunk_fp16cache(q, kn, vn, kc, vc, k16, v16, P0, P0, tab)
    api.device_status()
    ro, _, _ = oracle.prefill_chunk(to_bits(q), to_bits(kn), to_bits(vn), kc0, vc0, P0, th, ss)
    emax, emean = err_stats(to_f64(o), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)


def test_fp16cache_rejects_bad_arguments():
    w = SMALL
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=10, Tq=20, T_max=40)
    tab, _, _ = _tables(w)
    k16 = torch.zeros(kc.shape, dtype=torch.float16, device="cuda")
    v16 = torch.zeros(vc.shape, dtype=torch.float16, device="cuda")
    with pytest.raises(api.YarnAttnError) as ei:
        api.attn_prefill_chunk_fp16cache(q, kn, vn, kc, vc, k16, v16, 11, 10, tab)
    assert ei.value.code == api.YR_EINVAL and "cache16_len" in str(ei.value)
    with pytest.raises(api.YarnAttnError):
        api.attn_prefill_chunk_fp16cache(q, kn, vn, kc, vc, k16, v16, 0, 25, tab)  # > T_max
    api.device_status()


@pytest.mark.parametrize("P0,Tq,window,n_sink", [(5000, 100, 0, 0), (3000, 64, 1000, 4),
                                                 (2000, 300, 0, 0)])
def test_fp16cache_split_kv_against_the_oracle_and_unsplit(P0, Tq, window, n_sink):
    # few query blocks against a long prefix: the keys are cut into shares (split-KV)
    w = SMALL
    T_max = P0 + Tq
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=P0, Tq=Tq, T_max=T_max)
    kc0, vc0 = to_bits(kc), to_bits(vc)
    tab, th, ss = _tables(w)
    k16, v16 = kc.to(torch.float16), vc.to(torch.float16)
    kc2, vc2, k16b, v16b = kc.clone(), vc.clone(), k16.clone(), v16.clone()
    lse = torch.empty(q.shape[:3], device="cuda")
    o = api.attn_prefill_chunk_fp16cache(q, kn, vn, kc, vc, k16, v16, P0, P0, tab, window,
                                         n_sink, lse=lse)
    o1 = api.attn_prefill_chunk_fp16cache(q, kn, vn, kc2, vc2, k16b, v16b, P0, P0, tab, window,
                                          n_sink, split=False)
    api.device_status()
    ro, rl, _ = oracle.prefill_chunk(to_bits(q), to_bits(kn), to_bits(vn), kc0, vc0, P0, th, ss,
                                     window, n_sink)
    emax, emean = err_stats(to_f64(o), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(to_f64(lse), rl)[0] <= LSE_ABS
    # the same operands, merged in another order: within one bf16 rounding of each other
    a, b = o.float(), o1.float()
    assert torch.all((a - b).abs() <= b.abs() * 2.0 ** -8 + 2e-3)
    assert torch.equal(kc, kc2) and torch.equal(k16, k16b)


def test_fp16cache_alibi_and_range_check():
    # ALiBi through the fp16-copy form; a prefix value past the fp16 limit in the slots the
    # call converts is reported as YR_ERANGE
    w = dataclasses.replace(SMALL, method="alibi")
    P0, Tq, T_max = 3000, 100, 3100
    q, kn, vn, kc, vc = synth.chunk_inputs(w, "cuda", P0=P0, Tq=Tq, T_max=T_max)
    kc0, vc0 = to_bits(kc), to_bits(vc)
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, "alibi")
    k16 = torch.zeros(kc.shape, dtype=torch.float16, device="cuda")
    v16 = torch.zeros(vc.shape, dtype=torch.float16, device="cuda")
    o = api.attn_prefill_chunk_fp16cache(q, kn, vn, kc, vc, k16, v16, 0, P0, tab)
    api.device_status()
    ro, _, _ = oracle.prefill_chunk(to_bits(q), to_bits(kn), to_bits(vn), kc0, vc0, P0,
                                    np.zeros(w.d // 2), 1.0 / np.sqrt(w.d),
                                    slopes=oracle.alibi_slopes(w.Hq))
    emax, emean = err_stats(to_f64(o), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    vc[0, 1, 17, 3] = 70000.0
    api.attn_prefill_chunk_fp16cache(q, kn, vn, kc, vc, k16, v16, 10, P0, tab)
    with pytest.raises(api.YarnAttnError) as ei:
        api.device_status()
    assert ei.value.code == api.YR_ERANGE
