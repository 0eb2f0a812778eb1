"""Inputs away from N(0, 1): peaked softmax, values near the fp16 limit, and values past it.

The prefill kernels hand the rotated queries and keys, the values and the
probabilities to the tensor cores as fp16 (11-bit significand, largest finite
value 65504).  Three things are checked here against the fp64 oracle:

* Peaked softmax (queries scaled by 8, 16 and 30 with the 128K workload's YaRN table)
  drives the online softmax through its tile-max and rescale path and makes a
  fresh row reject its trial reference of 0.  fp16 storage of a rotated operand
  moves a logit by up to ~2^-11 of its size, so with logits of tens of units the
  result differs from exact attention by more than the N(0, 1) tolerance; what
  is exact is attention of the operands as rounded.  The reference is therefore
  the oracle's attention on its own rotated q and k and on v, each rounded to
  fp16 by the test (numpy), and the output must match it within the stated
  tolerance plus the bf16 rounding of the output itself: a softmax this peaked
  copies single values of v, up to ~4.5 here, where one bf16 rounding reaches
  2^-9 |o| (0.009 at |o| = 4.5), so the bound per element is
  1e-2 + 2^-8 |o| and for the mean 1e-3 + 2^-9 mean|o|.
* Tiny logits (q = 0, q / 64): the first tile's probability sum falls below the
  trial-reference window, and q = 0 has a closed form (prefix means of v).
* Values near the fp16 limit (|v| up to 60000, |k~| ~ 10^4) keep their relative
  precision, so o / c matches the oracle's o / c within the N(0, 1) tolerances.
* A rotated query or key, or a value, at or past 65520 (or NaN) is reported as
  YR_ERANGE by yr_device_status instead of passing silently as infinity; 65280,
  the largest bf16 value below the limit, is not.
"""
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


W128K = synth.LLAMA3_128K


def _table(w):
    return api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)


def _oracle_table(w):
    return oracle.rope_theta(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)


def _scaled_inputs(w, T, cq=1.0, ck=1.0, cv=1.0, Hq=8, Hkv=2, v_uniform=False):
    q, k, v = synth.prefill_inputs(dataclasses.replace(w, Hq=Hq, Hkv=Hkv), "cpu", T=T)
    q = (q.float() * cq).to(torch.bfloat16)
    k = (k.float() * ck).to(torch.bfloat16)
    if v_uniform:
        g = torch.Generator().manual_seed(77)
        v = ((torch.rand(v.shape, generator=g) * 2 - 1) * cv).to(torch.bfloat16)
    else:
        v = (v.float() * cv).to(torch.bfloat16)
    return q, k, v


def _rotated(bits, th):
    B, H, T, d = bits.shape
    pos = np.broadcast_to(np.arange(T, dtype=np.float64), (B, H, T)).reshape(-1)
    return oracle.rotate(bits, pos, th).reshape(B, H, T, d)


def _f16(x):
    return np.asarray(x, np.float64).astype(np.float16).astype(np.float64)


def _run_gpu(q, k, v, tab, window=0, n_sink=0):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    lse = torch.empty(q.shape[:3], device="cuda")
    qrot = torch.empty(q.shape, device="cuda")
    o = api.attn_prefill(qd, kd, vd, tab, True, window, n_sink, lse=lse, q_rot_dbg=qrot)
    api.device_status()
    return to_f64(o), to_f64(lse), to_f64(qrot)


@pytest.mark.parametrize("cq,flip", [(8.0, 0.0), (16.0, 0.0), (30.0, 1e-2)])
@pytest.mark.parametrize("window,n_sink", [(0, 0), (200, 4)])
def test_peaked_softmax_matches_exact_attention_of_the_rounded_operands(cq, flip, window,
                                                                        n_sink):
    # `flip`: the kernel rotates in fp32 (angle within ~3e-7 turns), the oracle in fp64;
    # an element whose exact value lies that close to the midpoint between two fp16 values
    # rounds to the other neighbour on the GPU.  At |q~| up to ~135 (x30) one such flip
    # moves a logit by up to ss * 2^-4 * |k~_i| ~ 0.01, and in a row where two keys nearly
    # tie that moves o by up to ~0.01 more; below 2^6 (x8, x16) the effect is within the
    # stated tolerance already.
    w, T = W128K, 700
    q, k, v = _scaled_inputs(w, T, cq=cq)
    o, lse, qrot = _run_gpu(q, k, v, _table(w), window, n_sink)
    th, _, ss = _oracle_table(w)
    qb, kb, vb = to_bits(q), to_bits(k), to_bits(v)
    qr, kr = _rotated(qb, th), _rotated(kb, th)
    assert err_stats(qrot, qr)[0] <= ROT_ABS
    ro, rl = oracle.attn_rotated_f64(_f16(qr), _f16(kr), _f16(to_f64(v)), ss, True, window,
                                     n_sink)
    got = o.reshape(ro.shape)
    err = np.abs(got - ro)
    assert np.all(err <= O_MAX_ABS + flip + np.abs(ro) * 2.0 ** -8), float(err.max())
    assert err.mean() <= O_MEAN_ABS + np.abs(ro).mean() * 2.0 ** -9, float(err.mean())
    # a rotated operand the kernel computes in fp32 can land one fp16 step away from the
    # oracle's fp64 rotation rounded to fp16: a logit moves by up to 2^-11 of its size
    assert np.all(np.abs(lse.reshape(-1) - rl) <= LSE_ABS + np.abs(rl) * 2.0 ** -11)
    # against exact attention of the unrounded inputs: the logit shifts of fp16 storage
    # are the only difference, a few hundredths at most here
    ex, _, _ = oracle.attn_rows(qb, kb, vb, th, ss, True, window, n_sink)
    assert np.abs(got - ex).max() <= 0.1
    assert np.isfinite(got).all()


@pytest.mark.parametrize("cq", [0.0, 1.0 / 64])
def test_tiny_logits_and_zero_queries(cq):
    w, T = W128K, 600
    q, k, v = _scaled_inputs(w, T, cq=cq)
    o, lse, _ = _run_gpu(q, k, v, _table(w), 0, 0)
    th, _, ss = _oracle_table(w)
    ro, rl, _ = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss)
    emax, emean = err_stats(o.reshape(ro.shape), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(lse.reshape(-1), rl)[0] <= LSE_ABS
    if cq == 0.0:
        # every visible key weighs the same: the running mean of v (closed form)
        vv = to_f64(v)
        g = q.shape[1] // v.shape[1]
        means = np.cumsum(vv, axis=2) / np.arange(1, T + 1)[None, None, :, None]
        want = np.repeat(means, g, axis=1).reshape(ro.shape)
        assert np.abs(o.reshape(ro.shape) - want).max() <= O_MAX_ABS


@pytest.mark.parametrize("ck,cv,uniform", [(1.0, 60000.0, True), (3000.0, 1.0, False),
                                           (2000.0, 10000.0, False)])
def test_values_near_the_fp16_limit_keep_their_relative_precision(ck, cv, uniform):
    w, T = W128K, 520
    q, k, v = _scaled_inputs(w, T, cq=1.0 / ck, ck=ck, cv=cv, v_uniform=uniform)
    assert float(v.float().abs().max()) < 65520 and float(k.float().abs().max()) < 65520 / 1.5
    o, _, _ = _run_gpu(q, k, v, _table(w), 0, 0)
    th, _, ss = _oracle_table(w)
    ro, _, _ = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss)
    emax, emean = err_stats(o.reshape(ro.shape) / cv, ro / cv)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)


def _expect_range_error(fn):
    fn()
    with pytest.raises(api.YarnAttnError) as ei:
        api.device_status()
    assert ei.value.code == api.YR_ERANGE, str(ei.value)
    assert "fp16" in str(ei.value)


def test_out_of_range_operands_are_reported():
    w, T = synth.sweep("rope", False), 300   # plain RoPE: theta_0 = 1 rad per position
    tab = _table(w)
    q, k, v = [t.cuda() for t in _scaled_inputs(w, T)]
    ref = api.attn_prefill(q, k, v, tab)
    api.device_status()

    # the largest bf16 value below the limit passes; the next one (65536) does not
    v_edge = v.clone()
    v_edge[0, 1, 17, 5] = 65280.0
    api.attn_prefill(q, k, v_edge, tab)
    api.device_status()
    v_bad = v.clone()
    v_bad[0, 1, 17, 5] = 65536.0
    _expect_range_error(lambda: api.attn_prefill(q, k, v_bad, tab))
    v_nan = v.clone()
    v_nan[0, 0, 200, 100] = float("nan")
    _expect_range_error(lambda: api.attn_prefill(q, k, v_nan, tab))

    # (65024, 65024) fits at position 0 but rotates past the limit at position 1
    q_rot_bad = q.clone()
    q_rot_bad[0, 3, 0, 0:2] = 65024.0
    api.attn_prefill(q_rot_bad, k, v, tab)
    api.device_status()
    q_rot_bad[0, 3, 1, 0:2] = 65024.0
    _expect_range_error(lambda: api.attn_prefill(q_rot_bad, k, v, tab))
    k_rot_bad = k.clone()
    k_rot_bad[0, 0, 1, 0:2] = 65024.0
    _expect_range_error(lambda: api.attn_prefill(q, k_rot_bad, v, tab))

    # the chunk path converts the cached prefix: a value there past the limit
    P0, Tq = 256, 44
    kc, vc = torch.zeros_like(k), v.clone()
    kc[:, :, :P0] = k[:, :, :P0]
    vc[0, 1, 7, 3] = 70000.0
    _expect_range_error(lambda: api.attn_prefill_chunk(
        q[:, :, P0:P0 + Tq].contiguous(), k[:, :, P0:P0 + Tq].contiguous(),
        v[:, :, P0:P0 + Tq].contiguous(), kc, vc, P0, tab))

    # and the context stays usable: a clean call afterwards is unchanged
    again = api.attn_prefill(q, k, v, tab)
    assert api.device_status() == api.YR_OK
    assert torch.equal(again, ref)
