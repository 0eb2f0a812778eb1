"""Pins for the fp64 oracle: each check ties it to something other than itself.

The pins are closed forms, worked numbers printed on the pages
(tests/golden/*.json, each with its citation), special cases that reduce to a
library routine (torch float64 SDPA, scipy logsumexp/softmax), an independent
complex-number formulation of the rotation, invariants and brute force on tiny
inputs.  They are chosen so that a dropped term, a flipped sign, a wrong index
or a transposed operand in the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle

RNG = np.random.default_rng(1234)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def complex_rotate(x: np.ndarray, pos, theta) -> np.ndarray:
    """RoPE as complex multiplication: (x_2i + i x_2i+1) * exp(i pos theta_i)."""
    z = x[..., 0::2] + 1j * x[..., 1::2]
    pos = np.asarray(pos, dtype=np.float64)[..., None]
    w = z * np.exp(1j * pos * theta)
    out = np.empty(x.shape, dtype=np.float64)
    out[..., 0::2] = w.real
    out[..., 1::2] = w.imag
    return out


# ----------------------------------------------------------------- the table

@pytest.mark.parametrize("base,d", [(10000.0, 128), (500000.0, 128), (10000.0, 64)])
def test_rope_theta_closed_form(base, d):
    th, ms, ss = oracle.rope_theta(d, base, 4096, 1.0, "rope")
    assert th[0] == 1.0                                   # base^0
    assert th[d // 4] == pytest.approx(base ** -0.5, rel=1e-15)  # i = d/4 -> base^(-1/2)
    ratios = th[1:] / th[:-1]                             # geometric with ratio base^(-2/d)
    np.testing.assert_allclose(ratios, base ** (-2.0 / d), rtol=1e-13)
    assert ms == 1.0 and ss == pytest.approx(1.0 / math.sqrt(d), rel=1e-15)


@pytest.mark.parametrize("method", ["pi", "ntk", "yarn"])
@pytest.mark.parametrize("d,base,L", [(64, 10000.0, 64), (128, 10000.0, 4096), (128, 500000.0, 8192)])
def test_scale_one_reduces_to_rope(method, d, base, L):
    ref, _, _ = oracle.rope_theta(d, base, L, 1.0, "rope")
    th, ms, ss = oracle.rope_theta(d, base, L, 1.0, method)
    # exact in the mathematics; gamma*theta + (1-gamma)*theta rounds within an ulp or two
    np.testing.assert_allclose(th, ref, rtol=1e-15, atol=0)
    assert ms == 1.0 and ss == 1.0 / math.sqrt(d)


@pytest.mark.parametrize("s", [2.0, 4.0, 16.0])
def test_pi_divides_every_frequency(s):
    ref, _, _ = oracle.rope_theta(128, 10000.0, 4096, 1.0, "rope")
    th, ms, _ = oracle.rope_theta(128, 10000.0, 4096, s, "pi")
    np.testing.assert_allclose(th * s, ref, rtol=1e-15)
    assert ms == 1.0


def test_pi_equals_rope_at_position_over_s():
    d, s = 64, 4.0
    rope, _, _ = oracle.rope_theta(d, 10000.0, 64, 1.0, "rope")
    pi, _, _ = oracle.rope_theta(d, 10000.0, 64, s, "pi")
    x = bf16_bits(RNG.standard_normal((50, d)))
    m = RNG.integers(0, 200000, size=50).astype(np.float64)
    np.testing.assert_allclose(oracle.rotate(x, m, pi), oracle.rotate(x, m / s, rope),
                               rtol=0, atol=1e-9)


def test_ntk_base_worked_number(golden):
    g = golden("pages_worked_numbers.json")["ntk_base"]
    th, _, _ = oracle.rope_theta(g["d"], g["base"], 4096, g["s"], "ntk")
    # theta'_1 = base'^(-2/d)  =>  base' = theta'_1^(-d/2)
    base_eff = th[1] ** (-g["d"] / 2)
    assert base_eff == pytest.approx(g["printed_base"], rel=g["rel_tol"])
    assert base_eff == pytest.approx(g["base"] * g["s"] ** (g["d"] / (g["d"] - 2)), rel=1e-12)
    ref, _, _ = oracle.rope_theta(g["d"], g["base"], 4096, 1.0, "rope")
    assert th[0] == ref[0] == 1.0      # the highest frequency is kept
    assert th[-1] < ref[-1] / 7.9      # the lowest is slowed almost by s


def _bands(d, base, L, alpha, beta):
    """Band edges from the wavelength definition lambda_i = 2 pi / theta_i: dims with
    L/lambda_i > beta keep theta, dims with L/lambda_i < alpha take theta/s."""
    i = np.arange(d // 2)
    r = L * base ** (-2.0 * i / d) / (2 * math.pi)
    return i[r > beta], i[(r >= alpha) & (r <= beta)], i[r < alpha]


@pytest.mark.parametrize("d,base,L,s,expect", [
    (64, 10000.0, 64, 4.0, (0, 9, 23)),        # tiny workload: no unchanged band
    (128, 10000.0, 4096, 4.0, (21, 25, 18)),   # 16K workload: 0-20 | 21-45 | 46-63
    (128, 500000.0, 8192, 16.0, (19, 16, 29)),  # 128K workload: 0-18 | 19-34 | 35-63
])
def test_yarn_band_endpoints(golden, d, base, L, s, expect):
    g = golden("pages_worked_numbers.json")["yarn_defaults"]
    rope, _, _ = oracle.rope_theta(d, base, L, 1.0, "rope")
    th, ms, ss = oracle.rope_theta(d, base, L, s, "yarn", g["alpha"], g["beta"])
    hi, ramp, lo = _bands(d, base, L, g["alpha"], g["beta"])
    assert (len(hi), len(ramp), len(lo)) == expect
    np.testing.assert_array_equal(th[hi], rope[hi])                 # extrapolated band
    np.testing.assert_allclose(th[lo], rope[lo] / s, rtol=1e-15)    # interpolated band
    inner = ramp[1:-1]
    assert np.all(th[inner] < rope[inner]) and np.all(th[inner] > rope[inner] / s)
    # the fraction kept unscaled falls monotonically across the ramp
    frac = (th[ramp] - rope[ramp] / s) / (rope[ramp] - rope[ramp] / s)
    assert np.all(np.diff(frac) < 0)


@pytest.mark.parametrize("s,m_expect", [(4.0, 1.1386294361119890), (16.0, 1.2772588722239781),
                                        (1.0, 1.0)])
def test_yarn_temperature(golden, s, m_expect):
    g = golden("pages_worked_numbers.json")["temperature"]
    for d in (64, 128):
        _, ms, ss = oracle.rope_theta(d, 10000.0, 4096, s, "yarn")
        assert ms == pytest.approx(g["coef"] * math.log(s) + g["offset"], rel=1e-15)
        assert ms == pytest.approx(m_expect, rel=1e-15)
        assert ss == pytest.approx(ms * ms / math.sqrt(d), rel=1e-15)
    assert oracle.rope_theta(64, 10000.0, 64, 4.0, "yarn")[2] == pytest.approx(0.162060, abs=5e-7)
    assert oracle.rope_theta(128, 5e5, 8192, 16.0, "yarn")[2] == pytest.approx(0.144196, abs=5e-7)


@pytest.mark.parametrize("method", ["rope", "pi", "ntk", "yarn"])
def test_theta_strictly_decreasing(method):
    th, _, _ = oracle.rope_theta(128, 10000.0, 4096, 16.0, method)
    assert np.all(np.diff(th) < 0) and np.all(th > 0)


def test_invalid_table_arguments_rejected():
    for args in [(63, 1e4, 64, 4.0, "yarn"), (64, 1e4, 64, 0.5, "pi"), (64, 1.0, 64, 2.0, "rope")]:
        with pytest.raises(ValueError):
            oracle.rope_theta(*args)
    with pytest.raises(ValueError):
        oracle.rope_theta(64, 1e4, 64, 2.0, "yarn", 32.0, 1.0)


# --------------------------------- table variants: dynamic NTK, dimension ramp, factors

@pytest.mark.parametrize("L_cur", [1, 100, 4095, 4096])
def test_dynamic_ntk_is_rope_up_to_L_train(L_cur):
    # s = max(1, L_cur / L_train): no scaling while the sequence fits the training length
    rope, _, _ = oracle.rope_theta(128, 10000.0, 4096, 1.0, "rope")
    th, ms, _ = oracle.rope_theta(128, 10000.0, 4096, 1.0, "ntk_dynamic", L_cur=L_cur)
    np.testing.assert_array_equal(th, rope)
    assert ms == 1.0


@pytest.mark.parametrize("k", [2, 3, 8])
def test_dynamic_ntk_equals_static_ntk_at_the_ratio(golden, k):
    dyn, _, _ = oracle.rope_theta(128, 10000.0, 4096, 1.0, "ntk_dynamic", L_cur=k * 4096)
    stat, _, _ = oracle.rope_theta(128, 10000.0, 4096, float(k), "ntk")
    np.testing.assert_allclose(dyn, stat, rtol=1e-15)
    if k == 8:  # the page's worked number: base ~ 10000 * 8^(128/126) ~ 82,000
        g = golden("pages_worked_numbers.json")["ntk_base"]
        assert dyn[1] ** (-64) == pytest.approx(g["printed_base"], rel=g["rel_tol"])


@pytest.mark.parametrize("d,base,L,s,low,high", [
    (128, 10000.0, 4096, 4.0, 20, 46),    # 16K workload: r-space bands 0-20 | 21-45 | 46-63
    (128, 500000.0, 8192, 16.0, 18, 35),  # 128K workload: r-space bands 0-18 | 19-34 | 35-63
])
def test_yarn_dimension_ramp_edges_and_midpoint(golden, d, base, L, s, low, high):
    g = golden("pages_worked_numbers.json")["yarn_defaults"]
    rope, _, _ = oracle.rope_theta(d, base, L, 1.0, "rope")
    th, ms, ss = oracle.rope_theta(d, base, L, s, "yarn_dimramp", g["alpha"], g["beta"])
    # outside the ramp: the same bands as the wavelength split (pinned above)
    hi, _, lo = _bands(d, base, L, g["alpha"], g["beta"])
    assert hi.max() == low and lo.min() == high
    np.testing.assert_array_equal(th[: low + 1], rope[: low + 1])
    np.testing.assert_allclose(th[high:], rope[high:] / s, rtol=1e-15)
    # inside: linear in the index, so kept fractions of mirrored indices add up to one
    frac = (th - rope / s) / (rope - rope / s)
    for i in range(low, high + 1):
        assert frac[i] == pytest.approx((high - i) / (high - low), abs=1e-12)
        assert frac[i] + frac[low + high - i] == pytest.approx(1.0, abs=1e-12)
    # the same temperature as YaRN
    assert ms == pytest.approx(0.1 * math.log(s) + 1.0, rel=1e-15)
    assert ss == pytest.approx(ms * ms / math.sqrt(d), rel=1e-15)


def test_factor_table_reductions():
    d, base, L, s = 128, 10000.0, 4096, 8.0
    rope, _, _ = oracle.rope_theta(d, base, L, 1.0, "rope")
    pi, _, _ = oracle.rope_theta(d, base, L, s, "pi")
    yarn, _, _ = oracle.rope_theta(d, base, L, s, "yarn")
    th, ms, ss = oracle.rope_theta(d, base, L, 1.0, "factors", factors=np.ones(d // 2))
    np.testing.assert_array_equal(th, rope)
    assert ms == 1.0 and ss == pytest.approx(1 / math.sqrt(d), rel=1e-15)
    th, _, _ = oracle.rope_theta(d, base, L, 1.0, "factors", factors=np.full(d // 2, s))
    np.testing.assert_allclose(th, pi, rtol=1e-15)
    th, ms, ss = oracle.rope_theta(d, base, L, 1.0, "factors", factors=rope / yarn,
                                   attn_factor=1.2)
    np.testing.assert_allclose(th, yarn, rtol=1e-14)
    assert ms == 1.2 and ss == pytest.approx(1.44 / math.sqrt(d), rel=1e-15)


def test_table_variant_arguments_rejected():
    with pytest.raises(ValueError):
        oracle.rope_theta(64, 1e4, 64, 1.0, "ntk_dynamic", L_cur=0)
    with pytest.raises(ValueError):
        oracle.rope_theta(64, 1e4, 64, 1.0, "factors")
    for bad in (np.zeros(32), np.full(32, -1.0)):
        with pytest.raises(ValueError):
            oracle.rope_theta(64, 1e4, 64, 1.0, "factors", factors=bad)
    with pytest.raises(ValueError):
        oracle.rope_theta(64, 1e4, 64, 2.0, "yarn_dimramp", 32.0, 1.0)


# -------------------------------------------------------------- the rotation

def test_rotation_matrix_from_the_page(golden):
    g = golden("rope_unit_rotation.json")
    for c in g["cases"]:
        th = np.array([c["theta"]])
        e0 = bf16_bits(np.array([[1.0, 0.0]]))
        e1 = bf16_bits(np.array([[0.0, 1.0]]))
        np.testing.assert_allclose(oracle.rotate(e0, c["m"], th)[0], c["e0_to"], atol=1e-15)
        np.testing.assert_allclose(oracle.rotate(e1, c["m"], th)[0], c["e1_to"], atol=1e-15)


@pytest.mark.parametrize("method", ["rope", "pi", "ntk", "yarn"])
def test_rotation_matches_complex_form(method):
    th, _, _ = oracle.rope_theta(128, 500000.0, 8192, 16.0, method)
    x = bf16_bits(RNG.standard_normal((64, 128)))
    pos = RNG.integers(0, 131073, size=64).astype(np.float64)
    got = oracle.rotate(x, pos, th)
    want = complex_rotate(bits_to_f64(x), pos, th)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_rotation_identity_and_norm():
    th, _, _ = oracle.rope_theta(64, 10000.0, 64, 4.0, "yarn")
    x = bf16_bits(RNG.standard_normal((32, 64)))
    np.testing.assert_array_equal(oracle.rotate(x, 0.0, th), bits_to_f64(x))
    y = oracle.rotate(x, RNG.integers(0, 10 ** 6, size=32).astype(np.float64), th)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(bits_to_f64(x), axis=1),
                               rtol=1e-14)
    # pair norms are preserved individually: no pair mixes with another
    p_in = bits_to_f64(x).reshape(32, 32, 2)
    p_out = y.reshape(32, 32, 2)
    np.testing.assert_allclose(np.hypot(p_out[..., 0], p_out[..., 1]),
                               np.hypot(p_in[..., 0], p_in[..., 1]), rtol=1e-14)


@pytest.mark.parametrize("method", ["rope", "yarn"])
def test_relative_position_property(method):
    th, _, _ = oracle.rope_theta(128, 10000.0, 4096, 4.0, method)
    q = bf16_bits(RNG.standard_normal((20, 128)))
    k = bf16_bits(RNG.standard_normal((20, 128)))
    m = RNG.integers(0, 50000, size=20).astype(np.float64)
    n = RNG.integers(0, 50000, size=20).astype(np.float64)
    delta = RNG.integers(1, 80000, size=20).astype(np.float64)
    a = np.sum(oracle.rotate(q, m, th) * oracle.rotate(k, n, th), axis=1)
    b = np.sum(oracle.rotate(q, m + delta, th) * oracle.rotate(k, n + delta, th), axis=1)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-9)
    # and it does change with m - n
    c = np.sum(oracle.rotate(q, m + delta, th) * oracle.rotate(k, n, th), axis=1)
    assert np.max(np.abs(a - c)) > 1e-3


# ------------------------------------------------- the half-split pair layout

def complex_rotate_half(x: np.ndarray, pos, theta) -> np.ndarray:
    """Half-split RoPE as complex multiplication: (x_i + i x_{i+d/2}) * exp(i pos theta_i)."""
    h = x.shape[-1] // 2
    z = x[..., :h] + 1j * x[..., h:]
    pos = np.asarray(pos, dtype=np.float64)[..., None]
    w = z * np.exp(1j * pos * theta)
    return np.concatenate([w.real, w.imag], axis=-1)


@pytest.mark.parametrize("d", [64, 128])
def test_half_layout_matches_its_complex_form(d):
    th, _, _ = oracle.rope_theta(d, 500000.0, 8192, 16.0, "yarn")
    x = bf16_bits(RNG.standard_normal((48, d)))
    pos = RNG.integers(0, 131073, size=48).astype(np.float64)
    got = oracle.rotate(x, pos, th, pairs="half")
    np.testing.assert_allclose(got, complex_rotate_half(bits_to_f64(x), pos, th), rtol=0,
                               atol=1e-12)
    # not the interleaved rotation (the two layouts pair different elements)
    assert np.abs(got - oracle.rotate(x, pos, th)).max() > 1e-2


def test_half_layout_is_the_interleaved_rotation_of_the_permuted_vector():
    d = 128
    th, _, _ = oracle.rope_theta(d, 10000.0, 4096, 4.0, "yarn")
    x = RNG.standard_normal((16, d))
    pos = RNG.integers(0, 70000, size=16).astype(np.float64)
    perm = np.empty(d, dtype=np.int64)           # interleaved slot -> half-split element
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    inter = oracle.rotate_f64(x[:, perm], pos, th)
    half = oracle.rotate_f64(x, pos, th, pairs="half")
    np.testing.assert_allclose(half[:, perm], inter, rtol=0, atol=1e-13)


def test_half_layout_relative_position_and_norm():
    th, _, _ = oracle.rope_theta(64, 10000.0, 64, 4.0, "yarn")
    q = bf16_bits(RNG.standard_normal((20, 64)))
    k = bf16_bits(RNG.standard_normal((20, 64)))
    m = RNG.integers(0, 50000, size=20).astype(np.float64)
    n = RNG.integers(0, 50000, size=20).astype(np.float64)
    delta = RNG.integers(1, 80000, size=20).astype(np.float64)
    rq = oracle.rotate(q, m, th, pairs="half")
    a = np.sum(rq * oracle.rotate(k, n, th, pairs="half"), axis=1)
    b = np.sum(oracle.rotate(q, m + delta, th, pairs="half") *
               oracle.rotate(k, n + delta, th, pairs="half"), axis=1)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-9)
    np.testing.assert_allclose(np.linalg.norm(rq, axis=1), np.linalg.norm(bits_to_f64(q), axis=1),
                               rtol=1e-14)


# ------------------------------------------------------------- the attention

def _rand_qkv(B, Hq, Hkv, T, d):
    q = bf16_bits(RNG.standard_normal((B, Hq, T, d)))
    k = bf16_bits(RNG.standard_normal((B, Hkv, T, d)))
    v = bf16_bits(RNG.standard_normal((B, Hkv, T, d)))
    return q, k, v


def _mask(T, causal, window, n_sink):
    m = np.arange(T)[:, None]
    n = np.arange(T)[None, :]
    vis = np.ones((T, T), bool)
    if causal:
        vis &= n <= m
    if window > 0:
        vis &= ((m - n) < window) | (n < n_sink)
    return vis


@pytest.mark.parametrize("causal,window,n_sink", [(True, 0, 0), (True, 7, 0), (True, 9, 3),
                                                  (False, 0, 0)])
def test_matches_library_sdpa_float64(causal, window, n_sink):
    B, Hq, Hkv, T, d = 2, 4, 2, 37, 16
    th, _, ss = oracle.rope_theta(d, 10000.0, 16, 4.0, "yarn")
    q, k, v = _rand_qkv(B, Hq, Hkv, T, d)
    o, lse, _ = oracle.attn_rows(q, k, v, th, ss, causal, window, n_sink)
    pos = np.arange(T, dtype=np.float64)
    qr = torch.from_numpy(complex_rotate(bits_to_f64(q), pos, th))
    kr = torch.from_numpy(complex_rotate(bits_to_f64(k), pos, th))
    vv = torch.from_numpy(bits_to_f64(v))
    g = Hq // Hkv
    kr = kr.repeat_interleave(g, dim=1)
    vv = vv.repeat_interleave(g, dim=1)
    mask = torch.from_numpy(_mask(T, causal, window, n_sink))
    ref = torch.nn.functional.scaled_dot_product_attention(qr, kr, vv, attn_mask=mask, scale=ss)
    np.testing.assert_allclose(o.reshape(B, Hq, T, d), ref.numpy(), rtol=0, atol=1e-12)
    scores = torch.einsum("bhmd,bhnd->bhmn", qr, kr).numpy() * ss
    scores = np.where(mask.numpy(), scores, -np.inf)
    np.testing.assert_allclose(lse.reshape(B, Hq, T), scipy.special.logsumexp(scores, axis=-1),
                               rtol=0, atol=1e-12)


def test_rotated_f64_equals_attn_rows_on_its_own_rotation():
    B, Hq, Hkv, T, d = 2, 6, 2, 45, 16
    th, _, ss = oracle.rope_theta(d, 10000.0, 16, 4.0, "yarn")
    q, k, v = _rand_qkv(B, Hq, Hkv, T, d)
    pos = np.arange(T, dtype=np.float64)
    qr = oracle.rotate(q, np.broadcast_to(pos, (B, Hq, T)).reshape(-1), th)
    kr = oracle.rotate(k, np.broadcast_to(pos, (B, Hkv, T)).reshape(-1), th)
    for causal, w, s in [(True, 0, 0), (True, 6, 2), (False, 0, 0)]:
        o1, l1, _ = oracle.attn_rows(q, k, v, th, ss, causal, w, s)
        o2, l2 = oracle.attn_rotated_f64(qr, kr, bits_to_f64(v), ss, causal, w, s)
        np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-13)
    rows = np.array([0, 5, 44, 45 * 7 + 3, B * Hq * T - 1])
    o3, l3 = oracle.attn_rotated_f64(qr, kr, bits_to_f64(v), ss, rows=rows)
    o1, l1, _ = oracle.attn_rows(q, k, v, th, ss)
    np.testing.assert_allclose(o3, o1[rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l3, l1[rows], rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal,window,n_sink", [(True, 0, 0), (True, 5, 2), (False, 0, 0)])
def test_rotated_f64_matches_library_sdpa_on_non_bf16_values(causal, window, n_sink):
    # operands that are no bf16 (or fp16) values, large enough for a peaked softmax
    B, Hq, Hkv, T, d = 1, 4, 1, 29, 12
    q = RNG.standard_normal((B, Hq, T, d)) * 7.3
    k = RNG.standard_normal((B, Hkv, T, d)) * 1.1
    v = RNG.standard_normal((B, Hkv, T, d)) * 3e4
    ss = 0.1442
    o, lse = oracle.attn_rotated_f64(q, k, v, ss, causal, window, n_sink)
    mask = torch.from_numpy(_mask(T, causal, window, n_sink))
    kt = torch.from_numpy(k).repeat_interleave(Hq, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(Hq, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), kt, vt,
                                                           attn_mask=mask, scale=ss)
    np.testing.assert_allclose(o.reshape(B, Hq, T, d), ref.numpy(), rtol=1e-12, atol=1e-8)
    scores = np.einsum("bhmd,bhnd->bhmn", q, kt.numpy()) * ss
    scores = np.where(mask.numpy(), scores, -np.inf)
    np.testing.assert_allclose(lse.reshape(B, Hq, T), scipy.special.logsumexp(scores, axis=-1),
                               rtol=0, atol=1e-10)


def test_rotated_f64_zero_query_gives_prefix_means():
    T, d = 120, 3
    k = RNG.standard_normal((1, 1, T, d))
    v = RNG.standard_normal((1, 1, T, d))
    cs = np.vstack([np.zeros((1, d)), np.cumsum(v[0, 0], axis=0)])
    o, _ = oracle.attn_rotated_f64(np.zeros((1, 1, T, d)), k, v, 0.3, True, 0, 0)
    np.testing.assert_allclose(o, cs[1:] / np.arange(1, T + 1)[:, None], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,window,n_sink", [(True, 0, 0), (True, 9, 3)])
def test_half_layout_attention_matches_library_sdpa(causal, window, n_sink):
    B, Hq, Hkv, T, d = 1, 4, 2, 41, 16
    th, _, ss = oracle.rope_theta(d, 10000.0, 16, 4.0, "yarn")
    q, k, v = _rand_qkv(B, Hq, Hkv, T, d)
    o, lse, qr_o = oracle.attn_rows(q, k, v, th, ss, causal, window, n_sink, want_qrot=True,
                                    pairs="half")
    pos = np.arange(T, dtype=np.float64)
    qr = torch.from_numpy(complex_rotate_half(bits_to_f64(q), pos, th))
    kr = torch.from_numpy(complex_rotate_half(bits_to_f64(k), pos, th))
    np.testing.assert_allclose(qr_o.reshape(B, Hq, T, d), qr.numpy(), rtol=0, atol=1e-12)
    g = Hq // Hkv
    mask = torch.from_numpy(_mask(T, causal, window, n_sink))
    ref = torch.nn.functional.scaled_dot_product_attention(
        qr, kr.repeat_interleave(g, dim=1), torch.from_numpy(bits_to_f64(v)).repeat_interleave(g, dim=1),
        attn_mask=mask, scale=ss)
    np.testing.assert_allclose(o.reshape(B, Hq, T, d), ref.numpy(), rtol=0, atol=1e-12)


def test_half_layout_decode_and_chunk_equal_the_prefill_rows():
    B, Hq, Hkv, T, d = 1, 4, 2, 50, 16
    th, _, ss = oracle.rope_theta(d, 10000.0, 16, 4.0, "yarn")
    q, k, v = _rand_qkv(B, Hq, Hkv, T, d)
    o, _, _ = oracle.attn_rows(q, k, v, th, ss, pairs="half")
    o = o.reshape(B, Hq, T, d)
    # a cache holding the half-split rotation of keys 0..L-1, then the token at L
    pos = np.broadcast_to(np.arange(T, dtype=np.float64), (B, Hkv, T)).reshape(-1)
    kc = bf16_bits(oracle.rotate(k, pos, th, pairs="half").reshape(B, Hkv, T, d))
    L = 37
    od, _, _, _ = oracle.decode(q[:, :, L], k[:, :, L], v[:, :, L], kc, v, np.array([L]), th, ss,
                                pairs="half")
    # brute force: the query and the new key rotated at L in the half layout (complex form),
    # the cached keys as given
    g = Hq // Hkv
    for h in range(Hq):
        qv = complex_rotate_half(bits_to_f64(q[0, h, L]), L, th)
        keys = np.vstack([bits_to_f64(kc[0, h // g, :L]),
                          complex_rotate_half(bits_to_f64(k[0, h // g, L]), L, th)[None]])
        sc = ss * keys @ qv
        p_ = np.exp(sc - sc.max())
        want = (p_ / p_.sum()) @ bits_to_f64(v[0, h // g, :L + 1])
        np.testing.assert_allclose(od[0, h], want, rtol=0, atol=1e-12)
    # and close to the exact prefill row (the cached keys went through bf16)
    np.testing.assert_allclose(od, o[:, :, L], rtol=0, atol=5e-2)
    oc, _, kr = oracle.prefill_chunk(q[:, :, L:], k[:, :, L:], v[:, :, L:], kc, v, L, th, ss,
                                     pairs="half")
    np.testing.assert_allclose(oc[:, :, 0], od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(kr.reshape(-1, d),
                               oracle.rotate(k[:, :, L:], pos.reshape(B, Hkv, T)[:, :, L:].reshape(-1),
                                             th, pairs="half").reshape(-1, d), rtol=0, atol=1e-13)


def test_rows_sum_to_one_through_v_ones():
    B, Hq, Hkv, T, d = 1, 4, 2, 64, 8
    th, _, ss = oracle.rope_theta(d, 10000.0, 16, 4.0, "yarn")
    q, k, _ = _rand_qkv(B, Hq, Hkv, T, d)
    ones = bf16_bits(np.ones((B, Hkv, T, d)))
    for causal, w, s in [(True, 0, 0), (True, 5, 2), (False, 0, 0)]:
        o, _, _ = oracle.attn_rows(q, k, ones, th, ss, causal, w, s)
        np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)


def test_single_token_returns_v0():
    th, _, ss = oracle.rope_theta(16, 10000.0, 16, 4.0, "yarn")
    q, k, v = _rand_qkv(1, 2, 1, 1, 16)
    o, lse, _ = oracle.attn_rows(q, k, v, th, ss)
    np.testing.assert_array_equal(o.reshape(2, 16), np.repeat(bits_to_f64(v).reshape(1, 16), 2, 0))
    qr = oracle.rotate(q.reshape(2, 16), 0.0, th)
    kr = oracle.rotate(k.reshape(1, 16), 0.0, th)
    np.testing.assert_allclose(lse, ss * (qr @ kr[0]), rtol=1e-14)


def test_zero_query_gives_prefix_means():
    # q = 0 makes every visible key equally weighted: O_m is the mean of v over visible keys,
    # i.e. a running mean (causal) or a windowed running mean.
    T, d = 300, 4
    th, _, ss = oracle.rope_theta(d, 10000.0, 16, 4.0, "yarn")
    q = bf16_bits(np.zeros((1, 1, T, d)))
    k = bf16_bits(RNG.standard_normal((1, 1, T, d)))
    vf = RNG.standard_normal((1, 1, T, d))
    v = bf16_bits(vf)
    vd = bits_to_f64(v)[0, 0]
    cs = np.vstack([np.zeros((1, d)), np.cumsum(vd, axis=0)])
    o, _, _ = oracle.attn_rows(q, k, v, th, ss, True, 0, 0)
    np.testing.assert_allclose(o, cs[1:] / np.arange(1, T + 1)[:, None], rtol=0, atol=1e-12)
    W = 50
    o, _, _ = oracle.attn_rows(q, k, v, th, ss, True, W, 0)
    lo = np.maximum(np.arange(T) - W + 1, 0)
    want = (cs[np.arange(T) + 1] - cs[lo]) / (np.arange(T) + 1 - lo)[:, None]
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-12)


def test_sink_window_effective_context_from_the_page(golden):
    g = golden("pages_worked_numbers.json")["sink_window"]
    W, S = g["window"], g["n_sink"]
    T, d = W + S + 100, 2
    th, _, ss = oracle.rope_theta(d, 10000.0, 16, 4.0, "yarn")
    q = bf16_bits(np.zeros((1, 1, T, d)))
    k = bf16_bits(RNG.standard_normal((1, 1, T, d)))
    vf = np.zeros((1, 1, T, d))
    vf[0, 0, :S, 0] = 1.0     # marks the sink tokens
    vf[0, 0, :, 1] = 1.0      # every token
    v = bf16_bits(vf)
    rows = np.arange(W + S, T, dtype=np.int64)  # far enough that no sink is inside the window
    o, _, _ = oracle.attn_rows(q, k, v, th, ss, True, W, S, rows=rows)
    # uniform weights over "4 + last 4096" keys: the sink share is 4 / 4100
    np.testing.assert_allclose(o[:, 0], S / g["effective_context"], rtol=1e-13)
    np.testing.assert_allclose(o[:, 1], 1.0, rtol=1e-13)


def test_window_at_least_T_is_dense():
    th, _, ss = oracle.rope_theta(16, 10000.0, 16, 4.0, "yarn")
    q, k, v = _rand_qkv(1, 2, 1, 40, 16)
    dense, _, _ = oracle.attn_rows(q, k, v, th, ss, True, 0, 0)
    for w, s in [(40, 0), (41, 3), (1000, 5)]:
        win, _, _ = oracle.attn_rows(q, k, v, th, ss, True, w, s)
        np.testing.assert_array_equal(win, dense)


def test_gqa_mapping_contiguous_groups():
    B, Hq, Hkv, T, d = 1, 8, 2, 12, 4
    th, _, ss = oracle.rope_theta(d, 10000.0, 16, 4.0, "yarn")
    q, k, _ = _rand_qkv(B, Hq, Hkv, T, d)
    vf = np.zeros((B, Hkv, T, d))
    for j in range(Hkv):
        vf[:, j] = j + 1.0
    o, _, _ = oracle.attn_rows(q, k, bf16_bits(vf), th, ss)
    o = o.reshape(B, Hq, T, d)
    for h in range(Hq):
        np.testing.assert_allclose(o[0, h], h // (Hq // Hkv) + 1.0, rtol=1e-14)


def test_sampled_rows_equal_full_rows():
    th, _, ss = oracle.rope_theta(16, 10000.0, 16, 4.0, "yarn")
    q, k, v = _rand_qkv(2, 4, 2, 50, 16)
    full, lse_full, _ = oracle.attn_rows(q, k, v, th, ss, True, 9, 2)
    rows = np.array([0, 7, 49, 50, 123, 399], dtype=np.int64)
    part, lse_part, qr = oracle.attn_rows(q, k, v, th, ss, True, 9, 2, rows=rows, want_qrot=True)
    np.testing.assert_array_equal(part, full[rows])
    np.testing.assert_array_equal(lse_part, lse_full[rows])
    pos = (rows % 50).astype(np.float64)
    np.testing.assert_allclose(qr, oracle.rotate(q.reshape(-1, 16)[rows], pos, th), atol=0)


# ------------------------------------------------------------------------- ALiBi

@pytest.mark.parametrize("H", [1, 4, 8, 12, 32])
def test_alibi_slopes_geometric_series(H):
    # the page's series: 2^(-8/H), 2^(-16/H), ... one term per head
    m = oracle.alibi_slopes(H)
    assert m[0] == pytest.approx(2.0 ** (-8.0 / H), rel=1e-15)
    np.testing.assert_allclose(m[1:] / m[:-1], 2.0 ** (-8.0 / H), rtol=1e-14)
    assert m[-1] == pytest.approx(2.0 ** -8, rel=1e-15)


@pytest.mark.parametrize("window,n_sink", [(0, 0), (6, 2)])
def test_alibi_against_library_sdpa_with_bias(window, n_sink):
    B, Hq, Hkv, T, d = 1, 4, 2, 19, 16
    ss = 1.0 / math.sqrt(d)
    theta = np.zeros(d // 2)  # ALiBi rotates nothing
    q = bf16_bits(RNG.standard_normal((B, Hq, T, d)))
    k = bf16_bits(RNG.standard_normal((B, Hkv, T, d)))
    v = bf16_bits(RNG.standard_normal((B, Hkv, T, d)))
    slopes = oracle.alibi_slopes(Hq)
    o, lse, _ = oracle.attn_rows(q, k, v, theta, ss, True, window, n_sink, slopes=slopes)
    o = o.reshape(B, Hq, T, d)
    mpos = np.arange(T)[:, None]
    npos = np.arange(T)[None, :]
    vis = npos <= mpos
    if window:
        vis = vis & (((mpos - npos) < window) | (npos < n_sink))
    for h in range(Hq):
        bias = np.where(vis, -slopes[h] * (mpos - npos), -np.inf)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(bits_to_f64(q[0, h]))[None],
            torch.from_numpy(bits_to_f64(k[0, h // 2]))[None],
            torch.from_numpy(bits_to_f64(v[0, h // 2]))[None],
            attn_mask=torch.from_numpy(bias)[None], scale=ss)[0].numpy()
        np.testing.assert_allclose(o[0, h], ref, atol=1e-12)


def test_alibi_zero_slopes_and_cross_function_identities():
    B, Hq, Hkv, T, d = 1, 2, 1, 12, 8
    ss = 1.0 / math.sqrt(d)
    theta = np.zeros(d // 2)
    q = bf16_bits(RNG.standard_normal((B, Hq, T, d)))
    k = bf16_bits(RNG.standard_normal((B, Hkv, T, d)))
    v = bf16_bits(RNG.standard_normal((B, Hkv, T, d)))
    plain, _, _ = oracle.attn_rows(q, k, v, theta, ss)
    zero, _, _ = oracle.attn_rows(q, k, v, theta, ss, slopes=np.zeros(Hq))
    np.testing.assert_array_equal(plain, zero)
    # with no rotation the cache holds the raw keys: the last rows of a prefill equal a
    # chunk over the same keys at the same positions, and its last row equals decode
    slopes = oracle.alibi_slopes(Hq)
    full, fl, _ = oracle.attn_rows(q, k, v, theta, ss, slopes=slopes)
    P0 = 5
    kc = np.zeros((B, Hkv, T, d), np.uint16)
    vc = np.zeros((B, Hkv, T, d), np.uint16)
    kc[:, :, :P0], vc[:, :, :P0] = k[:, :, :P0], v[:, :, :P0]
    ch, cl, _ = oracle.prefill_chunk(q[:, :, P0:], k[:, :, P0:], v[:, :, P0:], kc, vc, P0, theta,
                                     ss, slopes=slopes)
    np.testing.assert_allclose(ch, full.reshape(B, Hq, T, d)[:, :, P0:], rtol=1e-13, atol=1e-15)
    # and decode of the last token equals the last prefill row
    od, ld, _, _ = oracle.decode(q[:, :, T - 1], k[:, :, T - 1], v[:, :, T - 1], kc * 0 + k,
                                 vc * 0 + v, np.array([T - 1], np.int32), theta, ss,
                                 slopes=slopes)
    np.testing.assert_allclose(od, full.reshape(B, Hq, T, d)[:, :, T - 1], rtol=1e-13,
                               atol=1e-15)


# ----------------------------------------------------------------- the decode

@pytest.mark.parametrize("window,n_sink", [(0, 0), (6, 0), (6, 2)])
def test_decode_brute_force(window, n_sink):
    B, Hq, Hkv, d, T_max = 3, 4, 2, 16, 30
    th, _, ss = oracle.rope_theta(d, 500000.0, 8, 16.0, "yarn")
    qn = bf16_bits(RNG.standard_normal((B, Hq, d)))
    kn = bf16_bits(RNG.standard_normal((B, Hkv, d)))
    vn = bf16_bits(RNG.standard_normal((B, Hkv, d)))
    kc = bf16_bits(RNG.standard_normal((B, Hkv, T_max, d)))
    vc = bf16_bits(RNG.standard_normal((B, Hkv, T_max, d)))
    L = np.array([0, 13, 29], dtype=np.int32)
    o, lse, kr, qr = oracle.decode(qn, kn, vn, kc, vc, L, th, ss, window, n_sink)
    g = Hq // Hkv
    for b in range(B):
        qrot = complex_rotate(bits_to_f64(qn[b]), float(L[b]), th)
        krot = complex_rotate(bits_to_f64(kn[b]), float(L[b]), th)
        np.testing.assert_allclose(qr[b], qrot, atol=1e-12)
        np.testing.assert_allclose(kr[b], krot, atol=1e-12)
        for h in range(Hq):
            j = h // g
            keys = np.vstack([bits_to_f64(kc[b, j, :L[b]]), krot[j][None]])
            vals = np.vstack([bits_to_f64(vc[b, j, :L[b]]), bits_to_f64(vn[b, j])[None]])
            n = np.arange(L[b] + 1)
            vis = np.ones(L[b] + 1, bool) if window == 0 else ((L[b] - n) < window) | (n < n_sink)
            sc = np.where(vis, ss * keys @ qrot[h], -np.inf)
            np.testing.assert_allclose(o[b, h], scipy.special.softmax(sc) @ vals, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], scipy.special.logsumexp(sc), atol=1e-12)


# ------------------------------------------------- chunked prefill on a cache prefix

def _chunk_inputs(B, Hq, Hkv, Tq, d, T_max):
    q = bf16_bits(RNG.standard_normal((B, Hq, Tq, d)))
    kn = bf16_bits(RNG.standard_normal((B, Hkv, Tq, d)))
    vn = bf16_bits(RNG.standard_normal((B, Hkv, Tq, d)))
    kc = bf16_bits(RNG.standard_normal((B, Hkv, T_max, d)))
    vc = bf16_bits(RNG.standard_normal((B, Hkv, T_max, d)))
    return q, kn, vn, kc, vc


@pytest.mark.parametrize("window,n_sink", [(0, 0), (7, 0), (7, 3)])
def test_chunk_brute_force_against_library_softmax(window, n_sink):
    B, Hq, Hkv, Tq, d, P0, T_max = 2, 4, 2, 9, 16, 11, 24
    th, _, ss = oracle.rope_theta(d, 10000.0, 8, 4.0, "yarn")
    q, kn, vn, kc, vc = _chunk_inputs(B, Hq, Hkv, Tq, d, T_max)
    o, lse, kr = oracle.prefill_chunk(q, kn, vn, kc, vc, P0, th, ss, window, n_sink)
    g = Hq // Hkv
    for b in range(B):
        for j in range(Hkv):
            krot = complex_rotate(bits_to_f64(kn[b, j]), np.arange(P0, P0 + Tq, dtype=float), th)
            np.testing.assert_allclose(kr[b, j], krot, atol=1e-12)
            keys = torch.from_numpy(np.vstack([bits_to_f64(kc[b, j, :P0]), krot]))
            vals = torch.from_numpy(np.vstack([bits_to_f64(vc[b, j, :P0]), bits_to_f64(vn[b, j])]))
            for h in range(j * g, (j + 1) * g):
                qrot = complex_rotate(bits_to_f64(q[b, h]), np.arange(P0, P0 + Tq, dtype=float), th)
                m = np.arange(P0, P0 + Tq)[:, None]
                n = np.arange(P0 + Tq)[None, :]
                vis = n <= m
                if window:
                    vis = vis & (((m - n) < window) | (n < n_sink))
                ref = torch.nn.functional.scaled_dot_product_attention(
                    torch.from_numpy(qrot)[None], keys[None], vals[None],
                    attn_mask=torch.from_numpy(vis)[None], scale=ss)[0].numpy()
                np.testing.assert_allclose(o[b, h], ref, atol=1e-12)
                sc = np.where(vis, ss * qrot @ keys.numpy().T, -np.inf)
                np.testing.assert_allclose(lse[b, h], scipy.special.logsumexp(sc, axis=1), atol=1e-12)


def test_chunk_of_one_token_is_decode():
    B, Hq, Hkv, d, T_max, P0 = 2, 8, 2, 32, 40, 17
    th, _, ss = oracle.rope_theta(d, 500000.0, 16, 16.0, "yarn")
    q, kn, vn, kc, vc = _chunk_inputs(B, Hq, Hkv, 1, d, T_max)
    o, lse, kr = oracle.prefill_chunk(q, kn, vn, kc, vc, P0, th, ss, 9, 2)
    od, lsed, krd, _ = oracle.decode(q[:, :, 0], kn[:, :, 0], vn[:, :, 0], kc, vc,
                                     np.full(B, P0, np.int32), th, ss, 9, 2)
    np.testing.assert_allclose(o[:, :, 0], od, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse[:, :, 0], lsed, rtol=1e-14)
    np.testing.assert_allclose(kr[:, :, 0], krd, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("window,n_sink", [(0, 0), (5, 2)])
def test_chunk_at_position_zero_is_full_prefill(window, n_sink):
    B, Hq, Hkv, Tq, d = 1, 4, 1, 21, 16
    th, _, ss = oracle.rope_theta(d, 10000.0, 16, 2.0, "ntk")
    q, kn, vn, kc, vc = _chunk_inputs(B, Hq, Hkv, Tq, d, Tq)
    o, lse, _ = oracle.prefill_chunk(q, kn, vn, kc, vc, 0, th, ss, window, n_sink)
    ro, rl, _ = oracle.attn_rows(q, kn, vn, th, ss, True, window, n_sink)
    np.testing.assert_allclose(o.reshape(ro.shape), ro, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse.reshape(-1), rl, rtol=1e-14)


def test_chunk_rejects_overflowing_cache():
    th, _, ss = oracle.rope_theta(8, 10000.0, 8, 1.0, "rope")
    q, kn, vn, kc, vc = _chunk_inputs(1, 1, 1, 4, 8, 10)
    with pytest.raises(ValueError):
        oracle.prefill_chunk(q, kn, vn, kc, vc, 7, th, ss)


def test_decode_rejects_full_cache():
    d = 8
    th, _, ss = oracle.rope_theta(d, 10000.0, 8, 2.0, "yarn")
    z = bf16_bits(np.zeros((1, 1, d)))
    c = bf16_bits(np.zeros((1, 1, 4, d)))
    with pytest.raises(ValueError):
        oracle.decode(z, z, z, c, c, np.array([4], np.int32), th, ss)


# --------------------------------------------------------- KV-cache formula

def test_kv_cache_bytes_worked_numbers(golden):
    for row in golden("pages_worked_numbers.json")["kv_cache"]:
        got = oracle.kv_cache_bytes(row["n_layers"], row["n_kv_heads"], row["head_dim"],
                                    row["seq_len"], row["batch"], row["dtype_bytes"])
        if "printed_gb" in row:
            assert got / 1e9 == pytest.approx(row["printed_gb"], rel=row["rel_tol"])
        else:
            assert got / 2 ** 30 == pytest.approx(row["printed_gib"], rel=row["rel_tol"])


@pytest.mark.parametrize("i0", [5, 20, 40])
@pytest.mark.parametrize("f", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_yarn_ramp_interior_at_constructed_points(i0, f):
    # Inside YaRN's ramp the reading is linear in r = L_train / lambda_i.  Choose the base
    # so that pair i0 sits at r = alpha + f (beta - alpha): its frequency must then be the
    # plain mix f theta + (1 - f) theta / s.  A ramp in log r or in the pair index, a
    # swapped mix, or swapped band edges all miss these values.
    d, L, s, alpha, beta = 128, 4096, 16.0, 1.0, 32.0
    r = alpha + f * (beta - alpha)
    base = (L / (2.0 * math.pi * r)) ** (d / (2.0 * i0))
    th, _, _ = oracle.rope_theta(d, base, L, s, "yarn", alpha, beta)
    rope, _, _ = oracle.rope_theta(d, base, L, 1.0, "rope")
    assert rope[i0] * L / (2.0 * math.pi) == pytest.approx(r, rel=1e-12)
    assert th[i0] / rope[i0] == pytest.approx(f + (1.0 - f) / s, rel=1e-12)
