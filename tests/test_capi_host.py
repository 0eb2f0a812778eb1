"""C-ABI checks that need no GPU: the library loads, exports every declared entry
point, builds the same table as the oracle, and rejects bad arguments on the host
before touching a device."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle
from yarn_position_scaling_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.load()


def test_library_exports_every_declared_symbol(lib):
    with open(os.path.join(ROOT, "include", "yarnattn.h")) as f:
        header = f.read()
    declared = set(re.findall(r"^\w[\w\s\*]*?\b(yr_\w+)\s*\(", header, flags=re.M))
    assert declared == set(api.SYMBOLS)
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in yarnattn.h but not exported"
    assert lib.yr_version() == 10000


def test_error_codes_match_the_header():
    with open(os.path.join(ROOT, "include", "yarnattn.h")) as f:
        header = f.read()
    codes = dict(re.findall(r"^#define (YR_E\w+|YR_OK) \(?(-?\d+)\)?", header, flags=re.M))
    assert set(codes) == {"YR_OK", "YR_EINVAL", "YR_EUNSUPPORTED", "YR_ECUDA", "YR_ETIMEOUT",
                          "YR_ERANGE"}
    for name, value in codes.items():
        assert getattr(api, name) == int(value), name


@pytest.mark.parametrize("method", ["rope", "pi", "ntk", "yarn"])
@pytest.mark.parametrize("d,base,L,s", [(64, 10000.0, 64, 4.0), (128, 10000.0, 4096, 4.0),
                                        (128, 500000.0, 8192, 16.0), (128, 10000.0, 4096, 1.0)])
def test_table_matches_oracle(lib, method, d, base, L, s):
    t = api.rope_freq_table(d, base, L, s, method)
    th, ms, ss = oracle.rope_theta(d, base, L, s, method)
    got = np.array(t.inv_freq[: d // 2])
    np.testing.assert_allclose(got, th, rtol=4e-15, atol=0)
    np.testing.assert_allclose(np.array(t.turns[: d // 2]), th / (2 * math.pi), rtol=4e-15)
    assert t.mscale == pytest.approx(ms, rel=1e-15)
    assert t.softmax_scale == pytest.approx(ss, rel=1e-15)
    assert t.head_dim == d and t.method == api.METHODS[method]


@pytest.mark.parametrize("method,kw", [
    ("ntk_dynamic", {"L_cur": 1}), ("ntk_dynamic", {"L_cur": 4096}), ("ntk_dynamic", {"L_cur": 131072}),
    ("yarn_dimramp", {}),
    ("factors", {"factors": np.geomspace(1.0, 16.0, 64)}),
    ("factors", {"factors": np.linspace(1.0, 4.0, 64), "attn_factor": 1.3}),
])
@pytest.mark.parametrize("base,L,s", [(10000.0, 4096, 4.0), (500000.0, 8192, 16.0)])
def test_table_variants_match_oracle(lib, method, kw, base, L, s):
    t = api.rope_freq_table(128, base, L, s, method, **kw)
    th, ms, ss = oracle.rope_theta(128, base, L, s, method, **kw)
    np.testing.assert_allclose(np.array(t.inv_freq[:64]), th, rtol=4e-15, atol=0)
    np.testing.assert_allclose(np.array(t.turns[:64]), th / (2 * math.pi), rtol=4e-15)
    assert t.mscale == pytest.approx(ms, rel=1e-15)
    assert t.softmax_scale == pytest.approx(ss, rel=1e-15)
    assert t.method == api.METHODS[method]


def test_alibi_table_rotates_nothing(lib):
    t = api.rope_freq_table(128, 1e4, 4096, 1.0, "alibi")
    assert all(x == 0.0 for x in t.inv_freq[:64]) and all(x == 0.0 for x in t.turns[:64])
    assert t.mscale == 1.0 and t.softmax_scale == pytest.approx(1 / math.sqrt(128), rel=1e-15)
    assert t.method == api.ALIBI


def test_table_variant_digests(lib):
    dyn = [api.rope_freq_table(128, 1e4, 4096, 1.0, "ntk_dynamic", L_cur=L).digest
           for L in (4096, 8192, 8192)]
    assert dyn[1] == dyn[2] and dyn[0] != dyn[1]
    f = np.linspace(1.0, 4.0, 64)
    a = api.rope_freq_table(128, 1e4, 4096, 1.0, "factors", factors=f).digest
    b = api.rope_freq_table(128, 1e4, 4096, 1.0, "factors", factors=f * 1.0001).digest
    c = api.rope_freq_table(128, 1e4, 4096, 1.0, "factors", factors=f, attn_factor=1.2).digest
    assert len({a, b, c}) == 3


@pytest.mark.parametrize("method,kw", [
    ("ntk_dynamic", {"L_cur": 0}), ("factors", {}), ("factors", {"factors": np.zeros(64)}),
    ("factors", {"factors": np.full(64, np.inf)}), ("yarn_dimramp", {"alpha": 32.0, "beta": 1.0}),
])
def test_table_variant_arguments_rejected(lib, method, kw):
    with pytest.raises(RuntimeError):
        api.rope_freq_table(128, 1e4, 4096, 2.0, method, **kw)


def test_table_digest_identifies_the_position_policy(lib):
    a = api.rope_freq_table(128, 10000.0, 4096, 4.0, "yarn")
    b = api.rope_freq_table(128, 10000.0, 4096, 4.0, "yarn")
    c = api.rope_freq_table(128, 10000.0, 4096, 8.0, "yarn")
    d = api.rope_freq_table(128, 10000.0, 4096, 4.0, "pi")
    e = api.rope_freq_table(128, 10000.0, 8192, 4.0, "pi")  # L_train does not shape PI
    assert a.digest == b.digest
    assert len({a.digest, c.digest, d.digest}) == 3
    assert d.digest == e.digest


@pytest.mark.parametrize("args", [
    (63, 1e4, 64, 4.0, "yarn"), (130, 1e4, 64, 4.0, "rope"), (64, 1.0, 64, 2.0, "rope"),
    (64, 1e4, 64, 0.5, "pi"), (64, 1e4, 0, 2.0, "yarn"), (64, 1e4, 64, float("nan"), "ntk")])
def test_table_rejects_bad_parameters(lib, args):
    with pytest.raises(api.YarnAttnError) as ei:
        api.rope_freq_table(*args)
    assert ei.value.code == api.YR_EINVAL


def test_table_rejects_reversed_ramp(lib):
    with pytest.raises(api.YarnAttnError):
        api.rope_freq_table(64, 1e4, 64, 2.0, "yarn", alpha=32.0, beta=1.0)


# Host-side validation happens before any CUDA call, so fake (never dereferenced)
# pointers are enough to exercise it on a machine without a GPU.
FAKE = ctypes.c_void_p(1 << 20)
NUL = ctypes.c_void_p(0)


def _prefill(lib, tab, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=NUL, kc=NUL, qd=NUL, kd=NUL, B=1, Hq=4, Hkv=2,
             T=256, d=64, causal=1, window=0, n_sink=0, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    null_strides = ctypes.POINTER(ctypes.c_int64)()
    return lib.yr_attn_prefill(a["q"], a["k"], a["v"], a["o"], a["lse"], a["kc"], a["qd"], a["kd"],
                               a["B"], a["Hq"], a["Hkv"], a["T"], a["d"], a.get("qs", null_strides),
                               null_strides, null_strides, null_strides, null_strides,
                               ctypes.byref(tab), a["causal"], a["window"], a["n_sink"], a["ws"],
                               a["ws_bytes"], NUL)


@pytest.mark.parametrize("kw,code", [
    (dict(q=NUL), api.YR_EINVAL), (dict(Hq=3), api.YR_EINVAL), (dict(T=0), api.YR_EINVAL),
    (dict(d=96), api.YR_EUNSUPPORTED), (dict(d=128), api.YR_EINVAL),  # table is d=64
    (dict(causal=0, window=16), api.YR_EINVAL), (dict(n_sink=4), api.YR_EINVAL),
    (dict(window=-1), api.YR_EINVAL), (dict(causal=2), api.YR_EINVAL),
    (dict(ws_bytes=100), api.YR_EINVAL), (dict(ws=ctypes.c_void_p((1 << 20) + 16)), api.YR_EINVAL),
    (dict(q=ctypes.c_void_p((1 << 20) + 2)), api.YR_EINVAL),
    (dict(qs=(ctypes.c_int64 * 3)(4096, 1024, 12)), api.YR_EINVAL),
])
def test_prefill_rejects_bad_arguments_on_host(lib, kw, code):
    tab = api.rope_freq_table(64, 10000.0, 64, 4.0, "yarn")
    rc = _prefill(lib, tab, **kw)
    assert rc == code
    assert lib.yr_last_error().decode().startswith("yr_attn_prefill")


def _decode(lib, tab, **kw):
    a = dict(qn=FAKE, kn=FAKE, vn=FAKE, kc=FAKE, vc=FAKE, cl=FAKE, o=FAKE, B=2, Hq=8, Hkv=2,
             d=64, T_max=4096, window=0, n_sink=0, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    return lib.yr_attn_decode(a["qn"], a["kn"], a["vn"], a["kc"], a["vc"], a["cl"], a["o"], NUL,
                              NUL, a["B"], a["Hq"], a["Hkv"], a["d"], a["T_max"], ctypes.byref(tab),
                              a["window"], a["n_sink"], a["ws"], a["ws_bytes"], NUL)


@pytest.mark.parametrize("kw,code", [
    (dict(cl=NUL), api.YR_EINVAL), (dict(Hq=7), api.YR_EINVAL), (dict(T_max=0), api.YR_EINVAL),
    (dict(d=80), api.YR_EUNSUPPORTED), (dict(Hq=68, Hkv=2), api.YR_EUNSUPPORTED),
    (dict(n_sink=2), api.YR_EINVAL), (dict(ws_bytes=8), api.YR_EINVAL),
])
def test_decode_rejects_bad_arguments_on_host(lib, kw, code):
    tab = api.rope_freq_table(64, 10000.0, 64, 4.0, "yarn")
    assert _decode(lib, tab, **kw) == code
    assert lib.yr_last_error().decode().startswith("yr_attn_decode")


def test_workspace_sizes(lib):
    # rotated keys and values in fp16
    assert api.attn_prefill_workspace_bytes(1, 8, 131072, 128) == 2 * 8 * 131072 * 128 * 2
    # the chunk's split-KV workspace: up to 16 shares of fp32 o and lse
    assert api.attn_prefill_chunk_split_bytes(1, 32, 256, 128) == 16 * 32 * 256 * 129 * 4
    # one partial slot per block of the balanced split that can hold part of a segment:
    # blocks hold at least 2048 keys, so a segment of T_max keys touches ceil(T_max/2048)+1
    parts = (131073 + 2047) // 2048 + 1
    assert api.attn_decode_workspace_bytes(8, 32, 8, 128, 131073) == 8 * 8 * parts * 4 * 130 * 4
    assert api.attn_decode_workspace_bytes(8, 30, 8, 128, 100) == 0


def test_table_rejects_unknown_pair_layout(lib):
    with pytest.raises(api.YarnAttnError):
        api.rope_freq_table(128, 1e4, 4096, 4.0, "yarn", pairs=2)
    t_int = api.rope_freq_table(128, 1e4, 4096, 4.0, "yarn")
    t_half = api.rope_freq_table(128, 1e4, 4096, 4.0, "yarn", pairs="half")
    assert t_int.digest != t_half.digest
    assert list(t_int.inv_freq) == list(t_half.inv_freq)


def test_host_prefill_plan_checks_arguments_before_any_cuda_call(lib):
    # sizes: q and o [B,Hq,T,d], k and v [B,Hkv,T,d] bf16, each rounded up to 256 bytes,
    # plus one unit's prefill workspace (rotated keys and values of its KV heads, fp16)
    B, Hq, Hkv, T, d = 2, 4, 2, 16, 64
    r = lambda x: (x + 255) // 256 * 256  # noqa: E731
    want = 2 * r(B * Hq * T * d * 2) + 2 * r(B * Hkv * T * d * 2) + r(4 * 1 * T * d)
    assert lib.yr_host_prefill_workspace_bytes(B, Hq, Hkv, T, d, 2) == want  # 1 KV head a unit
    assert lib.yr_host_prefill_workspace_bytes(1, 3, 2, 16, 64, 0) == 0      # Hq % Hkv
    assert lib.yr_host_prefill_workspace_bytes(1, 4, 2, 16, 96, 0) == 0      # head size
    plan = ctypes.c_void_p()
    n = want
    assert lib.yr_host_prefill_create(ctypes.byref(plan), B, Hq, Hkv, T, d, 2, None, n) == \
        api.YR_EINVAL
    assert lib.yr_host_prefill_create(ctypes.byref(plan), B, Hq, Hkv, T, d, 2,
                                      ctypes.c_void_p(4096), n - 1) == api.YR_EINVAL
    assert "too small" in lib.yr_last_error().decode()
    assert lib.yr_host_prefill_create(ctypes.byref(plan), B, Hq, Hkv, T, d, 2,
                                      ctypes.c_void_p(4096 + 16), n) == api.YR_EINVAL
    assert "aligned" in lib.yr_last_error().decode()
    assert lib.yr_host_prefill_run(None, None, None, None, None, None, 1, 0, 0, None) == \
        api.YR_EINVAL
    assert lib.yr_host_prefill_destroy(None) == api.YR_OK
