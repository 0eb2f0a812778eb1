"""Seeded random configurations of the three entry points against the fp64 oracle.

The other GPU tests pick their shapes by hand (tile edges, ragged tails, window
edges).  These draw them: batch, heads and grouping, head size, length, causal
or not, window and sinks, the position method (ALiBi included) and, for the
prefill, the pair layout, from one fixed seed, so the list is the same on every
run and a failure names its case.  Every output element, the log-sum-exp and the
rotated operands are compared with the same tolerances as the hand-picked cases.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from tests._util import O_MAX_ABS, O_MEAN_ABS, ROT_ABS, err_stats, to_bits, to_f64
from tests.test_gpu_chunk import run_chunk
from tests.test_gpu_decode import run_decode
from yarn_position_scaling_b200 import api, build, synth

pytestmark = pytest.mark.gpu

METHODS = ["rope", "pi", "ntk", "yarn"]
LSE_ABS = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    api.load()
    assert torch.cuda.is_available()


def _heads(rng):
    hkv = int(rng.choice([1, 2, 4]))
    return hkv * int(rng.choice([1, 2, 3, 4])), hkv


def _prefill_cases(n, seed=2024):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        hq, hkv = _heads(rng)
        T = int(rng.integers(1, 700))
        causal = bool(rng.random() < 0.8)
        window = int(rng.integers(1, T + 64)) if causal and rng.random() < 0.5 else 0
        n_sink = int(rng.integers(0, 9)) if window else 0
        cases.append(dict(B=int(rng.choice([1, 2])), Hq=hq, Hkv=hkv, d=int(rng.choice([64, 128])),
                          T=T, causal=causal, window=window, n_sink=n_sink,
                          method=str(rng.choice(METHODS + ["alibi"])),
                          scale=float(rng.choice([1.0, 4.0, 16.0])),
                          pairs=str(rng.choice(["interleaved", "half"]))))
    return cases


def _decode_cases(n, seed=2025):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        hq, hkv = _heads(rng)
        T_max = int(rng.integers(2, 5000))
        lens = [int(x) for x in rng.integers(0, T_max, size=int(rng.integers(1, 5)))]
        window = int(rng.integers(1, T_max + 64)) if rng.random() < 0.5 else 0
        cases.append(dict(Hq=hq, Hkv=hkv, d=int(rng.choice([64, 128])), T_max=T_max, lens=lens,
                          window=window, n_sink=int(rng.integers(0, 9)) if window else 0,
                          method=str(rng.choice(METHODS))))
    return cases


def _chunk_cases(n, seed=2026):
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(n):
        hq, hkv = _heads(rng)
        P0 = int(rng.integers(0, 2000))
        Tq = int(rng.integers(1, 600))
        window = int(rng.integers(1, P0 + Tq + 64)) if rng.random() < 0.5 else 0
        cases.append(dict(Hq=hq, Hkv=hkv, d=int(rng.choice([64, 128])), P0=P0, Tq=Tq,
                          B=int(rng.choice([1, 2])), window=window,
                          n_sink=int(rng.integers(0, 9)) if window else 0,
                          method=str(rng.choice(METHODS))))
    return cases


def _ids(cases):
    return ["-".join(f"{k}{v}" for k, v in c.items() if k != "lens") for c in cases]


PREFILL = _prefill_cases(40)
DECODE = _decode_cases(16)
CHUNK = _chunk_cases(16)


@pytest.mark.parametrize("c", PREFILL, ids=_ids(PREFILL))
def test_prefill_random_configurations(c):
    w = dataclasses.replace(synth.TINY, method=c["method"], scale=c["scale"], d=c["d"],
                            Hq=c["Hq"], Hkv=c["Hkv"])
    alibi = c["method"] == "alibi"
    T, B, d = c["T"], c["B"], c["d"]
    q, k, v = synth.prefill_inputs(w, "cuda", T=T, B=B)
    tab = api.rope_freq_table(d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta,
                              pairs=c["pairs"])
    lse = torch.empty(q.shape[:3], device="cuda")
    qd = torch.empty(q.shape, device="cuda")
    kd = torch.empty(k.shape, device="cuda")
    o = api.attn_prefill(q, k, v, tab, c["causal"], c["window"], c["n_sink"], lse=lse,
                         q_rot_dbg=qd, k_rot_dbg=kd)
    api.device_status()
    if alibi:
        th, ss, slopes = np.zeros(d // 2), 1.0 / np.sqrt(d), oracle.alibi_slopes(c["Hq"])
    else:
        th, _, ss = oracle.rope_theta(d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
        slopes = None
    ro, rl, rq = oracle.attn_rows(to_bits(q), to_bits(k), to_bits(v), th, ss, c["causal"],
                                  c["window"], c["n_sink"], want_qrot=True, pairs=c["pairs"],
                                  slopes=slopes)
    emax, emean = err_stats(to_f64(o).reshape(ro.shape), ro)
    assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)
    assert err_stats(to_f64(lse).reshape(-1), rl)[0] <= LSE_ABS
    assert err_stats(to_f64(qd).reshape(rq.shape), rq)[0] <= ROT_ABS
    pos = np.tile(np.arange(T, dtype=np.float64), B * c["Hkv"])
    rk = oracle.rotate(to_bits(k).reshape(-1, d), pos, th, pairs=c["pairs"])
    assert err_stats(to_f64(kd).reshape(rk.shape), rk)[0] <= ROT_ABS


@pytest.mark.parametrize("c", DECODE, ids=_ids(DECODE))
def test_decode_random_configurations(c):
    w = dataclasses.replace(synth.DECODE, Hq=c["Hq"], Hkv=c["Hkv"], d=c["d"], method=c["method"])
    run_decode(w, c["lens"], c["T_max"], window=c["window"], n_sink=c["n_sink"])


@pytest.mark.parametrize("c", CHUNK, ids=_ids(CHUNK))
def test_chunk_random_configurations(c):
    w = dataclasses.replace(synth.CHUNK, Hq=c["Hq"], Hkv=c["Hkv"], d=c["d"], method=c["method"])
    run_chunk(w, c["P0"], c["Tq"], c["P0"] + c["Tq"] + 17, B=c["B"], window=c["window"],
              n_sink=c["n_sink"])
