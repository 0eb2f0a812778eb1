"""Host logic that needs no GPU: work accounting and the seeded workload recipe."""
import numpy as np
import pytest
import torch

from yarn_position_scaling_b200 import metrics, synth


def brute_visible(T, causal, window, n_sink):
    m = np.arange(T)[:, None]
    n = np.arange(T)[None, :]
    vis = np.ones((T, T), bool)
    if causal:
        vis &= n <= m
    if window:
        vis &= ((m - n) < window) | (n < n_sink)
    return vis.sum(1)


@pytest.mark.parametrize("T,causal,window,n_sink", [(1, True, 0, 0), (300, True, 0, 0),
                                                    (300, False, 0, 0), (300, True, 64, 0),
                                                    (300, True, 64, 4), (300, True, 500, 7),
                                                    (257, True, 1, 0), (400, True, 100, 150)])
def test_visible_counts_match_brute_force(T, causal, window, n_sink):
    np.testing.assert_array_equal(metrics.visible_counts(T, causal, window, n_sink),
                                  brute_visible(T, causal, window, n_sink))


def test_flop_convention_matches_the_pages_table(golden):
    g = golden("pages_worked_numbers.json")
    rows = g["dense_flops_per_head"]
    for r in rows["rows"]:
        # dense (every query sees every key), one head, batch 1
        got = metrics.prefill_flops(1, 1, r["T"], rows["d"], causal=False)
        assert got == pytest.approx(r["printed_flop"], rel=r["rel_tol"])
    a = g["attention_core_70b"]
    got = metrics.prefill_flops(1, a["heads"], a["T"], a["d"], causal=False) * a["layers"]
    assert got == pytest.approx(a["printed_flop"], rel=a["rel_tol"])


def test_page_sink_window_count(golden):
    g = golden("pages_worked_numbers.json")["sink_window"]
    c = metrics.visible_counts(10000, True, g["window"], g["n_sink"])
    assert c[-1] == g["effective_context"]
    assert metrics.decode_visible_keys(10 ** 6, g["window"], g["n_sink"]) == g["effective_context"]


def test_workload_flops():
    w = synth.LLAMA2_16K
    assert metrics.prefill_flops(w.B, w.Hq, w.T, w.d) == pytest.approx(2.199e12, rel=1e-3)
    w = synth.LLAMA3_128K
    assert metrics.prefill_flops(w.B, w.Hq, w.T, w.d) == pytest.approx(1.407e14, rel=1e-3)
    dense, win = synth.SWEEP[0], synth.SWEEP[1]
    assert metrics.prefill_flops(1, 32, 65536, 128) == pytest.approx(3.518e13, rel=1e-3)
    assert metrics.prefill_flops(1, 32, 65536, 128, True, win.window, win.n_sink) == \
        pytest.approx(4.265e12, rel=1e-3)
    assert dense.window == 0 and win.window == 4096 and win.n_sink == 4


def test_decode_bytes():
    assert metrics.decode_kv_bytes([0], 8, 128) == 2 * 8 * 128 * 2
    assert metrics.decode_kv_bytes([99, 9], 2, 64) == 2 * 110 * 2 * 64 * 2
    assert metrics.decode_visible_keys(99, 10, 3) == 13
    lens = synth.cache_lengths(synth.DECODE)
    b = metrics.decode_kv_bytes(lens.tolist(), 8, 128)
    assert 1.3e9 < b < 4.3e9  # 8 sequences of 32K..128K keys


def test_synthetic_inputs_are_seeded_and_shaped():
    w = synth.TINY
    q1, k1, v1 = synth.prefill_inputs(w)
    q2, k2, v2 = synth.prefill_inputs(w)
    assert q1.shape == (1, 4, 256, 64) and k1.shape == (1, 2, 256, 64)
    assert q1.dtype == torch.bfloat16
    assert torch.equal(q1, q2) and torch.equal(v1, v2) and not torch.equal(q1[0, :2], k1[0])
    x = q1.float()
    assert abs(x.mean().item()) < 0.05 and abs(x.std().item() - 1.0) < 0.05
    lens = synth.cache_lengths(synth.DECODE)
    assert lens.dtype == torch.int32 and lens.shape == (8,)
    assert int(lens.min()) >= 32768 and int(lens.max()) <= 131072
    assert torch.equal(lens, synth.cache_lengths(synth.DECODE))


@pytest.mark.parametrize("window,n_sink", [(0, 0), (64, 4)])
def test_chunk_flops_reduce_to_prefill_and_decode(window, n_sink):
    # a chunk at position 0 is a causal prefill; a one-token chunk is a decode step
    assert metrics.chunk_flops(2, 8, 128, 0, 300, window, n_sink) == \
        metrics.prefill_flops(2, 8, 300, 128, True, window, n_sink)
    assert metrics.chunk_flops(1, 8, 128, 5000, 1, window, n_sink) == \
        metrics.decode_flops([5000], 8, 128, window, n_sink)
    # splitting a prompt into prefix + chunk splits its FLOPs
    assert metrics.chunk_flops(1, 4, 64, 0, 700, window, n_sink) == \
        metrics.chunk_flops(1, 4, 64, 0, 300, window, n_sink) + \
        metrics.chunk_flops(1, 4, 64, 300, 400, window, n_sink)


def test_chunk_inputs_are_seeded_and_shaped():
    w = synth.CHUNK
    a = synth.chunk_inputs(w, "cpu", P0=10, Tq=5, T_max=20)
    b = synth.chunk_inputs(w, "cpu", P0=10, Tq=5, T_max=20)
    assert [t.shape for t in a] == [(1, 32, 5, 128), (1, 8, 5, 128), (1, 8, 5, 128),
                                    (1, 8, 20, 128), (1, 8, 20, 128)]
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert all(t.dtype == torch.bfloat16 for t in a)
