"""Seeded synthetic workloads (shapes, seeds, value distributions).

This module holds no attention or position arithmetic: it only names the
workloads and draws their inputs.  Tests, the benchmark and the smoke check
use it for both the CUDA path and the CPU oracle, so the two always see the
same bytes.

Recipe: Q, K, V (and the decode KV cache) are i.i.d. N(0, 1) drawn in fp32
from a ``torch.Generator`` seeded with the workload's seed, then rounded to
bf16.  Decode cache lengths are integers drawn uniformly from [32768, 131072]
with a CPU generator on the same seed.  The pages evaluate on trained models
and long-context suites that are not available here; these synthetic tensors
stand in for the activations of the named model shapes.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill", "decode" or "chunk"
    seed: int
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int               # prefill length, or T_max for decode
    method: str          # rope | pi | ntk | yarn
    base: float
    L_train: int
    scale: float
    alpha: float = 1.0
    beta: float = 32.0
    causal: bool = True
    window: int = 0
    n_sink: int = 0
    len_lo: int = 0      # decode: cache-length range (inclusive)
    len_hi: int = 0
    P0: int = 0          # chunk: position of the chunk's first token (cached prefix length)
    Tq: int = 0          # chunk: tokens in the chunk (T is the cache capacity T_max)

    def describe(self) -> dict:
        return dataclasses.asdict(self)


TINY = Workload("tiny_gqa_prefill", "prefill", 0, 1, 4, 2, 64, 256, "yarn", 10000.0, 64, 4.0)
LLAMA2_16K = Workload("llama2_7b_16k_prefill", "prefill", 1, 1, 32, 32, 128, 16384, "yarn",
                      10000.0, 4096, 4.0)
LLAMA3_128K = Workload("llama3_8b_128k_gqa_prefill", "prefill", 2, 1, 32, 8, 128, 131072, "yarn",
                       500000.0, 8192, 16.0)
DECODE = Workload("decode_b8_gqa_128k", "decode", 3, 8, 32, 8, 128, 131073, "yarn", 500000.0,
                  8192, 16.0, len_lo=32768, len_hi=131072)
# The last 4096 tokens of a 128K Llama-3-8B-shaped prompt, after a cached 124K prefix.
CHUNK = Workload("chunk_llama3_8b_124k_plus_4k", "chunk", 5, 1, 32, 8, 128, 131072, "yarn",
                 500000.0, 8192, 16.0, P0=126976, Tq=4096)
# The same heads and table at 2^20 tokens: the largest single-GPU prefill of the path.
LLAMA3_1M = Workload("llama3_8b_1m_gqa_prefill", "prefill", 6, 1, 32, 8, 128, 1 << 20, "yarn",
                     500000.0, 8192, 16.0)


def sweep(method: str, windowed: bool) -> Workload:
    """Method/structure sweep at T=65536: dense causal, or W=4096 with 4 sink tokens."""
    return Workload(f"sweep_{method}_{'w4096s4' if windowed else 'dense'}", "prefill", 4, 1, 32,
                    8, 128, 65536, method, 10000.0, 4096, 16.0,
                    window=4096 if windowed else 0, n_sink=4 if windowed else 0)


SWEEP = [sweep(m, w) for m in ("rope", "pi", "ntk", "yarn") for w in (False, True)]
ALL = {w.name: w for w in [TINY, LLAMA2_16K, LLAMA3_128K, DECODE, CHUNK, LLAMA3_1M] + SWEEP}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, seed: int, device="cpu", offset: int = 0) -> torch.Tensor:
    """i.i.d. N(0,1) in fp32 from a generator seeded with seed*1000+offset, rounded to bf16."""
    g = _gen(seed * 1000 + offset, device)
    return torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32).to(
        torch.bfloat16)


def prefill_inputs(w: Workload, device="cpu", T: int | None = None, B: int | None = None):
    """Q [B,Hq,T,d], K and V [B,Hkv,T,d], contiguous bf16."""
    T = w.T if T is None else T
    B = w.B if B is None else B
    q = randn_bf16((B, w.Hq, T, w.d), w.seed, device, 0)
    k = randn_bf16((B, w.Hkv, T, w.d), w.seed, device, 1)
    v = randn_bf16((B, w.Hkv, T, w.d), w.seed, device, 2)
    return q, k, v


def cache_lengths(w: Workload, B: int | None = None) -> torch.Tensor:
    """Integer cache lengths uniform in [len_lo, len_hi] (int32, CPU)."""
    B = w.B if B is None else B
    g = _gen(w.seed * 1000 + 9, "cpu")
    return torch.randint(w.len_lo, w.len_hi + 1, (B,), generator=g, dtype=torch.int64).to(
        torch.int32)


def decode_inputs(w: Workload, device="cpu", T_max: int | None = None, B: int | None = None):
    """q_new [B,Hq,d]; k_new, v_new [B,Hkv,d]; caches [B,Hkv,T_max,d] (N(0,1), treated as
    already rotated); cache_len int32 [B] on CPU."""
    T_max = w.T if T_max is None else T_max
    B = w.B if B is None else B
    q_new = randn_bf16((B, w.Hq, w.d), w.seed, device, 3)
    k_new = randn_bf16((B, w.Hkv, w.d), w.seed, device, 4)
    v_new = randn_bf16((B, w.Hkv, w.d), w.seed, device, 5)
    k_cache = randn_bf16((B, w.Hkv, T_max, w.d), w.seed, device, 6)
    v_cache = randn_bf16((B, w.Hkv, T_max, w.d), w.seed, device, 7)
    return q_new, k_new, v_new, k_cache, v_cache, cache_lengths(w, B)


def chunk_inputs(w: Workload, device="cpu", P0: int | None = None, Tq: int | None = None,
                 T_max: int | None = None, B: int | None = None):
    """q [B,Hq,Tq,d]; k_new, v_new [B,Hkv,Tq,d]; caches [B,Hkv,T_max,d] whose slots before P0
    stand for already rotated keys (N(0,1) like the rest)."""
    P0 = w.P0 if P0 is None else P0
    Tq = w.Tq if Tq is None else Tq
    T_max = w.T if T_max is None else T_max
    B = w.B if B is None else B
    q = randn_bf16((B, w.Hq, Tq, w.d), w.seed, device, 10)
    k_new = randn_bf16((B, w.Hkv, Tq, w.d), w.seed, device, 11)
    v_new = randn_bf16((B, w.Hkv, Tq, w.d), w.seed, device, 12)
    k_cache = randn_bf16((B, w.Hkv, T_max, w.d), w.seed, device, 13)
    v_cache = randn_bf16((B, w.Hkv, T_max, w.d), w.seed, device, 14)
    return q, k_new, v_new, k_cache, v_cache
