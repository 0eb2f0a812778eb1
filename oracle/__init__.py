"""fp64 CPU oracle for YaRN-RoPE causal GQA attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never does: it shares
no code with the CUDA library and is not a fallback for it.

The arithmetic lives in ``yarn_oracle.c`` (plain C, double precision, OpenMP
over independent rows), compiled with gcc into ``oracle/_build/liboracle.so``.
This module only marshals numpy arrays into it.  Inputs are bf16 bit patterns
(``uint16``), widened exactly to double inside the C code.

Parity status (see the header of ``yarn_oracle.c``): every function is pinned
by a test in ``tests/test_oracle_pins.py``.  The interior of the YaRN ramp is a
reading of the pages (linear in r, where they print no value); the oracle is
pinned to that reading's closed form at constructed points.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

ROPE, PI, NTK, YARN = 0, 1, 2, 3
NTK_DYNAMIC, YARN_DIMRAMP, FACTORS = 4, 5, 6
METHODS = {"rope": ROPE, "pi": PI, "ntk": NTK, "yarn": YARN, "ntk_dynamic": NTK_DYNAMIC,
           "yarn_dimramp": YARN_DIMRAMP, "factors": FACTORS}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "yarn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile yarn_oracle.c into oracle/_build/liboracle.so (gcc, -O2, OpenMP)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-D_DEFAULT_SOURCE", "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i32p = ctypes.POINTER(ctypes.c_int32)
        c_int, c_long, c_double = ctypes.c_int, ctypes.c_long, ctypes.c_double
        lib.oracle_rope_theta.argtypes = [c_int, c_double, c_int, c_double, c_int,
                                          c_double, c_double, dp, dp, dp]
        lib.oracle_rope_theta.restype = c_int
        lib.oracle_rope_theta_ext.argtypes = [c_int, c_double, c_int, c_double, c_int,
                                              c_double, c_double, c_int, dp, c_double,
                                              dp, dp, dp]
        lib.oracle_rope_theta_ext.restype = c_int
        lib.oracle_rotate_rows.argtypes = [u16p, c_long, c_int, dp, dp, c_int, dp]
        lib.oracle_rotate_rows.restype = None
        lib.oracle_rotate_rows_f64.argtypes = [dp, c_long, c_int, dp, dp, c_int, dp]
        lib.oracle_rotate_rows_f64.restype = None
        lib.oracle_attn_rows.argtypes = [u16p, u16p, u16p, c_int, c_int, c_int, c_int, c_int,
                                         dp, c_double, c_int, c_int, c_int, i64p, c_long,
                                         dp, dp, dp, dp, c_int]
        lib.oracle_attn_rows.restype = c_int
        lib.oracle_attn_rotated_f64.argtypes = [dp, dp, dp, c_int, c_int, c_int, c_int, c_int,
                                                c_double, c_int, c_int, c_int, i64p, c_long,
                                                dp, dp, dp]
        lib.oracle_attn_rotated_f64.restype = c_int
        lib.oracle_decode.argtypes = [u16p, u16p, u16p, u16p, u16p, c_int, i32p,
                                      c_int, c_int, c_int, c_int, dp, c_double, c_int, c_int,
                                      dp, dp, dp, dp, dp, c_int]
        lib.oracle_decode.restype = c_int
        lib.oracle_prefill_chunk.argtypes = [u16p, u16p, u16p, u16p, u16p, c_int, c_int,
                                             c_int, c_int, c_int, c_int, c_int, dp, c_double,
                                             c_int, c_int, dp, dp, dp, dp, c_int]
        lib.oracle_prefill_chunk.restype = c_int
        lib.oracle_alibi_slopes.argtypes = [c_int, dp]
        lib.oracle_alibi_slopes.restype = None
        lib.oracle_kv_cache_bytes.argtypes = [c_double] * 6
        lib.oracle_kv_cache_bytes.restype = c_double
        _lib = lib
        return lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _bits(x) -> np.ndarray:
    """bf16 data (uint16 bit patterns as numpy, or a torch bf16 tensor) -> contiguous uint16."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch  # only for the view; the oracle does no torch arithmetic
        x = x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(x)
    if a.dtype != np.uint16:
        raise TypeError(f"expected bf16 bit patterns (uint16), got {a.dtype}")
    return a


def rope_theta(d: int, base: float, L_train: int, s: float, method, alpha: float = 1.0,
               beta: float = 32.0, L_cur: int = 0, factors=None, attn_factor: float = 0.0):
    """theta'_i (float64[d/2]), mscale and softmax_scale for one method.  L_cur is the
    current sequence length (dynamic NTK); factors the per-dimension divisors and
    attn_factor the temperature of the factor method."""
    lib = _load()
    m = METHODS[method] if isinstance(method, str) else int(method)
    th = np.zeros(d // 2, dtype=np.float64)
    ms = ctypes.c_double()
    ss = ctypes.c_double()
    f = None if factors is None else np.ascontiguousarray(factors, dtype=np.float64)
    if f is not None and f.shape != (d // 2,):
        raise ValueError("factors must hold d/2 values")
    rc = lib.oracle_rope_theta_ext(int(d), float(base), int(L_train), float(s), m, float(alpha),
                                   float(beta), int(L_cur),
                                   None if f is None else _ptr(f, ctypes.c_double),
                                   float(attn_factor), _ptr(th, ctypes.c_double),
                                   ctypes.byref(ms), ctypes.byref(ss))
    if rc != 0:
        raise ValueError("oracle_rope_theta: invalid arguments")
    return th, ms.value, ss.value


PAIRS = {"interleaved": 0, "half": 1}


def _pairs(pairs) -> int:
    return PAIRS[pairs] if isinstance(pairs, str) else int(pairs)


def rotate(x_bits, pos, theta, pairs="interleaved") -> np.ndarray:
    """Rotate rows of bf16 bits (shape [..., d]) at positions pos (broadcast to rows).
    pairs: "interleaved" (2i, 2i+1) or "half" (i, i + d/2)."""
    lib = _load()
    x = _bits(x_bits)
    d = x.shape[-1]
    rows = x.reshape(-1, d)
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.float64),
                                             (rows.shape[0],)))
    th = np.ascontiguousarray(theta, dtype=np.float64)
    out = np.empty(rows.shape, dtype=np.float64)
    lib.oracle_rotate_rows(_ptr(rows, ctypes.c_uint16), rows.shape[0], d,
                           _ptr(p, ctypes.c_double), _ptr(th, ctypes.c_double), _pairs(pairs),
                           _ptr(out, ctypes.c_double))
    return out.reshape(x.shape)


def rotate_f64(x, pos, theta, pairs="interleaved") -> np.ndarray:
    """Rotate float64 rows (shape [..., d]) at positions pos."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    d = x.shape[-1]
    rows = x.reshape(-1, d)
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.float64),
                                             (rows.shape[0],)))
    th = np.ascontiguousarray(theta, dtype=np.float64)
    out = np.empty(rows.shape, dtype=np.float64)
    lib.oracle_rotate_rows_f64(_ptr(rows, ctypes.c_double), rows.shape[0], d,
                               _ptr(p, ctypes.c_double), _ptr(th, ctypes.c_double),
                               _pairs(pairs), _ptr(out, ctypes.c_double))
    return out.reshape(x.shape)


def _slopes(slopes, Hq):
    if slopes is None:
        return ctypes.POINTER(ctypes.c_double)(), None
    a = np.ascontiguousarray(slopes, dtype=np.float64)
    if a.shape != (Hq,):
        raise ValueError("slopes must hold one value per query head")
    return _ptr(a, ctypes.c_double), a


def alibi_slopes(H: int) -> np.ndarray:
    """ALiBi slope of each of H heads (geometric series 2^(-8/H), 2^(-16/H), ...)."""
    out = np.zeros(H, dtype=np.float64)
    _load().oracle_alibi_slopes(int(H), _ptr(out, ctypes.c_double))
    return out


def attn_rows(q_bits, k_bits, v_bits, theta, softmax_scale, causal=True, window=0, n_sink=0,
              rows=None, want_qrot=False, slopes=None, pairs="interleaved"):
    """Exact attention for selected rows.

    q [B,Hq,T,d], k/v [B,Hkv,T,d] as bf16 bits.  rows: flat indices
    (b*Hq+h)*T+m (None = all).  slopes: per query head, subtracted times (m - n) from
    the scaled logits (ALiBi); None = no bias.  Returns (o [n,d], lse [n], q_rot [n,d]
    or None).
    """
    lib = _load()
    q, k, v = _bits(q_bits), _bits(k_bits), _bits(v_bits)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or v.shape != k.shape:
        raise ValueError("shape mismatch")
    th = np.ascontiguousarray(theta, dtype=np.float64)
    if rows is None:
        n = B * Hq * T
        rp = ctypes.POINTER(ctypes.c_int64)()
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.shape[0]
        rp = _ptr(rows, ctypes.c_int64)
    o = np.empty((n, d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    qr = np.empty((n, d), dtype=np.float64) if want_qrot else None
    sp, _keep = _slopes(slopes, Hq)
    rc = lib.oracle_attn_rows(_ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
                              _ptr(v, ctypes.c_uint16), B, Hq, Hkv, T, d,
                              _ptr(th, ctypes.c_double), float(softmax_scale), int(bool(causal)),
                              int(window), int(n_sink), rp, n, _ptr(o, ctypes.c_double),
                              _ptr(lse, ctypes.c_double),
                              _ptr(qr, ctypes.c_double) if qr is not None
                              else ctypes.POINTER(ctypes.c_double)(), sp, _pairs(pairs))
    if rc != 0:
        raise ValueError(f"oracle_attn_rows failed ({rc})")
    return o, lse, qr


def attn_rotated_f64(q_rot, k_rot, v, softmax_scale, causal=True, window=0, n_sink=0,
                     rows=None, slopes=None):
    """Exact attention on float64 operands whose queries and keys are already rotated:
    q_rot [B,Hq,T,d], k_rot and v [B,Hkv,T,d].  rows as in attn_rows.  Returns
    (o [n,d], lse [n])."""
    lib = _load()
    q = np.ascontiguousarray(q_rot, dtype=np.float64)
    k = np.ascontiguousarray(k_rot, dtype=np.float64)
    vv = np.ascontiguousarray(v, dtype=np.float64)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or vv.shape != k.shape:
        raise ValueError("shape mismatch")
    if rows is None:
        n = B * Hq * T
        rp = ctypes.POINTER(ctypes.c_int64)()
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.shape[0]
        rp = _ptr(rows, ctypes.c_int64)
    o = np.empty((n, d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    sp, _keep = _slopes(slopes, Hq)
    rc = lib.oracle_attn_rotated_f64(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double),
                                     _ptr(vv, ctypes.c_double), B, Hq, Hkv, T, d,
                                     float(softmax_scale), int(bool(causal)), int(window),
                                     int(n_sink), rp, n, _ptr(o, ctypes.c_double),
                                     _ptr(lse, ctypes.c_double), sp)
    if rc != 0:
        raise ValueError(f"oracle_attn_rotated_f64 failed ({rc})")
    return o, lse


def decode(q_new, k_new, v_new, k_cache, v_cache, cache_len, theta, softmax_scale,
           window=0, n_sink=0, slopes=None, pairs="interleaved"):
    """Exact single-token decode.  Returns (o [B,Hq,d], lse [B,Hq], k_rot_new [B,Hkv,d],
    q_rot_new [B,Hq,d])."""
    lib = _load()
    qn, kn, vn = _bits(q_new), _bits(k_new), _bits(v_new)
    kc, vc = _bits(k_cache), _bits(v_cache)
    B, Hq, d = qn.shape
    Hkv = kn.shape[1]
    T_max = kc.shape[2]
    cl = np.ascontiguousarray(cache_len, dtype=np.int32)
    th = np.ascontiguousarray(theta, dtype=np.float64)
    o = np.empty((B, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    kr = np.empty((B, Hkv, d), dtype=np.float64)
    qr = np.empty((B, Hq, d), dtype=np.float64)
    sp, _keep = _slopes(slopes, Hq)
    rc = lib.oracle_decode(_ptr(qn, ctypes.c_uint16), _ptr(kn, ctypes.c_uint16),
                           _ptr(vn, ctypes.c_uint16), _ptr(kc, ctypes.c_uint16),
                           _ptr(vc, ctypes.c_uint16), T_max, _ptr(cl, ctypes.c_int32),
                           B, Hq, Hkv, d, _ptr(th, ctypes.c_double), float(softmax_scale),
                           int(window), int(n_sink), _ptr(o, ctypes.c_double),
                           _ptr(lse, ctypes.c_double), _ptr(kr, ctypes.c_double),
                           _ptr(qr, ctypes.c_double), sp, _pairs(pairs))
    if rc != 0:
        raise ValueError(f"oracle_decode failed ({rc})")
    return o, lse, kr, qr


def prefill_chunk(q, k_new, v_new, k_cache, v_cache, P0, theta, softmax_scale, window=0,
                  n_sink=0, slopes=None, pairs="interleaved"):
    """A chunk of Tq tokens at positions P0.. against a rotated cache prefix (slots < P0).
    q bf16 [B,Hq,Tq,d]; k_new, v_new bf16 [B,Hkv,Tq,d]; caches bf16 [B,Hkv,T_max,d].
    Returns (o [B,Hq,Tq,d], lse [B,Hq,Tq], k_rot_new [B,Hkv,Tq,d]) in float64."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k_new), _bits(v_new)
    kc, vc = _bits(k_cache), _bits(v_cache)
    B, Hq, Tq, d = qb.shape
    Hkv = kb.shape[1]
    T_max = kc.shape[2]
    o = np.zeros((B, Hq, Tq, d), dtype=np.float64)
    lse = np.zeros((B, Hq, Tq), dtype=np.float64)
    kr = np.zeros((B, Hkv, Tq, d), dtype=np.float64)
    th = np.ascontiguousarray(theta, dtype=np.float64)
    sp, _keep = _slopes(slopes, Hq)
    rc = lib.oracle_prefill_chunk(_ptr(qb, ctypes.c_uint16), _ptr(kb, ctypes.c_uint16),
                                  _ptr(vb, ctypes.c_uint16), _ptr(kc, ctypes.c_uint16),
                                  _ptr(vc, ctypes.c_uint16), int(T_max), int(P0), B, Hq, Hkv,
                                  Tq, d, _ptr(th, ctypes.c_double), float(softmax_scale),
                                  int(window), int(n_sink), _ptr(o, ctypes.c_double),
                                  _ptr(lse, ctypes.c_double), _ptr(kr, ctypes.c_double), sp,
                                  _pairs(pairs))
    if rc != 0:
        raise ValueError(f"oracle_prefill_chunk failed ({rc})")
    return o, lse, kr


def kv_cache_bytes(n_layers, n_kv_heads, head_dim, seq_len, batch=1, dtype_bytes=2) -> float:
    return _load().oracle_kv_cache_bytes(float(n_layers), float(n_kv_heads), float(head_dim),
                                         float(seq_len), float(batch), float(dtype_bytes))
