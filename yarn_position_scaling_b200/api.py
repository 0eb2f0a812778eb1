"""ctypes binding of libyarnattn.so (include/yarnattn.h), same names as the C ABI.

Argument marshalling only: tensors are passed as raw device pointers with
their strides, on the current PyTorch stream.  Every computation happens in
the library's CUDA kernels; there is no CPU path.  Loading fails loudly if the
library has not been built (``python -m yarn_position_scaling_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB

YR_OK, YR_EINVAL, YR_EUNSUPPORTED, YR_ECUDA, YR_ETIMEOUT, YR_ERANGE = 0, -1, -2, -3, -4, -5
ROPE, PI, NTK, YARN = 0, 1, 2, 3
NTK_DYNAMIC, YARN_DIMRAMP, FACTORS, ALIBI = 4, 5, 6, 7
PAIR_INTERLEAVED, PAIR_HALF = 0, 1
PAIRS = {"interleaved": PAIR_INTERLEAVED, "half": PAIR_HALF}
METHODS = {"rope": ROPE, "pi": PI, "ntk": NTK, "yarn": YARN, "ntk_dynamic": NTK_DYNAMIC,
           "yarn_dimramp": YARN_DIMRAMP, "factors": FACTORS, "alibi": ALIBI}
SYMBOLS = ("yr_rope_freq_table", "yr_attn_prefill_workspace_bytes", "yr_attn_prefill",
           "yr_prefill_prepare_kv", "yr_prefill_attend", "yr_attn_prefill_chunk",
           "yr_attn_prefill_chunk_fp16cache", "yr_attn_prefill_chunk_split_bytes",
           "yr_prefill_prepare_kv_at",
           "yr_prefill_attend_block", "yr_attn_merge",
           "yr_attn_decode_workspace_bytes", "yr_attn_decode", "yr_attn_decode_noalloc",
           "yr_host_prefill_workspace_bytes", "yr_host_prefill_create", "yr_host_prefill_run",
           "yr_host_prefill_destroy", "yr_device_status", "yr_last_error", "yr_version")


class YarnAttnError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"[{code}] {message}")
        self.code = code


class RopeParams(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int), ("base", ctypes.c_double), ("L_train", ctypes.c_int),
                ("scale", ctypes.c_double), ("method", ctypes.c_int), ("alpha", ctypes.c_double),
                ("beta", ctypes.c_double), ("L_cur", ctypes.c_int),
                ("factors", ctypes.POINTER(ctypes.c_double)), ("attn_factor", ctypes.c_double),
                ("pairs", ctypes.c_int)]


class RopeTable(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int), ("method", ctypes.c_int),
                ("inv_freq", ctypes.c_double * 64), ("turns", ctypes.c_double * 64),
                ("mscale", ctypes.c_double), ("softmax_scale", ctypes.c_double),
                ("digest", ctypes.c_uint64), ("pairs", ctypes.c_int)]


_lib = None


def load(path: str | None = None, make_default: bool = False) -> ctypes.CDLL:
    """Load libyarnattn.so (once).  Raises if it is missing.  With `path`, load that build
    of the library instead; make_default=True makes it the one every call below uses."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB
    if not os.path.exists(p):
        raise RuntimeError(f"libyarnattn.so not found at {p}: build it with "
                           "`python -m yarn_position_scaling_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i64p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64)
    ci, cs = ctypes.c_int, ctypes.c_size_t
    lib.yr_rope_freq_table.argtypes = [ctypes.POINTER(RopeParams), ctypes.POINTER(RopeTable)]
    lib.yr_rope_freq_table.restype = ci
    lib.yr_attn_prefill_workspace_bytes.argtypes = [ci, ci, ci, ci]
    lib.yr_attn_prefill_workspace_bytes.restype = cs
    lib.yr_attn_prefill.argtypes = ([vp] * 8 + [ci] * 5 + [i64p] * 5 +
                                    [ctypes.POINTER(RopeTable), ci, ci, ci, vp, cs, vp])
    lib.yr_attn_prefill.restype = ci
    lib.yr_prefill_prepare_kv.argtypes = ([vp] * 4 + [ci] * 4 + [i64p] * 3 +
                                          [ctypes.POINTER(RopeTable), vp, cs, vp])
    lib.yr_prefill_prepare_kv.restype = ci
    lib.yr_prefill_attend.argtypes = ([vp] * 4 + [ci] * 5 + [i64p] * 2 +
                                      [ctypes.POINTER(RopeTable), ci, ci, ci, vp, cs, vp])
    lib.yr_prefill_attend.restype = ci
    lib.yr_attn_prefill_chunk.argtypes = ([vp] * 7 + [ci] * 7 +
                                          [ctypes.POINTER(RopeTable), ci, ci, vp, cs, vp])
    lib.yr_attn_prefill_chunk.restype = ci
    lib.yr_attn_prefill_chunk_fp16cache.argtypes = ([vp] * 7 + [ci] + [vp] * 2 + [ci] * 7 +
                                                    [ctypes.POINTER(RopeTable), ci, ci, vp, cs,
                                                     vp])
    lib.yr_attn_prefill_chunk_split_bytes.argtypes = [ci] * 4
    lib.yr_attn_prefill_chunk_split_bytes.restype = cs
    lib.yr_attn_prefill_chunk_fp16cache.restype = ci
    lib.yr_prefill_prepare_kv_at.argtypes = ([vp] * 4 + [ci] * 4 + [i64p] * 3 +
                                             [ctypes.POINTER(RopeTable), ci, vp, cs, vp])
    lib.yr_prefill_prepare_kv_at.restype = ci
    lib.yr_prefill_attend_block.argtypes = ([vp] * 3 + [ci] * 6 + [i64p] +
                                            [ctypes.POINTER(RopeTable)] + [ci] * 5 + [vp, cs, vp])
    lib.yr_prefill_attend_block.restype = ci
    lib.yr_attn_merge.argtypes = [vp] * 5 + [ctypes.c_longlong, ci, ci, vp]
    lib.yr_attn_merge.restype = ci
    lib.yr_attn_decode_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
    lib.yr_attn_decode_workspace_bytes.restype = cs
    lib.yr_attn_decode.argtypes = ([vp] * 9 + [ci] * 5 +
                                   [ctypes.POINTER(RopeTable), ci, ci, vp, cs, vp])
    lib.yr_attn_decode.restype = ci
    lib.yr_attn_decode_noalloc.argtypes = ([vp] * 9 + [ci] * 5 +
                                           [ctypes.POINTER(RopeTable), ci, ci, vp])
    lib.yr_attn_decode_noalloc.restype = ci
    lib.yr_host_prefill_workspace_bytes.argtypes = [ci] * 6
    lib.yr_host_prefill_workspace_bytes.restype = cs
    lib.yr_host_prefill_create.argtypes = [ctypes.POINTER(vp)] + [ci] * 6 + [vp, cs]
    lib.yr_host_prefill_create.restype = ci
    lib.yr_host_prefill_run.argtypes = [vp] * 5 + [ctypes.POINTER(RopeTable), ci, ci, ci, vp]
    lib.yr_host_prefill_run.restype = ci
    lib.yr_host_prefill_destroy.argtypes = [vp]
    lib.yr_host_prefill_destroy.restype = ci
    lib.yr_device_status.argtypes = [vp]
    lib.yr_device_status.restype = ci
    lib.yr_last_error.argtypes = []
    lib.yr_last_error.restype = ctypes.c_char_p
    lib.yr_version.argtypes = []
    lib.yr_version.restype = ci
    if path is None or make_default:
        _lib = lib
    return lib


def _check(rc: int):
    if rc != YR_OK:
        raise YarnAttnError(rc, load().yr_last_error().decode())


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _strides(t: torch.Tensor):
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a 4-D tensor [B, H, T, d] with unit stride over d")
    return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))


def rope_freq_table(head_dim: int, base: float, L_train: int, scale: float, method,
                    alpha: float = 1.0, beta: float = 32.0, L_cur: int = 0, factors=None,
                    attn_factor: float = 0.0, pairs="interleaved") -> RopeTable:
    """Frequency/temperature table for one position method (host only).  L_cur is the
    current sequence length (dynamic NTK); factors the d/2 per-dimension divisors and
    attn_factor the temperature of the factor method; pairs "interleaved" (2i, 2i+1) or
    "half" (i, i + d/2)."""
    m = METHODS[method] if isinstance(method, str) else int(method)
    pr = PAIRS[pairs] if isinstance(pairs, str) else int(pairs)
    fac = None
    if factors is not None:
        fac = (ctypes.c_double * len(factors))(*[float(x) for x in factors])
    p = RopeParams(int(head_dim), float(base), int(L_train), float(scale), m, float(alpha),
                   float(beta), int(L_cur),
                   ctypes.cast(fac, ctypes.POINTER(ctypes.c_double)) if fac is not None else None,
                   float(attn_factor), pr)
    out = RopeTable()
    _check(load().yr_rope_freq_table(ctypes.byref(p), ctypes.byref(out)))
    return out


def attn_prefill_workspace_bytes(B: int, Hkv: int, T: int, d: int) -> int:
    return int(load().yr_attn_prefill_workspace_bytes(B, Hkv, T, d))


def attn_decode_workspace_bytes(B: int, Hq: int, Hkv: int, d: int, T_max: int) -> int:
    return int(load().yr_attn_decode_workspace_bytes(B, Hq, Hkv, d, T_max))


def attn_prefill(q, k, v, table: RopeTable, causal: bool = True, window: int = 0,
                 n_sink: int = 0, out=None, lse=None, k_cache=None, q_rot_dbg=None,
                 k_rot_dbg=None, workspace=None, stream=None):
    """Attention prefill.  q [B,Hq,T,d], k/v [B,Hkv,T,d] bf16 CUDA tensors (any strides with
    unit stride over d).  Returns the output tensor [B,Hq,T,d] bf16."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty((B, Hq, T, d), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        workspace = torch.empty(attn_prefill_workspace_bytes(B, Hkv, T, d), dtype=torch.uint8,
                                device=q.device)
    kc_strides = _strides(k_cache) if k_cache is not None else None
    rc = load().yr_attn_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(k_cache), _ptr(q_rot_dbg),
        _ptr(k_rot_dbg), B, Hq, Hkv, T, d, _strides(q), _strides(k), _strides(v), _strides(out),
        kc_strides, ctypes.byref(table), int(bool(causal)), int(window), int(n_sink),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc)
    return out


class HostPrefill:
    """Prefill from pinned host tensors into a pinned host output through the library's
    host-buffer entry point (yr_host_prefill_*): the work is cut into (batch, KV-head
    group) units whose host-to-device copies, kernels and device-to-host copies overlap
    on three streams, and successive calls overlap unit by unit.  The device workspace
    is allocated once here for the shape; call it repeatedly for prompts of that shape."""

    def __init__(self, B, Hq, Hkv, T, d, device="cuda", units_per_batch=None):
        self.shape = (B, Hq, Hkv, T, d)
        lib = load()
        n = int(units_per_batch or 0)
        nbytes = int(lib.yr_host_prefill_workspace_bytes(B, Hq, Hkv, T, d, n))
        if nbytes == 0:
            raise ValueError("HostPrefill: invalid sizes")
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=torch.device(device))
        self._lib = lib
        self.plan = ctypes.c_void_p()
        _check(lib.yr_host_prefill_create(ctypes.byref(self.plan), B, Hq, Hkv, T, d, n,
                                          _ptr(self.ws), nbytes))

    def __call__(self, q, k, v, table: RopeTable, causal: bool = True, window: int = 0,
                 n_sink: int = 0, out=None, stream=None):
        """q [B,Hq,T,d], k/v [B,Hkv,T,d] bf16 in pinned host memory, contiguous.  Returns
        `out` (pinned, allocated if None).  All work is ordered before the stream's later
        work; synchronise it before reading `out` or changing the inputs."""
        B, Hq, Hkv, T, d = self.shape
        if q.shape != (B, Hq, T, d) or k.shape != (B, Hkv, T, d) or v.shape != k.shape:
            raise ValueError("HostPrefill: tensor shapes differ from the ones it was built for")
        for t in (q, k, v):
            if t.is_cuda or not t.is_pinned() or not t.is_contiguous() or \
                    t.dtype != torch.bfloat16:
                raise ValueError("HostPrefill expects contiguous bf16 tensors in pinned host "
                                 "memory")
        if out is None:
            out = torch.empty((B, Hq, T, d), dtype=torch.bfloat16).pin_memory()
        _check(self._lib.yr_host_prefill_run(self.plan, _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                             ctypes.byref(table), int(bool(causal)), int(window),
                                             int(n_sink), _stream(stream)))
        return out

    def close(self):
        if self.plan:
            self._lib.yr_host_prefill_destroy(self.plan)
            self.plan = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def prefill_prepare_kv(k, v, table: RopeTable, workspace, k_cache=None, k_rot_dbg=None,
                       stream=None):
    """First half of attn_prefill: rotated keys and values (fp16) into `workspace`."""
    B, Hkv, T, d = k.shape
    kc_strides = _strides(k_cache) if k_cache is not None else None
    rc = load().yr_prefill_prepare_kv(
        _ptr(k), _ptr(v), _ptr(k_cache), _ptr(k_rot_dbg), B, Hkv, T, d, _strides(k),
        _strides(v), kc_strides, ctypes.byref(table), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc)
    return workspace


def prefill_attend(q, Hkv: int, table: RopeTable, workspace, causal: bool = True,
                   window: int = 0, n_sink: int = 0, out=None, lse=None, q_rot_dbg=None,
                   stream=None):
    """Second half of attn_prefill: attention over a workspace from prefill_prepare_kv."""
    B, Hq, T, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, T, d), dtype=torch.bfloat16, device=q.device)
    rc = load().yr_prefill_attend(
        _ptr(q), _ptr(out), _ptr(lse), _ptr(q_rot_dbg), B, Hq, Hkv, T, d, _strides(q),
        _strides(out), ctypes.byref(table), int(bool(causal)), int(window), int(n_sink),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc)
    return out


def prefill_prepare_kv_at(k, v, table: RopeTable, workspace, k_pos0: int, stream=None):
    """prefill_prepare_kv for a block of keys at absolute positions k_pos0 .. k_pos0+T-1."""
    B, Hkv, T, d = k.shape
    rc = load().yr_prefill_prepare_kv_at(
        _ptr(k), _ptr(v), _ptr(None), _ptr(None), B, Hkv, T, d, _strides(k), _strides(v), None,
        ctypes.byref(table), int(k_pos0), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc)
    return workspace


def prefill_attend_block(q, Hkv: int, Tk: int, table: RopeTable, workspace, q_pos0: int,
                         k_pos0: int, causal: bool = True, window: int = 0, n_sink: int = 0,
                         out=None, lse=None, stream=None):
    """Attention of q [B,Hq,T,d] at positions q_pos0.. to the Tk keys at positions k_pos0..
    that prefill_prepare_kv_at left in `workspace`.  Returns (o fp32, lse fp32 [B,Hq,T]):
    the block's own normalised output and log-sum-exp, to be combined by attn_merge."""
    B, Hq, T, d = q.shape
    if out is None:
        out = torch.empty((B, Hq, T, d), dtype=torch.float32, device=q.device)
    if out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("prefill_attend_block writes a contiguous fp32 output")
    if lse is None:
        lse = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    rc = load().yr_prefill_attend_block(
        _ptr(q), _ptr(out), _ptr(lse), B, Hq, Hkv, T, int(Tk), d, _strides(q),
        ctypes.byref(table), int(bool(causal)), int(window), int(n_sink), int(q_pos0),
        int(k_pos0), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(rc)
    return out, lse


def attn_merge(o_part, lse_part, o_acc, lse_acc, out=None, init: bool = False, stream=None):
    """Fold a block partial (o_part fp32 [..., d], lse_part fp32 [...]) into the running
    (o_acc fp32, lse_acc fp32) in place by log-sum-exp weights.  init=True takes the
    accumulator as empty (first block).  If `out` (bf16, shaped like o_part) is given it
    receives the merged rows."""
    d = o_part.shape[-1]
    rows = lse_part.numel()
    for t in (o_part, lse_part, o_acc, lse_acc) + ((out,) if out is not None else ()):
        if not t.is_contiguous():
            raise ValueError("attn_merge expects contiguous tensors")
    rc = load().yr_attn_merge(_ptr(o_part), _ptr(lse_part), _ptr(o_acc), _ptr(lse_acc),
                              _ptr(out), rows, d, int(bool(init)), _stream(stream))
    _check(rc)
    return o_acc, lse_acc


def attn_prefill_chunk(q, k_new, v_new, k_cache, v_cache, P0: int, table: RopeTable,
                       window: int = 0, n_sink: int = 0, out=None, lse=None, workspace=None,
                       stream=None):
    """Chunked prefill after a cached prefix: q [B,Hq,Tq,d], k_new/v_new [B,Hkv,Tq,d] at
    positions P0.., caches [B,Hkv,T_max,d] (contiguous bf16; slots < P0 already rotated).
    Writes slots P0..P0+Tq-1 of the caches; returns the output [B,Hq,Tq,d] bf16."""
    B, Hq, Tq, d = q.shape
    Hkv, T_max = k_cache.shape[1], k_cache.shape[2]
    for t in (q, k_new, v_new, k_cache, v_cache):
        if not t.is_contiguous():
            raise ValueError("attn_prefill_chunk expects contiguous tensors")
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.empty(attn_prefill_workspace_bytes(B, Hkv, P0 + Tq, d),
                                dtype=torch.uint8, device=q.device)
    rc = load().yr_attn_prefill_chunk(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(lse),
        B, Hq, Hkv, Tq, d, int(P0), T_max, ctypes.byref(table), int(window), int(n_sink),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc)
    return out


def attn_prefill_chunk_split_bytes(B: int, Hq: int, Tq: int, d: int) -> int:
    return int(load().yr_attn_prefill_chunk_split_bytes(B, Hq, Tq, d))


def attn_prefill_chunk_fp16cache(q, k_new, v_new, k_cache, v_cache, k_cache16, v_cache16,
                                 cache16_len: int, P0: int, table: RopeTable, window: int = 0,
                                 n_sink: int = 0, out=None, lse=None, workspace=None,
                                 split: bool = True, stream=None):
    """Chunked prefill that keeps an fp16 copy of the cache (k_cache16, v_cache16 fp16
    [B,Hkv,T_max,d]) whose slots < cache16_len are already valid: only slots
    cache16_len..P0-1 are converted, and the chunk's slots are written to both copies.
    `workspace` holds split-KV partials (allocated here when None and split is True;
    split=False runs one CTA per query block).  Returns the output [B,Hq,Tq,d] bf16;
    afterwards slots < P0+Tq of the copy are valid."""
    B, Hq, Tq, d = q.shape
    Hkv, T_max = k_cache.shape[1], k_cache.shape[2]
    for t in (q, k_new, v_new, k_cache, v_cache, k_cache16, v_cache16):
        if not t.is_contiguous():
            raise ValueError("attn_prefill_chunk_fp16cache expects contiguous tensors")
    if k_cache16.dtype != torch.float16 or k_cache16.shape != k_cache.shape or \
            v_cache16.dtype != torch.float16 or v_cache16.shape != v_cache.shape:
        raise ValueError("the fp16 caches must be float16 tensors shaped like the caches")
    if out is None:
        out = torch.empty_like(q)
    if split and workspace is None:
        workspace = torch.empty(attn_prefill_chunk_split_bytes(B, Hq, Tq, d), dtype=torch.uint8,
                                device=q.device)
    if not split:
        workspace = None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().yr_attn_prefill_chunk_fp16cache(
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(k_cache16),
        _ptr(v_cache16), int(cache16_len), _ptr(out), _ptr(lse), B, Hq, Hkv, Tq, d, int(P0),
        T_max, ctypes.byref(table), int(window), int(n_sink), _ptr(workspace), ws_bytes,
        _stream(stream))
    _check(rc)
    return out


def attn_decode(q_new, k_new, v_new, k_cache, v_cache, cache_len, table: RopeTable,
                window: int = 0, n_sink: int = 0, out=None, lse=None, q_rot_dbg=None,
                workspace=None, stream=None):
    """Single-token decode.  q_new [B,Hq,d], k_new/v_new [B,Hkv,d], caches [B,Hkv,T_max,d]
    (contiguous bf16), cache_len int32 [B] on the device.  Writes slot cache_len[b] of the
    caches; returns the output [B,Hq,d] bf16."""
    B, Hq, d = q_new.shape
    Hkv, T_max = k_cache.shape[1], k_cache.shape[2]
    for t in (q_new, k_new, v_new, k_cache, v_cache, cache_len):
        if not t.is_contiguous():
            raise ValueError("attn_decode expects contiguous tensors")
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q_new.device)
    if workspace is None:
        workspace = torch.empty(attn_decode_workspace_bytes(B, Hq, Hkv, d, T_max),
                                dtype=torch.uint8, device=q_new.device)
    rc = load().yr_attn_decode(
        _ptr(q_new), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(cache_len),
        _ptr(out), _ptr(lse), _ptr(q_rot_dbg), B, Hq, Hkv, d, T_max, ctypes.byref(table),
        int(window), int(n_sink), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(rc)
    return out


def attn_decode_noalloc(q_new, k_new, v_new, k_cache, v_cache, cache_len, table: RopeTable,
                        window: int = 0, n_sink: int = 0, out=None, lse=None, q_rot_dbg=None,
                        stream=None):
    """attn_decode with the library's fixed scratch instead of a workspace: the library
    allocates nothing (for callers that cannot allocate device memory).  `out` must be given
    by such callers; it is allocated here only as a convenience when omitted."""
    B, Hq, d = q_new.shape
    Hkv, T_max = k_cache.shape[1], k_cache.shape[2]
    for t in (q_new, k_new, v_new, k_cache, v_cache, cache_len):
        if not t.is_contiguous():
            raise ValueError("attn_decode_noalloc expects contiguous tensors")
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=q_new.device)
    rc = load().yr_attn_decode_noalloc(
        _ptr(q_new), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(cache_len),
        _ptr(out), _ptr(lse), _ptr(q_rot_dbg), B, Hq, Hkv, d, T_max, ctypes.byref(table),
        int(window), int(n_sink), _stream(stream))
    _check(rc)
    return out


def device_status(stream=None) -> int:
    """Synchronise and read/clear the device status word; raises on a recorded fault."""
    rc = load().yr_device_status(_stream(stream))
    _check(rc)
    return rc


def version() -> int:
    return int(load().yr_version())
