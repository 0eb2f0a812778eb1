"""yr_attn_decode_noalloc against yr_attn_decode.

The no-allocation entry point serves callers that cannot allocate device memory
(a plugin whose host application owns all device memory, a serving loop that may
not call cudaMalloc once running).  It must give the same results as the entry
point that takes a workspace, call after call, although every call reuses one
fixed scratch array inside the library.  This file is collected last so that a
run that stops at the first failure has already run everything else.
"""
import ctypes
import dataclasses

import pytest
import torch

from yarn_position_scaling_b200 import api, build, synth

pytestmark = pytest.mark.gpu

O_MAX_ABS, O_MEAN_ABS = 1e-2, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    api.load()


def _case(lens, T_max, Hq, Hkv, d, seed_shift):
    w = dataclasses.replace(synth.DECODE, Hq=Hq, Hkv=Hkv, d=d, seed=synth.DECODE.seed + seed_shift)
    qn, kn, vn, kc, vc, _ = synth.decode_inputs(w, "cuda", T_max=T_max, B=len(lens))
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    tab = api.rope_freq_table(d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    return qn, kn, vn, kc, vc, cl, tab


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    cases = [([5, 2999, 700], 3000, 32, 8, 128, 0, 0, 1),
             ([4095, 1, 2048, 31], 4096, 16, 1, 64, 300, 4, 2)]
    for lens, T_max, Hq, Hkv, d, window, n_sink, shift in cases:
        qn, kn, vn, kc, vc, cl, tab = _case(lens, T_max, Hq, Hkv, d, shift)
        kc_ref, vc_ref = kc.clone(), vc.clone()
        ref = api.attn_decode(qn, kn, vn, kc_ref, vc_ref, cl, tab, window, n_sink)
        got = api.attn_decode_noalloc(qn, kn, vn, kc, vc, cl, tab, window, n_sink)
        api.device_status()
        err = (got.float() - ref.float()).abs()
        assert err.max().item() <= O_MAX_ABS and err.mean().item() <= O_MEAN_ABS
        assert torch.equal(kc, kc_ref) and torch.equal(vc, vc_ref)


def test_noalloc_rejects_calls_beyond_its_scratch():
    # 16 sequences x 8 KV heads x 16 chunks x 16 heads per group x (128+2) x 4 bytes
    # = 17,039,360 bytes, just over the 16 MiB scratch: refused before any launch.
    B, Hq, Hkv, d, T_max = 16, 128, 8, 128, 32768
    assert api.attn_decode_workspace_bytes(B, Hq, Hkv, d, T_max) > 16 * 1024 * 1024
    qn = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    kn = torch.zeros((B, Hkv, d), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B, Hkv, T_max, d), dtype=torch.bfloat16, device="cuda")
    cl = torch.zeros((B,), dtype=torch.int32, device="cuda")
    tab = api.rope_freq_table(d, 5e5, 8192, 16.0, "yarn")
    with pytest.raises(api.YarnAttnError) as ei:
        api.attn_decode_noalloc(qn, kn, kn, kc, kc, cl, tab)
    assert ei.value.code == api.YR_EINVAL
    assert "scratch" in str(ei.value)
    api.device_status()
