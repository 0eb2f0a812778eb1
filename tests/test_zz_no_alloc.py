"""yr_attn_decode_noalloc against yr_attn_decode and the oracle.

The no-allocation entry point serves callers that cannot allocate device memory
(a plugin whose host application owns all device memory, a serving loop that may
not call cudaMalloc once running).  It launches the same kernels with the same
partition as the entry point that takes a workspace, so its outputs must be
bit-identical to that entry point's, call after call, although every call reuses
one fixed scratch array inside the library: a merge that read partial results
left over from an earlier call would show up here.  This file is collected last
so that a run that stops at the first failure has already run everything else.
"""
import dataclasses

import pytest
import torch

import oracle
from tests._util import O_MAX_ABS, O_MEAN_ABS, err_stats, to_bits, to_f64
from yarn_position_scaling_b200 import api, build, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    api.load()


def _case(lens, T_max, Hq, Hkv, d, seed_shift):
    w = dataclasses.replace(synth.DECODE, Hq=Hq, Hkv=Hkv, d=d, seed=synth.DECODE.seed + seed_shift)
    qn, kn, vn, kc, vc, _ = synth.decode_inputs(w, "cuda", T_max=T_max, B=len(lens))
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    tab = api.rope_freq_table(d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    return w, qn, kn, vn, kc, vc, cl, tab


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    # The second case needs fewer partial-result slots than the first left in the
    # scratch, and the second call of each case follows a call with other inputs.
    cases = [([5, 2999, 700], 3000, 32, 8, 128, 0, 0, 1),
             ([4095, 1, 2048, 31], 4096, 16, 1, 64, 300, 4, 2),
             ([17], 100, 4, 2, 128, 0, 0, 3)]
    for lens, T_max, Hq, Hkv, d, window, n_sink, shift in cases:
        w, qn, kn, vn, kc, vc, cl, tab = _case(lens, T_max, Hq, Hkv, d, shift)
        kc0, vc0 = to_bits(kc), to_bits(vc)
        kc_ref, vc_ref = kc.clone(), vc.clone()
        lse_ref = torch.empty((len(lens), Hq), device="cuda")
        ref = api.attn_decode(qn, kn, vn, kc_ref, vc_ref, cl, tab, window, n_sink, lse=lse_ref)
        for _ in range(2):
            lse = torch.full((len(lens), Hq), float("nan"), device="cuda")
            got = api.attn_decode_noalloc(qn, kn, vn, kc, vc, cl, tab, window, n_sink, lse=lse)
            api.device_status()
            assert torch.equal(got, ref)
            assert torch.equal(lse, lse_ref)
            assert torch.equal(kc, kc_ref) and torch.equal(vc, vc_ref)
        # and directly against the fp64 oracle, within the decode tolerances
        th, _, ss = oracle.rope_theta(d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
        ro, _, _, _ = oracle.decode(to_bits(qn), to_bits(kn), to_bits(vn), kc0, vc0,
                                    cl.cpu().numpy(), th, ss, window, n_sink)
        emax, emean = err_stats(to_f64(got), ro)
        assert emax <= O_MAX_ABS and emean <= O_MEAN_ABS, (emax, emean)


def test_noalloc_rejects_calls_beyond_its_scratch():
    # 16 sequences x 8 KV heads x 17 partial-result slots (T_max / 2048 + 1) x 16 heads
    # per group x (128 + 2) floats x 4 bytes = 18,104,320 bytes, more than the 16 MiB
    # scratch: refused before any launch.
    B, Hq, Hkv, d, T_max = 16, 128, 8, 128, 32768
    assert api.attn_decode_workspace_bytes(B, Hq, Hkv, d, T_max) == 18104320
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
