"""Failure detection on the GPU, without a GPU fault.

A test hook, compiled only into the test build of the library
(libyarnattn_faulthooks.so), makes CTA 0's TMA producer skip the copies of one
key/value tile, so a wait that nothing will complete runs out of its (here 300 ms)
limit.  The kernel
must record the timeout in the device status word, drain its own copies and MMAs,
free its tensor memory and return; the host must report YR_ETIMEOUT; and the next
call on the same context must give exactly the result of a clean call.  It runs in
a child process so that the short wait limit and the hook stay out of this one.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent(f"""
    import os, sys
    sys.path.insert(0, {ROOT!r})
    import torch
    from yarn_position_scaling_b200 import api, build, synth
    api.load(build.build(fault_hooks=True), make_default=True)
    w = synth.LLAMA2_16K
    q, k, v = synth.prefill_inputs(w, "cuda", T=1024)
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    ref = api.attn_prefill(q, k, v, tab)
    api.device_status()
    os.environ["YR_FAULT_DROP_KV_TILE"] = "1"
    api.attn_prefill(q, k, v, tab)
    try:
        api.device_status()
        print("NO TIMEOUT REPORTED")
        sys.exit(3)
    except api.YarnAttnError as e:
        assert e.code == api.YR_ETIMEOUT, str(e)
        assert "timeout" in str(e), str(e)
        print("reported:", e)
    del os.environ["YR_FAULT_DROP_KV_TILE"]
    again = api.attn_prefill(q, k, v, tab)
    api.device_status()
    assert torch.equal(again, ref)
    print("CLEAN AFTER TIMEOUT")
""")


def test_prefill_wait_timeout_is_reported_and_the_context_stays_usable():
    env = dict(os.environ, YR_WAIT_TIMEOUT_MS="300")
    env.pop("YR_FAULT_DROP_KV_TILE", None)
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "CLEAN AFTER TIMEOUT" in r.stdout, r.stdout + r.stderr


PRODUCT_CHILD = textwrap.dedent(f"""
    import sys
    sys.path.insert(0, {ROOT!r})
    import torch
    from yarn_position_scaling_b200 import api, build, synth
    build.build()
    w = synth.LLAMA2_16K
    q, k, v = synth.prefill_inputs(w, "cuda", T=1024)
    tab = api.rope_freq_table(w.d, w.base, w.L_train, w.scale, w.method, w.alpha, w.beta)
    api.attn_prefill(q, k, v, tab)
    assert api.device_status() == api.YR_OK
    print("HOOK IGNORED")
""")


def test_product_build_ignores_the_test_hook():
    # The hook exists only in the test build: the product library drops no tile.
    env = dict(os.environ, YR_WAIT_TIMEOUT_MS="300", YR_FAULT_DROP_KV_TILE="1")
    r = subprocess.run([sys.executable, "-c", PRODUCT_CHILD], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "HOOK IGNORED" in r.stdout, r.stdout + r.stderr
