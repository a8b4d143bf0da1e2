"""Failure detection without a GPU fault: a bounded device wait made to run
out on purpose, and device allocations made to fail on the host.

* MOEQ_TEST_WAIT_CYCLES, read when a layer is created, shortens the limit
  of every wait the kernels make on one another (mbarriers, issue
  counters).  With a limit of a few cycles, waits give up as soon as data
  is not there yet: the kernel raises MOEQ_ERR_TIMEOUT in the layer status,
  stops issuing copies, drains what it already issued (a fixed, long limit),
  frees its tensor memory and returns.  The test checks the status, that
  the device is still usable, and that a layer with the normal limit then
  computes correctly on it.
* MOEQ_TEST_FAIL_ALLOC=n makes the library's n-th device allocation report
  out-of-memory; moeq_layer_create must then return OUT_OF_MEMORY and leave
  nothing allocated."""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest

from _gpu_util import assert_close, dev_layer, oracle_ref, run, synth, torch_mod

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# one layer per kernel family: decode MXFP4 (grouped GEMV), tensor-core
# MXFP4, tensor-core VQ13+R8, decode VQ13+R8 (grouped GEMV)
FAMILIES = {
    "decode_mxfp4": dict(fmt="mxfp4", act="bf16", H=2048, I=2048, E=16, k=8, T=4),
    "prefill_mxfp4": dict(fmt="mxfp4", act="bf16", H=1024, I=512, E=16, k=4, T=300),
    "vq13r8": dict(fmt="vq13r8", act="bf16", H=1024, I=512, E=16, k=4, T=300),
    "decode_vq13r8": dict(fmt="vq13r8", act="bf16", H=2048, I=2048, E=16, k=8, T=4),
}


@pytest.mark.parametrize("limit", [1, 20000])
@pytest.mark.parametrize("family", sorted(FAMILIES))
def test_wait_runs_out_and_the_device_stays_usable(family, limit, monkeypatch):
    from bit_quantized_moe_routed_b200 import moeq
    torch = torch_mod()
    cfg = synth.get_cfg("tiny_mxfp4", scale_exp=(-9, -5), **FAMILIES[family])
    L = synth.gen_layer(cfg, seed=71)
    x = synth.gen_activations(cfg, seed=71)
    ids, w = synth.gen_routing(cfg, seed=71)
    monkeypatch.setenv("MOEQ_TEST_WAIT_CYCLES", str(limit))
    short = dev_layer(L)
    monkeypatch.delenv("MOEQ_TEST_WAIT_CYCLES")
    n_timeout = 0
    for _ in range(3):
        run(short, cfg, x, ids, w)            # returns: every wait is bounded
        st = short.status(clear=True)
        assert st in (moeq.OK, moeq.TIMEOUT)
        n_timeout += st == moeq.TIMEOUT
    if family == "decode_vq13r8":
        # the VQ decode kernels wait once, for the books, which usually have
        # landed by then: whenever no wait ran out, the result is exact
        out = run(short, cfg, x, ids, w)
        if short.status(clear=True) == moeq.OK:
            assert_close(out, oracle_ref(L, x, ids, w), "bf16", "decode under a short limit")
    elif limit == 1:
        assert n_timeout == 3                  # a 1-cycle limit cannot be met
    torch.cuda.synchronize()                   # the context is intact
    short.close()
    # a layer with the normal limit on the same device computes correctly
    lay = dev_layer(L)
    out = run(lay, cfg, x, ids, w)
    assert lay.status() == moeq.OK
    assert_close(out, oracle_ref(L, x, ids, w), "bf16", f"{family} after timeouts")


_ALLOC_CHILD = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r})
    import torch
    torch.cuda.init()
    torch.cuda.set_device(0)
    from bit_quantized_moe_routed_b200 import moeq
    free0 = torch.cuda.mem_get_info()[0]
    created = False
    try:
        lay = moeq.Layer(1024, 1024, 64, 8, {max_tokens}, {fmt!r}, "bf16")
        created = True
        print("CREATED")
        lay.close()
    except moeq.MoeqError as e:
        print("ERR", e.code)
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    print("LEAK", free0 - free1)
    if not created:
        # the injected failure was used up: the next create succeeds
        lay = moeq.Layer(1024, 1024, 64, 8, {max_tokens}, {fmt!r}, "bf16")
        lay.close()
    print("DONE")
""")


@pytest.mark.parametrize("fmt,max_tokens", [("mxfp4", 8), ("mxfp4", 512), ("vq13r8", 512)])
@pytest.mark.parametrize("fail_at", [1, 3, 14, 18])
def test_failed_allocation_returns_out_of_memory_and_leaks_nothing(fmt, max_tokens, fail_at):
    from bit_quantized_moe_routed_b200 import moeq
    env = dict(os.environ, MOEQ_TEST_FAIL_ALLOC=str(fail_at))
    code = _ALLOC_CHILD.format(root=ROOT, fmt=fmt, max_tokens=max_tokens)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = r.stdout.split()
    assert "DONE" in lines
    if "CREATED" in lines:
        # fewer allocations than fail_at in this configuration: nothing to check
        assert fail_at > 14
        return
    i = lines.index("ERR")
    assert int(lines[i + 1]) == moeq.OUT_OF_MEMORY
    leak = int(lines[lines.index("LEAK") + 1])
    assert abs(leak) <= (2 << 20), f"{leak} bytes not returned after a failed create"
