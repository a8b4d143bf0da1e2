"""The MiMo-shaped workloads (hidden 4096, inter 2048, 256 experts, top-8)
against the oracle: every output row of every workload, the two 2048-token
prefill micro-batches included (the oracle's expert-by-expert leg computes
all 2048 rows in about a minute of host time)."""
import numpy as np
import pytest

from _gpu_util import assert_close, oracle, oracle_ref, run, synth

pytestmark = pytest.mark.gpu


def test_decode_mxfp4_batch1(mimo_layers):
    L, lay = mimo_layers["decode_mxfp4"]
    cfg = synth.get_cfg("decode_mxfp4")
    x = synth.gen_activations(cfg)
    ids, w = synth.gen_routing(cfg)
    out = run(lay, cfg, x, ids, w)
    assert_close(out, oracle_ref(L, x, ids, w), "bf16", "decode_mxfp4")


@pytest.mark.parametrize("T", [1, 4, 8])
@pytest.mark.parametrize("residual", [True, False])
def test_decode_vq(mimo_layers, T, residual):
    L, lay = mimo_layers["decode_vq" if residual else "decode_vq_off"]
    cfg = synth.get_cfg("decode_vq", T=T, fmt="vq13r8" if residual else "vq13")
    x = synth.gen_activations(cfg, seed=T)
    ids, w = synth.gen_routing(cfg, seed=T)
    out = run(lay, cfg, x, ids, w)
    assert_close(out, oracle_ref(L, x, ids, w), "bf16", f"decode_vq T={T} r={residual}")


def test_prefill_mxfp4_zipf_all_rows(mimo_layers):
    L, lay = mimo_layers["decode_mxfp4"]
    cfg = synth.get_cfg("prefill_mxfp4_zipf")
    x = synth.gen_activations(cfg)
    ids, w = synth.gen_routing(cfg)
    out = run(lay, cfg, x, ids, w)
    assert np.isfinite(out).all()
    ref, invalid = oracle.forward_by_expert(L, x, ids, w)
    assert invalid == 0
    assert_close(out, ref, "bf16", "prefill_mxfp4_zipf")


def test_prefill_vq_overflow_all_rows(mimo_layers):
    L, lay = mimo_layers["prefill_vq_overflow"]
    cfg = synth.get_cfg("prefill_vq_overflow")
    x = synth.gen_activations(cfg)
    ids, w = synth.gen_routing(cfg)
    out = run(lay, cfg, x, ids, w)
    assert np.isfinite(out).all()
    ref, invalid = oracle.forward_by_expert(L, x, ids, w)
    assert invalid == 0
    assert_close(out, ref, "bf16", "prefill_vq_overflow")
