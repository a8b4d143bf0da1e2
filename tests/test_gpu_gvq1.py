"""The GVQ1-style format (12-bit code stream + bit-12 plane, E4M3 book
entries with per-book scales) through the C ABI: dequant bit-exact against
the oracle, every forward path (f32 SIMT, bf16 at prefill sizes, the bf16
decode kernels) within the tolerance, and the upload checks."""
import numpy as np
import pytest

from _gpu_util import assert_close, dev_layer, oracle, oracle_ref, run, synth, torch_mod

pytestmark = pytest.mark.gpu


def _bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


@pytest.mark.parametrize("fmt,gains", [("gvq1", False), ("gvq1r8", True)])
def test_gvq1_dequant_bit_exact(fmt, gains):
    cfg = synth.get_cfg("tiny_mxfp4", fmt=fmt, gains=gains, act="bf16")
    L = synth.gen_layer(cfg, seed=111)
    lay = dev_layer(L)
    for e in range(cfg.E):
        for p in range(3):
            assert np.array_equal(_bits(lay.dequant(e, p).cpu().numpy()), _bits(oracle.dequant(L, e, p))), (e, p)


@pytest.mark.parametrize("act,T", [("f32", 4), ("bf16", 37)])
@pytest.mark.parametrize("fmt", ["gvq1", "gvq1r8"])
def test_gvq1_forward_general_paths(fmt, act, T):
    cfg = synth.get_cfg("tiny_mxfp4", fmt=fmt, act=act, gains=True, H=512, I=256, E=16, k=4, T=T)
    L = synth.gen_layer(cfg, seed=112)
    x = synth.gen_activations(cfg, seed=112)
    ids, w = synth.gen_routing(cfg, seed=112)
    lay = dev_layer(L)
    assert_close(run(lay, cfg, x, ids, w), oracle_ref(L, x, ids, w), act, f"{fmt} {act} T={T}")


@pytest.mark.parametrize("fmt", ["gvq1", "gvq1r8"])
def test_gvq1_prefill_runs_the_tensor_core_path(fmt):
    # more than 8 tokens: the VQ tensor-core kernels (route/bucket, route
    # tiles, gather, gate/up, down, cast: 6 launches; the SIMT path takes 4)
    # with the books expanded to bf16 at upload
    cfg = synth.get_cfg("tiny_mxfp4", fmt=fmt, act="bf16", gains=True, H=1024, I=512, E=16, k=4, T=300)
    L = synth.gen_layer(cfg, seed=113)
    x = synth.gen_activations(cfg, seed=113)
    ids, w = synth.gen_routing(cfg, seed=113)
    lay = dev_layer(L)
    n0 = lay.kernel_launches()
    out = run(lay, cfg, x, ids, w)
    assert lay.kernel_launches() - n0 == 6
    assert_close(out, oracle_ref(L, x, ids, w), "bf16", f"{fmt} prefill")


GVQ1_DECODE = [
    dict(H=2048, I=2048, E=16, k=8, T=1),
    dict(H=2048, I=2048, E=8, k=8, T=8),
    dict(H=4096, I=2048, E=64, k=8, T=3),
    dict(H=2048, I=4096, E=16, k=4, T=5),
]


@pytest.mark.parametrize("fmt,gains", [("gvq1", False), ("gvq1r8", True)])
@pytest.mark.parametrize("shape", GVQ1_DECODE, ids=[f"H{s['H']}I{s['I']}E{s['E']}k{s['k']}T{s['T']}" for s in GVQ1_DECODE])
def test_gvq1_decode_kernels(shape, fmt, gains):
    cfg = synth.get_cfg("decode_vq", fmt=fmt, gains=gains, **shape)
    L = synth.gen_layer(cfg, seed=113)
    x = synth.gen_activations(cfg, seed=113)
    ids, w = synth.gen_routing(cfg, seed=113)
    lay = dev_layer(L)
    n0 = lay.kernel_launches()
    out = run(lay, cfg, x, ids, w)
    assert lay.kernel_launches() - n0 == 2        # the two VQ decode kernels
    assert_close(out, oracle_ref(L, x, ids, w), "bf16", f"{fmt} {shape}")
    ids2, w2 = synth.gen_routing(cfg, seed=114)
    assert_close(run(lay, cfg, x, ids2, w2), oracle_ref(L, x, ids2, w2), "bf16", f"{fmt} {shape} second call")


def test_gvq1_mimo_decode_batch1():
    cfg = synth.get_cfg("decode_vq", fmt="gvq1r8")
    L = synth.gen_layer(cfg)
    x = synth.gen_activations(cfg, seed=5)
    ids, w = synth.gen_routing(cfg, seed=5)
    lay = dev_layer(L)
    assert_close(run(lay, cfg, x, ids, w), oracle_ref(L, x, ids, w), "bf16", "gvq1 MiMo T=1")


def test_gvq1_upload_rejects_nan_entries_and_bad_scales():
    from bit_quantized_moe_routed_b200 import moeq
    cfg = synth.get_cfg("tiny_mxfp4", fmt="gvq1r8", act="bf16")
    L = synth.gen_layer(cfg, seed=115)
    lay = moeq.Layer.for_cfg(cfg)
    bad = synth.gen_layer(cfg, seed=115)
    bad.gbook13 = bad.gbook13.copy()
    bad.gbook13[17, 3] = 0xFF                       # E4M3 NaN
    with pytest.raises(moeq.MoeqError) as ei:
        lay.upload(bad)
    assert ei.value.code == moeq.INVALID_ARGUMENT
    bad = synth.gen_layer(cfg, seed=115)
    bad.gscale = (float("inf"), 0.005)
    with pytest.raises(moeq.MoeqError):
        lay.upload(bad)
    lay.upload(L)                                   # the valid layer is accepted afterwards
    torch_mod().cuda.synchronize()
