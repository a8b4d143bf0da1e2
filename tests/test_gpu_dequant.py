"""moeq_dequant is bit-exact against the oracle's f32 weights."""
import numpy as np
import pytest

from _gpu_util import dev_layer, oracle, synth, torch_mod

pytestmark = pytest.mark.gpu


def _bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


@pytest.mark.parametrize("fmt,gains", [("mxfp4", False), ("vq13", False), ("vq13r8", False), ("vq13r8", True)])
def test_dequant_tiny_all_experts_bit_exact(fmt, gains):
    torch = torch_mod()
    cfg = synth.get_cfg("tiny_mxfp4", fmt=fmt, gains=gains)
    L = synth.gen_layer(cfg, seed=11)
    lay = dev_layer(L)
    for e in range(cfg.E):
        for p in range(3):
            got = lay.dequant(e, p).cpu().numpy()
            want = oracle.dequant(L, e, p)
            assert np.array_equal(_bits(got), _bits(want)), (fmt, e, p)
    torch.cuda.synchronize()


def test_dequant_mxfp4_extreme_scales_bit_exact():
    # E8M0 bytes 0 and 1 (f32 subnormal products), 253 and 254 (+-inf
    # overflow), every nibble (signed zero included)
    cfg = synth.get_cfg("tiny_mxfp4", E=2)
    L = synth.gen_layer(cfg, seed=12)
    rng = np.random.default_rng(0)
    for p in range(3):
        L.scales[p] = rng.choice(np.array([0, 1, 2, 126, 127, 128, 253, 254], np.uint8), size=L.scales[p].shape)
    lay = dev_layer(L)
    n_inf = n_sub = 0
    for e in range(cfg.E):
        for p in range(3):
            got = lay.dequant(e, p).cpu().numpy()
            want = oracle.dequant(L, e, p)
            assert np.array_equal(_bits(got), _bits(want)), (e, p)
            n_inf += int(np.isinf(want).sum())
            n_sub += int(((want != 0) & (np.abs(want) < np.finfo(np.float32).tiny)).sum())
    assert n_inf > 0 and n_sub > 0


def test_upload_rejects_nan_scale():
    from bit_quantized_moe_routed_b200 import moeq
    cfg = synth.get_cfg("tiny_mxfp4")
    L = synth.gen_layer(cfg)
    L.scales[2][3, 5, 1] = 255
    lay = moeq.Layer.for_cfg(cfg)
    with pytest.raises(moeq.MoeqError) as ei:
        lay.upload(L)
    assert ei.value.code == moeq.INVALID_ARGUMENT
    # forward before a successful upload
    torch = torch_mod()
    x = torch.zeros(cfg.T, cfg.H, device="cuda")
    ids = torch.zeros(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.zeros(cfg.T, cfg.k, device="cuda")
    with pytest.raises(moeq.MoeqError) as ei:
        lay.forward(x, ids, w)
    assert ei.value.code == moeq.NOT_UPLOADED


@pytest.mark.parametrize("name", ["decode_mxfp4", "decode_vq"])
def test_dequant_mimo_sampled_experts_bit_exact(name, mimo_layers):
    L, lay = mimo_layers[name]
    for e in (0, 13, 127, 184, 255):
        for p in range(3):
            got = lay.dequant(e, p).cpu().numpy()
            want = oracle.dequant(L, e, p)
            assert np.array_equal(_bits(got), _bits(want)), (name, e, p)
