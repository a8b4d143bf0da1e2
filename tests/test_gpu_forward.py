"""moeq_forward against the oracle on small and medium layers, plus the
invariants the pages fix (unrouted experts contribute nothing, no-route ids,
linearity in the routing weights, slot order, the host-buffer entry point)."""
import numpy as np
import pytest

from _gpu_util import (TOL, assert_close, dev_layer, oracle, oracle_ref, out_to_f64, rel_err_per_token, run,
                       synth, to_dev_inputs, torch_mod)

pytestmark = pytest.mark.gpu


def test_tiny_mxfp4_f32_config():
    cfg = synth.get_cfg("tiny_mxfp4")
    L = synth.gen_layer(cfg)
    x = synth.gen_activations(cfg)
    ids, w = synth.gen_routing(cfg)
    lay = dev_layer(L)
    out = run(lay, cfg, x, ids, w)
    assert_close(out, oracle_ref(L, x, ids, w), "f32", "tiny")


# medium layers: several 128-row tiles, ragged token counts, every format
MEDIUM = [
    dict(H=512, I=256, E=32, k=4, T=37),
    dict(H=1024, I=384, E=8, k=2, T=300),
]


@pytest.mark.parametrize("shape", MEDIUM, ids=["m37", "m300"])
@pytest.mark.parametrize("fmt,act,gains", [("mxfp4", "bf16", False), ("mxfp4", "f32", False),
                                           ("vq13", "bf16", False), ("vq13r8", "bf16", True),
                                           ("vq13r8", "f32", False)])
def test_medium_layers(shape, fmt, act, gains):
    cfg = synth.get_cfg("tiny_mxfp4", fmt=fmt, act=act, gains=gains, scale_exp=(-9, -5), **shape)
    L = synth.gen_layer(cfg, seed=21)
    x = synth.gen_activations(cfg, seed=21)
    ids, w = synth.gen_routing(cfg, seed=21)
    lay = dev_layer(L)
    out = run(lay, cfg, x, ids, w)
    assert_close(out, oracle_ref(L, x, ids, w), act, f"{fmt}/{act}/{shape}")


# A layer whose tensor-core work lists wrap the persistent grid several
# times: 1024 tokens x 8 routes over 64 experts is about 128 routes per
# expert, i.e. two 64-route tiles x 8 row tiles per expert, about 1000 work
# items per projection for 148 CTAs.  Every row is compared, so a fault in
# a late item (the accumulator double buffer, the scheduler's wrap-around)
# cannot hide.
WRAP = dict(H=1024, I=1024, E=64, k=8, T=1024)


@pytest.mark.parametrize("fmt", ["mxfp4", "vq13", "vq13r8"])
def test_wrapping_work_lists_every_row(fmt):
    cfg = synth.get_cfg("tiny_mxfp4", fmt=fmt, act="bf16", gains=(fmt == "vq13r8"), scale_exp=(-9, -5), **WRAP)
    L = synth.gen_layer(cfg, seed=51)
    x = synth.gen_activations(cfg, seed=51)
    ids, w = synth.gen_routing(cfg, seed=51)
    lay = dev_layer(L)
    out = run(lay, cfg, x, ids, w)
    ref, invalid = oracle.forward_by_expert(L, x, ids, w)
    assert invalid == 0
    assert_close(out, ref, "bf16", f"wrap {fmt}")
    # a second routing through the same layer (work lists rebuilt, nothing
    # carried over from the first call)
    ids2, w2 = synth.gen_routing(cfg.replace(routing="zipf", unrouted=(3,)), seed=52)
    out2 = run(lay, cfg, x, ids2, w2)
    ref2, _ = oracle.forward_by_expert(L, x, ids2, w2)
    assert_close(out2, ref2, "bf16", f"wrap {fmt} second call")


def _wide_range_x(cfg, seed):
    """bf16 activations whose every 32-value block holds one element of
    magnitude about 1e3 and 31 of about 1e-3: the widest spread the
    per-block scaling of the tensor-core MXFP4 path (and the per-token
    prescale of the decode path) has to carry."""
    rng = np.random.default_rng(seed)
    xf = rng.normal(0.0, 1e-3, size=(cfg.T, cfg.H)).astype(np.float32)
    big = rng.integers(0, 32, size=(cfg.T, cfg.H // 32))
    sign = rng.choice([-1.0, 1.0], size=big.shape)
    rows = np.arange(cfg.T)[:, None]
    xf[rows, np.arange(cfg.H // 32)[None, :] * 32 + big] = sign * rng.uniform(500.0, 2000.0, size=big.shape)
    return synth.bf16_bits_from_f32(xf)


@pytest.mark.parametrize("shape", [dict(H=1024, I=512, E=16, k=4, T=200),     # tensor-core MXFP4
                                   dict(H=2048, I=2048, E=16, k=8, T=4)],     # decode kernels
                         ids=["prefill", "decode"])
@pytest.mark.parametrize("fmt", ["mxfp4", "vq13r8"])
def test_wide_dynamic_range_inside_a_block(shape, fmt):
    cfg = synth.get_cfg("tiny_mxfp4", fmt=fmt, act="bf16", scale_exp=(-9, -5), **shape)
    L = synth.gen_layer(cfg, seed=61)
    x = _wide_range_x(cfg, 61)
    ids, w = synth.gen_routing(cfg, seed=61)
    lay = dev_layer(L)
    out = run(lay, cfg, x, ids, w)
    assert_close(out, oracle_ref(L, x, ids, w), "bf16", f"wide range {fmt} {shape}")


# decode-sized MXFP4 layers (1..8 tokens, bf16): the grouped-GEMV path
DECODE = [
    dict(H=2048, I=2048, E=16, k=2, T=1),
    dict(H=2048, I=2048, E=8, k=8, T=8),      # every expert gets 8 routes
    dict(H=2048, I=4096, E=32, k=8, T=5),
    dict(H=4096, I=2048, E=64, k=8, T=8),
]


@pytest.mark.parametrize("shape", DECODE, ids=[f"H{s['H']}I{s['I']}E{s['E']}k{s['k']}T{s['T']}" for s in DECODE])
def test_decode_mxfp4_shapes(shape):
    cfg = synth.get_cfg("decode_mxfp4", **shape)
    L = synth.gen_layer(cfg, seed=31)
    x = synth.gen_activations(cfg, seed=31)
    ids, w = synth.gen_routing(cfg, seed=31)
    lay = dev_layer(L)
    n0 = lay.kernel_launches()
    out = run(lay, cfg, x, ids, w)
    assert lay.kernel_launches() - n0 == 1        # the one-launch decode step
    assert_close(out, oracle_ref(L, x, ids, w), "bf16", str(shape))
    # a second call with another routing (per-tile counters must have reset)
    ids2, w2 = synth.gen_routing(cfg, seed=32)
    out2 = run(lay, cfg, x, ids2, w2)
    assert_close(out2, oracle_ref(L, x, ids2, w2), "bf16", str(shape) + " second call")


def test_decode_mxfp4_duplicates_no_routes_and_extreme_activations():
    from bit_quantized_moe_routed_b200 import moeq
    cfg = synth.get_cfg("decode_mxfp4", H=2048, I=2048, E=4, k=4, T=8)
    L = synth.gen_layer(cfg, seed=33)
    x = synth.gen_activations(cfg, seed=33)
    rng = np.random.default_rng(33)
    ids = rng.integers(0, 2, size=(cfg.T, cfg.k)).astype(np.int32)   # ~16 routes per expert, repeats
    ids[3, :] = -1                                                    # a token with no route
    ids[5, 2] = -1
    w = rng.normal(size=(cfg.T, cfg.k)).astype(np.float32)            # any sign, not normalised
    xf = synth.f32_from_bf16_bits(x)
    xf[1] = 0.0                                                       # an all-zero token
    xf[6] *= 2.0 ** 40                                                # a huge one
    xf[7] *= 2.0 ** -60                                               # a tiny one
    x = synth.bf16_bits_from_f32(xf)
    lay = dev_layer(L)
    out = run(lay, cfg, x, ids, w)
    ref = oracle_ref(L, x, ids, w)
    assert not out[1].any() and not out[3].any()
    assert_close(out, ref, "bf16", "duplicates/extremes")
    assert lay.status() == moeq.OK
    # no valid route at all: zeros
    out0 = run(lay, cfg, x, np.full_like(ids, -1), w)
    assert not out0.any()


def _cfg_small():
    return synth.get_cfg("tiny_mxfp4", H=512, I=256, E=32, k=4, T=37, act="bf16", scale_exp=(-9, -5))


def test_unrouted_experts_do_not_change_the_output():
    torch = torch_mod()
    cfg = _cfg_small().replace(E=64, T=8)   # 32 routes over 64 experts: many never routed
    L = synth.gen_layer(cfg, seed=3)
    x = synth.gen_activations(cfg, seed=3)
    ids, w = synth.gen_routing(cfg, seed=3)
    ids[:, 0] = -1                      # some no-route slots too
    used = set(ids.ravel().tolist())
    lay = dev_layer(L)
    out1 = run(lay, cfg, x, ids, w)
    L2 = synth.gen_layer(cfg, seed=3)
    rng = np.random.default_rng(5)
    n_pert = 0
    for e in range(cfg.E):
        if e not in used:
            n_pert += 1
            for p in range(3):
                L2.codes[p][e] = rng.integers(0, 256, size=L2.codes[p][e].shape, dtype=np.uint8)
    assert n_pert > 0
    lay2 = dev_layer(L2)
    out2 = run(lay2, cfg, x, ids, w)
    assert np.array_equal(out1, out2)
    assert_close(out1, oracle_ref(L, x, ids, w), "bf16")
    torch.cuda.synchronize()


def test_no_route_and_out_of_range_ids():
    from bit_quantized_moe_routed_b200 import moeq
    cfg = _cfg_small()
    L = synth.gen_layer(cfg, seed=4)
    x = synth.gen_activations(cfg, seed=4)
    ids, w = synth.gen_routing(cfg, seed=4)
    lay = dev_layer(L)
    ids2 = ids.copy()
    ids2[2, 1] = -1
    ids2[5, 3] = cfg.E
    ids2[7, 0] = -100
    out = run(lay, cfg, x, ids2, w)
    assert lay.status(clear=True) == moeq.ROUTE_OUT_OF_RANGE
    w2 = w.copy()
    w2[2, 1] = w2[5, 3] = w2[7, 0] = 0.0
    assert_close(out, oracle_ref(L, x, ids, w2), "bf16")
    # a token with every slot empty gets exactly zero
    ids3 = ids.copy()
    ids3[0, :] = -1
    out3 = run(lay, cfg, x, ids3, w)
    assert not out3[0].any()
    assert lay.status() == moeq.OK


def test_linear_in_weights_and_slot_permutation():
    cfg = _cfg_small().replace(fmt="vq13r8")
    L = synth.gen_layer(cfg, seed=6)
    x = synth.gen_activations(cfg, seed=6)
    ids, w = synth.gen_routing(cfg, seed=6)
    lay = dev_layer(L)
    ref = oracle_ref(L, x, ids, w)
    out1 = run(lay, cfg, x, ids, w)
    out2 = run(lay, cfg, x, ids, 2 * w)
    out3 = run(lay, cfg, x, ids[:, ::-1], w[:, ::-1])
    assert_close(out1, ref, "bf16")
    assert_close(out2, 2 * ref, "bf16")
    assert_close(out3, ref, "bf16")


def test_forward_host_and_profiled_match_forward():
    torch = torch_mod()
    cfg = _cfg_small()
    L = synth.gen_layer(cfg, seed=7)
    x = synth.gen_activations(cfg, seed=7)
    ids, w = synth.gen_routing(cfg, seed=7)
    lay = dev_layer(L)
    ref = run(lay, cfg, x, ids, w)
    oh = lay.forward_host(x, ids, w)
    outh = out_to_f64(torch.from_numpy(oh.view(np.int16)).view(torch.bfloat16))
    assert_close(outh, oracle_ref(L, x, ids, w), "bf16")
    xt, it, wt = to_dev_inputs(cfg, x, ids, w)
    out = torch.empty_like(xt)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    for e in ev:
        e.record()          # torch creates the CUDA event at its first record
    lay.forward_profiled(xt, it, wt, out, ev)
    torch.cuda.synchronize()
    assert_close(out_to_f64(out), oracle_ref(L, x, ids, w), "bf16")
    times = [ev[i].elapsed_time(ev[i + 1]) for i in range(4)]
    assert all(t >= 0 for t in times)
    # the same result as moeq_forward up to the order of the f32 additions of a
    # token's routes, which the prefill-sized paths do not fix (atomics)
    assert_close(out_to_f64(out), ref, "bf16")


def test_zero_tokens_is_a_noop_and_bad_sizes_fail():
    from bit_quantized_moe_routed_b200 import moeq
    torch = torch_mod()
    cfg = _cfg_small()
    lay = dev_layer(synth.gen_layer(cfg, seed=8))
    x = torch.zeros(0, cfg.H, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(0, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.zeros(0, cfg.k, device="cuda")
    lay.forward(x, ids, w)
    x = torch.zeros(cfg.T + 1, cfg.H, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(cfg.T + 1, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.zeros(cfg.T + 1, cfg.k, device="cuda")
    with pytest.raises(moeq.MoeqError) as ei:
        lay.forward(x, ids, w)
    assert ei.value.code == moeq.INVALID_ARGUMENT


@pytest.mark.gpu
@pytest.mark.parametrize("T", [1, 3])
def test_decode_mxfp4_token_lists_an_expert_twice(T):
    # fewer tokens than routes to one expert: the gate/up passes are as wide
    # as the partial-sum slots (T columns), so every route is kept
    cfg = synth.get_cfg("decode_mxfp4", H=2048, I=2048, E=16, k=8, T=T)
    L = synth.gen_layer(cfg, seed=41)
    x = synth.gen_activations(cfg, seed=41)
    ids, w = synth.gen_routing(cfg, seed=41)
    ids[:, 1] = ids[:, 0]          # slot 1 repeats slot 0's expert
    ids[0, 5] = ids[0, 0]          # and a third route to it for token 0
    lay = dev_layer(L)
    n0 = lay.kernel_launches()
    out = run(lay, cfg, x, ids, w)
    assert lay.kernel_launches() - n0 == 1        # the one-launch decode step
    assert_close(out, oracle_ref(L, x, ids, w), "bf16", f"repeated experts, T={T}")


# decode-sized VQ layers (1..8 tokens, bf16): the VQ grouped-GEMV kernels
VQ_DECODE = [
    dict(H=2048, I=2048, E=16, k=2, T=1),
    dict(H=2048, I=2048, E=8, k=8, T=8),      # every expert gets 8 routes
    dict(H=2048, I=4096, E=32, k=8, T=3),
    dict(H=4096, I=2048, E=64, k=8, T=8),
    dict(H=4096, I=4096, E=16, k=4, T=2),
]


@pytest.mark.parametrize("fmt,gains", [("vq13", False), ("vq13r8", True)])
@pytest.mark.parametrize("shape", VQ_DECODE, ids=[f"H{s['H']}I{s['I']}E{s['E']}k{s['k']}T{s['T']}" for s in VQ_DECODE])
def test_decode_vq_shapes(shape, fmt, gains):
    cfg = synth.get_cfg("decode_vq", fmt=fmt, gains=gains, **shape)
    L = synth.gen_layer(cfg, seed=35)
    x = synth.gen_activations(cfg, seed=35)
    ids, w = synth.gen_routing(cfg, seed=35)
    lay = dev_layer(L)
    n0 = lay.kernel_launches()
    out = run(lay, cfg, x, ids, w)
    assert lay.kernel_launches() - n0 == 2        # the two VQ decode kernels
    assert_close(out, oracle_ref(L, x, ids, w), "bf16", f"{fmt} {shape}")
    # a second call with another routing: the accumulator and the arrival
    # counter must have been cleared by the first
    ids2, w2 = synth.gen_routing(cfg, seed=36)
    out2 = run(lay, cfg, x, ids2, w2)
    assert_close(out2, oracle_ref(L, x, ids2, w2), "bf16", f"{fmt} {shape} second call")


def test_decode_vq_duplicates_no_routes_and_extremes():
    from bit_quantized_moe_routed_b200 import moeq
    cfg = synth.get_cfg("decode_vq", H=2048, I=2048, E=4, k=4, T=8, gains=True)
    L = synth.gen_layer(cfg, seed=37)
    x = synth.gen_activations(cfg, seed=37)
    rng = np.random.default_rng(37)
    ids = rng.integers(0, 2, size=(cfg.T, cfg.k)).astype(np.int32)   # repeats within tokens
    ids[3, :] = -1
    ids[5, 2] = -1
    ids[6, 1] = cfg.E + 2                                             # out of range: skipped, reported
    w = rng.normal(size=(cfg.T, cfg.k)).astype(np.float32)
    xf = synth.f32_from_bf16_bits(x)
    xf[1] = 0.0
    xf[4] *= 2.0 ** 30
    xf[7] *= 2.0 ** -50
    x = synth.bf16_bits_from_f32(xf)
    lay = dev_layer(L)
    out = run(lay, cfg, x, ids, w)
    assert lay.status(clear=True) == moeq.ROUTE_OUT_OF_RANGE
    w_ref = w.copy()
    w_ref[6, 1] = 0.0
    ref = oracle_ref(L, x, np.where(ids < cfg.E, ids, -1), w_ref)
    assert not out[1].any() and not out[3].any()
    assert_close(out, ref, "bf16", "vq duplicates/extremes")
    out0 = run(lay, cfg, x, np.full_like(ids, -1), w)
    assert not out0.any()
    assert lay.status() == moeq.OK
