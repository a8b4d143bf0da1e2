"""The synthetic inputs have the shapes, distributions and structure the
workload definitions ask for (routing, activations, MXFP4 scales, VQ books and
indices).  CPU only; layers are drawn at reduced H and I where the property
does not depend on them."""
import numpy as np
import pytest

import synth
from synth.gen import BOOK13_ROWS, BOOK8_ROWS, idx13_row_bytes


def test_uniform_routing_top_k_of_normal_logits():
    cfg = synth.get_cfg("decode_mxfp4", T=256)
    ids, w = synth.gen_routing(cfg, seed=3)
    assert ids.shape == (256, 8) and w.shape == (256, 8)
    assert ids.dtype == np.int32 and w.dtype == np.float32
    assert ((ids >= 0) & (ids < cfg.E)).all()
    assert all(len(set(r)) == cfg.k for r in ids.tolist())            # k distinct experts per token
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-6)  # softmax over the k
    assert (np.diff(w, axis=1) <= 0).all()                            # largest logit first
    # every expert is reachable and none dominates (uniform popularity)
    counts = np.bincount(ids.ravel(), minlength=cfg.E)
    assert counts.max() < 30 and (counts > 0).sum() > 200


def test_zipf_routing_unrouted_experts_and_popularity():
    cfg = synth.get_cfg("prefill_mxfp4_zipf")
    ids, w = synth.gen_routing(cfg)
    assert ids.shape == (2048, 8)
    assert not np.isin(ids, [13, 184]).any()                          # the two never-routed experts
    assert all(len(set(r)) == 8 for r in ids.tolist())
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-6)
    counts = np.sort(np.bincount(ids.ravel(), minlength=cfg.E))[::-1]
    assert (counts > 0).sum() >= cfg.E - 10                           # the tail is still routed
    # skewed: the top expert takes far more routes than the median one, and the
    # rank-frequency curve of the head falls off like a power law
    assert counts[0] > 10 * counts[len(counts) // 2]
    r = np.arange(2, 40)
    slope = np.polyfit(np.log(r), np.log(counts[r - 1]), 1)[0]
    assert -1.6 < slope < -0.3


def test_disjoint_decode_schedule():
    cfg = synth.get_cfg("decode_mxfp4")
    ids, w = synth.gen_disjoint_routing_schedule(cfg, 70)
    assert ids.shape == (70, 1, 8)
    n_sets = cfg.E // cfg.k
    sets = [frozenset(ids[i, 0].tolist()) for i in range(70)]
    for i in range(69):
        assert not sets[i] & sets[i + 1]                               # consecutive steps share no expert
    for i in range(70 - n_sets):
        assert sets[i] == sets[i + n_sets]                             # a set recurs after E/k steps
    assert len(set(sets[:n_sets])) == n_sets and len(frozenset().union(*sets[:n_sets])) == cfg.E
    np.testing.assert_allclose(w.sum(axis=2), 1.0, rtol=0, atol=1e-6)


@pytest.mark.parametrize("name,lo,hi", [("tiny_mxfp4", -8, -4), ("decode_mxfp4", -9, -5)])
def test_mxfp4_scale_exponents_and_codes(name, lo, hi):
    cfg = synth.get_cfg(name, H=256, I=128, E=4) if name != "tiny_mxfp4" else synth.get_cfg(name)
    L = synth.gen_layer(cfg)
    for p in range(3):
        N, K = cfg.shape(p)
        assert L.codes[p].shape == (cfg.E, N, K // 2) and L.scales[p].shape == (cfg.E, N, K // 32)
        s = L.scales[p]
        assert s.min() == 127 + lo and s.max() == 127 + hi             # E8M0 bytes over the whole range
        nib = np.concatenate([L.codes[p].ravel() & 15, L.codes[p].ravel() >> 4])
        hist = np.bincount(nib, minlength=16)
        assert (hist > 0.8 * nib.size / 16).all()                      # every E2M1 code, uniformly


def test_vq_books_indices_and_overflow_scaling():
    cfg = synth.get_cfg("decode_vq", H=256, I=128, E=4)
    L = synth.gen_layer(cfg)
    b13 = synth.f32_from_bf16_bits(L.book13).astype(np.float64)
    b8 = synth.f32_from_bf16_bits(L.book8).astype(np.float64)
    assert b13.shape == (BOOK13_ROWS, 8) and b8.shape == (BOOK8_ROWS, 8)
    assert abs(b13.std() / 0.02 - 1) < 0.03 and abs(b13.mean()) < 0.001
    assert abs(b8.std() / 0.005 - 1) < 0.1
    for p in range(3):
        N, K = cfg.shape(p)
        assert L.idx13[p].shape == (cfg.E, N, idx13_row_bytes(K))
        assert L.idx8[p].shape == (cfg.E, N, K // 8)
    # the overflow workload's base book is the same draw times 64, exactly
    ov = synth.get_cfg("prefill_vq_overflow", H=256, I=128, E=4)
    Lo = synth.gen_layer(ov)
    np.testing.assert_array_equal(synth.f32_from_bf16_bits(Lo.book13), 64 * synth.f32_from_bf16_bits(L.book13))
    np.testing.assert_array_equal(Lo.book8, L.book8)


@pytest.mark.parametrize("name,sigma", [("decode_mxfp4", 1.0), ("prefill_vq_overflow", 2.0)])
def test_activations_are_bf16_normal(name, sigma):
    cfg = synth.get_cfg(name, T=64)
    x = synth.gen_activations(cfg)
    assert x.dtype == np.uint16 and x.shape == (64, cfg.H)
    xf = synth.f32_from_bf16_bits(x).astype(np.float64)
    assert abs(xf.std() / sigma - 1) < 0.02 and abs(xf.mean()) < 0.02 * sigma
    # bf16 values: the low 16 bits of the f32 pattern are zero
    assert (xf.astype(np.float32).view(np.uint32) & 0xFFFF == 0).all()


def test_tiny_config_is_f32():
    cfg = synth.get_cfg("tiny_mxfp4")
    x = synth.gen_activations(cfg)
    assert x.dtype == np.float32 and x.shape == (4, 256)
    ids, w = synth.gen_routing(cfg)
    assert ids.shape == (4, 2)


def test_draws_depend_on_seed_and_component_only():
    cfg = synth.get_cfg("decode_mxfp4", T=8)
    a_ids, a_w = synth.gen_routing(cfg, seed=5)
    b_ids, b_w = synth.gen_routing(cfg, seed=5)
    np.testing.assert_array_equal(a_ids, b_ids)
    np.testing.assert_array_equal(a_w, b_w)
    c_ids, _ = synth.gen_routing(cfg, seed=6)
    assert not np.array_equal(a_ids, c_ids)
    # the activations do not move when the routing config changes
    np.testing.assert_array_equal(synth.gen_activations(cfg, seed=5),
                                  synth.gen_activations(cfg.replace(routing="zipf"), seed=5))


def test_gvq1_books_streams_and_scales():
    # GVQ1 layers: N(0,1) books rounded to E4M3 (no NaN byte), the book
    # scales carry sigma (and the overflow multiplier), 12-bit streams and
    # bit planes of the right sizes; without the residual stage no residual
    # book, indices or scale
    import torch
    from synth.gen import gvq1_code_row_bytes

    def e4m3_values(b):
        return torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)

    cfg = synth.get_cfg("decode_vq", H=256, I=128, E=4, fmt="gvq1r8")
    L = synth.gen_layer(cfg)
    assert L.gbook13.shape == (BOOK13_ROWS, 8) and L.gbook13.dtype == np.uint8
    assert L.gbook8.shape == (BOOK8_ROWS, 8)
    for book in (L.gbook13, L.gbook8):
        assert not np.isin(book, (0x7F, 0xFF)).any()
    v13 = e4m3_values(L.gbook13)
    assert abs(v13.std() - 1) < 0.03 and abs(v13.mean()) < 0.03
    assert L.gscale == (float(np.float32(0.02)), float(np.float32(0.005)))
    for p in range(3):
        N, K = cfg.shape(p)
        assert gvq1_code_row_bytes(K) == K * 3 // 16
        assert L.code12[p].shape == (cfg.E, N, K * 3 // 16)
        assert L.hi1[p].shape == (cfg.E, N, K // 64)
        assert L.idx8[p].shape == (cfg.E, N, K // 8)
    # the overflow workload's multiplier goes into the base book's scale
    ov = synth.get_cfg("prefill_vq_overflow", H=256, I=128, E=4, fmt="gvq1r8")
    Lo = synth.gen_layer(ov)
    np.testing.assert_array_equal(Lo.gbook13, L.gbook13)
    assert Lo.gscale[0] == float(np.float32(0.02 * 64))
    # no residual stage
    L0 = synth.gen_layer(cfg.replace(fmt="gvq1"))
    assert L0.gbook8 is None and all(a is None for a in L0.idx8) and L0.gscale[1] == 0.0
    np.testing.assert_array_equal(L0.gbook13, L.gbook13)
