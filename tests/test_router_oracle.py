"""Pins of the router oracle (sigmoid scores, top-k, normalised weights)
against closed forms, special cases and invariants, not against itself."""
import math

import numpy as np

from oracle.router import router_topk, topk_from_logits


def test_zero_activations_tie_every_expert():
    # z = 0 everywhere: every score is 1/2, the k lowest ids win, weights 1/k
    x = np.zeros((3, 16))
    Wr = np.random.default_rng(0).normal(size=(32, 16))
    ids, w, s = router_topk(x, Wr, 8)
    assert (ids == np.arange(8)).all()
    np.testing.assert_array_equal(w, np.float32(1 / 8))
    np.testing.assert_array_equal(s, 0.5)


def test_hand_example_closed_form():
    # sigma(ln 3) = 3/4, sigma(0) = 1/2, sigma(-ln 3) = 1/4
    Wr = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    x = np.array([[math.log(3.0), 0.0],            # z = (ln3, 0, ln3): tie 0/2 -> ids (0, 2)
                  [math.log(3.0), -math.log(3.0)]])  # z = (ln3, -ln3, 0): ids (0, 2), s (3/4, 1/2)
    ids, w, s = router_topk(x, Wr, 2)
    assert ids.tolist() == [[0, 2], [0, 2]]
    np.testing.assert_allclose(s[0], [0.75, 0.5, 0.75], rtol=1e-15)
    np.testing.assert_allclose(s[1], [0.75, 0.25, 0.5], rtol=1e-15)
    np.testing.assert_allclose(w[0], [0.5, 0.5], rtol=1e-7)
    np.testing.assert_allclose(w[1], [0.6, 0.4], rtol=1e-7)           # (3/4) / (5/4), (1/2) / (5/4)


def test_one_hot_router_selects_the_largest_activations():
    # Wr[e] = c * unit vector pi(e): z[t][e] = c * x[t][pi(e)], so the winners
    # are the experts whose coordinate holds one of the k largest x (argsort)
    rng = np.random.default_rng(1)
    E, k, T = 64, 8, 20
    pi = rng.permutation(E)
    Wr = np.zeros((E, E))
    Wr[np.arange(E), pi] = 2.5
    x = rng.normal(size=(T, E))
    ids, w, _ = router_topk(x, Wr, k)
    inv = np.argsort(pi)                      # coordinate -> expert
    for t in range(T):
        top_coords = np.argsort(-x[t], kind="stable")[:k]
        assert ids[t].tolist() == inv[top_coords].tolist()
        sel = 1 / (1 + np.exp(-2.5 * x[t][top_coords]))
        np.testing.assert_allclose(w[t], sel / sel.sum(), rtol=1e-6)


def test_relabelling_experts_relabels_the_selection():
    rng = np.random.default_rng(2)
    E, H, k = 48, 24, 6
    Wr = rng.normal(size=(E, H))
    x = rng.normal(size=(5, H))
    perm = rng.permutation(E)                 # new expert e' = perm[e]
    Wr2 = np.empty_like(Wr)
    Wr2[perm] = Wr
    ids, w, _ = router_topk(x, Wr, k)
    ids2, w2, _ = router_topk(x, Wr2, k)
    assert (perm[ids] == ids2).all()
    np.testing.assert_array_equal(w, w2)


def test_order_follows_logits_where_scores_saturate():
    # sigma(50) and sigma(60) are both 1.0 in float64: the logits still order them
    Wr = np.array([[50.0], [60.0], [-1.0]])
    ids, w, s = router_topk(np.ones((1, 1)), Wr, 2)
    assert s[0, 0] == s[0, 1] == 1.0
    assert ids.tolist() == [[1, 0]]
    np.testing.assert_allclose(w[0], [0.5, 0.5])


def test_weights_normalised_distinct_and_descending():
    rng = np.random.default_rng(3)
    Wr = rng.normal(size=(256, 64)) * 0.1
    x = rng.normal(size=(7, 64))
    ids, w, _ = router_topk(x, Wr, 8)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-6)
    assert (np.diff(w, axis=1) <= 0).all()
    assert all(len(set(r)) == 8 for r in ids.tolist())


def test_softmax_weighting_hand_example():
    # z = (ln 3, 0, -ln 3), k = 2: softmax over the selected (ln 3, 0) gives
    # (3/4, 1/4); the sigmoid reading gives (3/4, 1/2) / (5/4) = (0.6, 0.4)
    Wr = np.array([[1.0], [0.0], [-1.0]])
    x = np.array([[math.log(3.0)]])
    ids, w, _ = router_topk(x, Wr, 2, score="softmax")
    assert ids.tolist() == [[0, 1]]
    np.testing.assert_allclose(w[0], [0.75, 0.25], rtol=1e-7)
    ids2, w2, _ = router_topk(x, Wr, 2, score="sigmoid")
    assert ids2.tolist() == [[0, 1]]
    np.testing.assert_allclose(w2[0], [0.6, 0.4], rtol=1e-7)


def test_softmax_weighting_matches_the_workload_generator():
    # the expert path's synthetic routing (uniform) draws N(0,1) logits over E,
    # keeps the k largest and softmaxes them: the oracle's softmax reading on
    # those logits must give the same ids and weights
    import synth
    cfg = synth.get_cfg("decode_mxfp4", T=6)
    ids_g, w_g = synth.gen_routing(cfg, seed=9)
    logits = synth.gen._rng(9, 0).normal(0.0, 1.0, size=(cfg.T, cfg.E))
    ids, w = topk_from_logits(logits, cfg.k, "softmax")
    assert np.array_equal(ids, ids_g)
    np.testing.assert_allclose(w, w_g, rtol=1e-6)


def test_selection_uses_the_given_logits_exactly():
    # two logits one float32 ulp apart are ordered as given, ties by id
    z = np.array([[1.0, np.nextafter(np.float32(1.0), np.float32(2.0)), 1.0, -3.0]], np.float32)
    ids, w = topk_from_logits(z, 3)
    assert ids.tolist() == [[1, 0, 2]]
    assert abs(w.sum() - 1.0) < 1e-15
