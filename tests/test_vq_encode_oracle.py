"""Pins of the VQ encoder oracle against what the format and the mathematics
fix: exact codewords come back to their own index, a library distance
routine agrees on the unweighted case, ties go to the lowest index, a column
of weight zero is ignored, the base stream does not depend on the residual
stage, and the packed stream decodes back through the format oracle."""
import numpy as np
import pytest
from scipy.spatial.distance import cdist

import oracle
import synth
from oracle.vq_encode import encode_rows, pack_idx13, relative_mse, residual_stage


def _layer(fmt="vq13", gains=False, E=1, N=64, K=256, seed=0):
    # a one-expert "layer" whose gate projection is [N][K]
    cfg = synth.get_cfg("tiny_mxfp4", fmt=fmt, gains=gains, H=K, I=N, E=E, k=1, T=1)
    return cfg, synth.gen_layer(cfg, seed=seed)


def test_exact_codewords_round_trip_with_gains():
    cfg, L = _layer(gains=True, seed=1)
    W = oracle.dequant(L, 0, 0)                      # [N][K] exact f32 weights of random indices
    idx13, _, err13, _ = encode_rows(W, L.book13, gain=L.gain[0][0])
    want = np.array([[oracle.idx13(L.idx13[0][0, n], j) for j in range(cfg.H // 8)] for n in range(cfg.I)])
    assert np.array_equal(idx13, want)
    assert not err13.any()
    assert np.array_equal(pack_idx13(idx13), L.idx13[0][0])


def test_residual_round_trip_and_base_stream_independent_of_residual():
    cfg, L = _layer(fmt="vq13r8", seed=2)
    W = oracle.dequant(L, 0, 0)
    i13, i8, e13, e = encode_rows(W, L.book13, L.book8)
    want13 = np.array([[oracle.idx13(L.idx13[0][0, n], j) for j in range(cfg.H // 8)] for n in range(cfg.I)])
    hit = i13 == want13
    assert hit.mean() > 0.85                         # a residual seldom moves the nearest base entry
    assert np.array_equal(i8[hit], L.idx8[0][0][hit].astype(np.int32))
    assert not e[hit].any()
    # the 13-bit stage is the same with the residual stage off
    j13, _, f13, _ = encode_rows(W, L.book13, None)
    assert np.array_equal(j13, i13) and np.array_equal(f13, e13)


def test_unweighted_matches_a_library_nearest_neighbour():
    rng = np.random.default_rng(3)
    cfg, L = _layer(seed=3)
    W = rng.normal(0, 0.02, size=(16, 128)).astype(np.float32)
    idx13, _, err13, _ = encode_rows(W, L.book13)
    B = synth.f32_from_bf16_bits(L.book13).reshape(-1, 8).astype(np.float64)
    D = cdist(W.reshape(-1, 8).astype(np.float64), B, "sqeuclidean")
    assert np.array_equal(idx13.ravel(), D.argmin(axis=1))
    np.testing.assert_allclose(err13.ravel(), D.min(axis=1), rtol=1e-12, atol=1e-18)


def test_ties_take_the_lowest_index_and_zero_weight_columns_are_ignored():
    book = np.zeros((8192, 8), np.uint16)
    one = synth.bf16_bits_from_f32(np.ones(8, np.float32))
    book[5] = one
    book[9] = one                                   # a duplicate of entry 5
    book[7] = synth.bf16_bits_from_f32(np.array([1, 1, 1, 1, 1, 1, 1, 9], np.float32))
    w = np.ones((1, 64), np.float32)
    idx13, _, _, _ = encode_rows(w, book)
    assert (idx13 == 5).all()                       # 5 and 9 tie at 0; 5 is lower
    w[0, 7] = 9.0                                   # vector 0 now equals entry 7
    cw = np.ones(64)
    idx13, _, _, _ = encode_rows(w, book, col_weight=cw)
    assert idx13[0, 0] == 7
    cw[7] = 0.0                                     # ignore that column: 5 again (lowest of the exact fits)
    idx13, _, err13, _ = encode_rows(w, book, col_weight=cw)
    assert idx13[0, 0] == 5 and err13[0, 0] == 0.0


def test_packed_stream_decodes_through_the_format_oracle():
    rng = np.random.default_rng(4)
    idx = rng.integers(0, 8192, size=(5, 64))
    packed = pack_idx13(idx)
    for n in range(5):
        assert [oracle.idx13(packed[n], j) for j in range(64)] == idx[n].tolist()


def test_residual_stage_lowers_the_error_on_codebook_like_weights():
    # sanity analog of the page's relative-MSE drop with the residual stage:
    # weights drawn near the base book with a residual-book-sized offset
    cfg, L = _layer(fmt="vq13r8", seed=5)
    rng = np.random.default_rng(5)
    B = synth.f32_from_bf16_bits(L.book13).reshape(-1, 8)
    R = synth.f32_from_bf16_bits(L.book8).reshape(-1, 8)
    c = rng.integers(0, 8192, size=(32, 16))
    r = rng.integers(0, 256, size=(32, 16))
    W = (B[c] + R[r] + rng.normal(0, 0.002, size=(32, 16, 8))).reshape(32, 128).astype(np.float32)
    _, _, e13, e = encode_rows(W, L.book13, L.book8)
    m13, m = relative_mse(W, e13), relative_mse(W, e)
    assert m < 0.6 * m13, (m13, m)
    assert (e <= e13 + 1e-18).mean() > 0.9


def test_residual_stage_alone_matches_the_full_encoder():
    cfg, L = _layer(fmt="vq13r8", gains=True, seed=6)
    rng = np.random.default_rng(6)
    W = rng.normal(0, 0.02, size=(8, 128)).astype(np.float32)
    cw = rng.uniform(0.1, 1.0, size=128)
    i13, i8, _, e = encode_rows(W, L.book13, L.book8, L.gain[0][0][:8], cw)
    j8, f = residual_stage(W, L.book13, i13, L.book8, L.gain[0][0][:8], cw)
    assert np.array_equal(i8, j8) and np.array_equal(e, f)
