"""Pins of the oracle's GVQ1-style format (12-bit code stream + 1-bit plane,
1-byte E4M3 book entries with one f32 scale per book).  The pages fix only
"a 12-bit code stream plus a 1-bit plane" and 1-byte entries; the byte
layout and the E4M3 reading are this build's, so these pins check the
oracle against the definitions of those readings and against the VQ13
decode, not against page values."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle.vq_encode import pack_idx13


def test_e4m3_matches_torch_float8_for_every_byte():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = codes.to(torch.float32).numpy()
    for b in range(256):
        got = oracle.e4m3(b)
        if math.isnan(ref[b]):
            assert math.isnan(got), b
        else:
            assert got == float(ref[b]) and math.copysign(1, got) == math.copysign(1, float(ref[b])), b


def test_e4m3_closed_form_points():
    assert oracle.e4m3(0x38) == 1.0
    assert oracle.e4m3(0x7E) == 448.0
    assert oracle.e4m3(0x01) == 2.0 ** -9
    assert oracle.e4m3(0x08) == 2.0 ** -6
    assert oracle.e4m3(0xB8) == -1.0
    assert oracle.e4m3(0x80) == 0.0 and math.copysign(1, oracle.e4m3(0x80)) == -1.0
    assert math.isnan(oracle.e4m3(0x7F)) and math.isnan(oracle.e4m3(0xFF))


def test_gvq1_index_hand_vectors(golden):
    for row in golden("gvq1_vectors.txt"):
        b1 = row.index("|")
        b2 = row.index("|", b1 + 1)
        stream = np.array([int(v, 16) for v in row[:b1]], np.uint8)
        plane = np.array([int(v, 16) for v in row[b1 + 1:b2]], np.uint8)
        want = [int(v) for v in row[b2 + 1:]]
        assert [oracle.gvq1_idx(stream, plane, j) for j in range(8)] == want


def test_gvq1_index_round_trip_through_big_integers():
    rng = np.random.default_rng(7)
    idx = rng.integers(0, 8192, size=64)
    lo = sum(int(v & 0xFFF) << (12 * j) for j, v in enumerate(idx))
    hi = sum(int(v >> 12) << j for j, v in enumerate(idx))
    stream = np.frombuffer(lo.to_bytes(64 * 12 // 8, "little"), np.uint8)
    plane = np.frombuffer(hi.to_bytes(8, "little"), np.uint8)
    assert [oracle.gvq1_idx(stream, plane, j) for j in range(64)] == idx.tolist()


@pytest.mark.parametrize("r8,gains", [(False, False), (True, True)])
def test_gvq1_with_power_of_two_scales_equals_the_vq13_decode(r8, gains):
    # with book scales 2^-6 and 2^-8 every E4M3 value times its scale is a
    # bf16 value, so the GVQ1 weights must equal, bit for bit, the VQ13
    # weights of the same indices with those bf16 books
    fmt = "gvq1r8" if r8 else "gvq1"
    cfg = synth.get_cfg("tiny_mxfp4", fmt=fmt, gains=gains, act="bf16", E=3)
    G = synth.gen_layer(cfg, seed=8)
    G.gscale = (2.0 ** -6, 2.0 ** -8 if r8 else 0.0)
    V = synth.Layer(cfg=cfg.replace(fmt="vq13r8" if r8 else "vq13"))
    e4 = lambda b: np.array([oracle.e4m3(int(v)) for v in b.ravel()], np.float32).reshape(b.shape)
    V.book13 = synth.bf16_bits_from_f32(e4(G.gbook13) * np.float32(2.0 ** -6))
    assert np.array_equal(synth.f32_from_bf16_bits(V.book13), e4(G.gbook13) * np.float32(2.0 ** -6))
    if r8:
        V.book8 = synth.bf16_bits_from_f32(e4(G.gbook8) * np.float32(2.0 ** -8))
    for p in range(3):
        N, K = cfg.shape(p)
        idx = np.array([[[oracle.gvq1_idx(G.code12[p][e, n], G.hi1[p][e, n], j) for j in range(K // 8)]
                         for n in range(N)] for e in range(cfg.E)])
        V.idx13[p] = np.stack([pack_idx13(idx[e]) for e in range(cfg.E)])
        V.idx8[p] = G.idx8[p]
        V.gain[p] = G.gain[p]
    for e in range(cfg.E):
        for p in range(3):
            a, b = oracle.dequant(G, e, p), oracle.dequant(V, e, p)
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), (e, p)


def test_gvq1_general_scale_is_the_f32_product():
    cfg = synth.get_cfg("tiny_mxfp4", fmt="gvq1r8", act="bf16", E=1)
    G = synth.gen_layer(cfg, seed=9)
    s13, s8 = np.float32(G.gscale[0]), np.float32(G.gscale[1])
    W = oracle.dequant(G, 0, 0)
    n, j = 5, 3
    c = oracle.gvq1_idx(G.code12[0][0, n], G.hi1[0][0, n], j)
    r = int(G.idx8[0][0, n, j])
    for i in range(8):
        want = np.float32(np.float32(oracle.e4m3(int(G.gbook13[c, i]))) * s13) + \
            np.float32(np.float32(oracle.e4m3(int(G.gbook8[r, i]))) * s8)
        assert W[n, 8 * j + i] == np.float32(want)
