"""Pins of the oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print, hand-worked encodings, closed forms, brute force on tiny inputs
and invariants.  A plausible slip in the oracle (a wrong nibble order, a
dropped residual, a transposed matrix, silu applied to the wrong branch, a
wrong slot weight) fails at least one of them.
"""
import math
import struct

import numpy as np
import pytest

import oracle
import synth
from synth.gen import GATE, UP, DOWN


# ---------------------------------------------------------------- formats

def test_e2m1_table(golden):
    rows = golden("e2m1_table.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1(int(code))
        want = float(val)
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), (code, got, want)


def test_e8m0_closed_form():
    # 2^(b-127): the byte is a biased exponent with no mantissa.
    assert oracle.e8m0(127) == 1.0
    assert oracle.e8m0(128) == 2.0
    assert oracle.e8m0(126) == 0.5
    assert oracle.e8m0(0) == float.fromhex("0x1p-127")
    assert oracle.e8m0(254) == float.fromhex("0x1p+127")
    assert math.isnan(oracle.e8m0(255))
    for b in range(255):
        assert oracle.e8m0(b) == float.fromhex(f"0x1p{b - 127:+d}")


def test_mxfp4_products_exact_in_f32():
    # every E2M1 x E8M0 product below 2^128 is an f32 value (f32 subnormals
    # included), so the dequantised weight has a single exact f32 value; the
    # few at or above 2^128 (scale byte 253 with |e2m1| >= 4, 254 with >= 2)
    # round to +-inf under IEEE round-to-nearest.
    n_inf = 0
    for c in range(16):
        for b in range(255):
            v = oracle.e2m1(c) * oracle.e8m0(b)
            f = struct.unpack("f", struct.pack("f", v))[0] if abs(v) < 2.0 ** 128 else None
            if f is None:
                n_inf += 1
                assert abs(v) >= 2.0 ** 128
            else:
                assert f == v
    assert n_inf == 2 * (2 + 4)   # |e2m1| in {4, 6} at byte 253, {2, 3, 4, 6} at 254; both signs


def test_bf16_and_f16_widening():
    assert oracle.bf16_to_f32(0x3F80) == 1.0
    assert oracle.bf16_to_f32(0xC040) == -3.0
    assert oracle.bf16_to_f32(0x0001) == float.fromhex("0x1p-133")
    assert oracle.f16_to_f64(0x3C00) == 1.0
    assert oracle.f16_to_f64(0xC000) == -2.0
    assert oracle.f16_to_f64(0x0001) == float.fromhex("0x1p-24")
    assert oracle.f16_to_f64(0x7BFF) == 65504.0
    for bits in (0x3555, 0x0400, 0x03FF, 0xFBFF, 0x1234):
        assert oracle.f16_to_f64(bits) == float(np.array([bits], np.uint16).view(np.float16)[0])


def test_idx13_hand_vectors(golden):
    for row in golden("idx13_vectors.txt"):
        bar = row.index("|")
        stream = np.array([int(b, 16) for b in row[:bar]], np.uint8)
        want = [int(v) for v in row[bar + 1:]]
        assert len(stream) == 13 and len(want) == 8
        assert [oracle.idx13(stream, j) for j in range(8)] == want


def test_idx13_roundtrip_bigint():
    # the stream read as one little-endian integer: index j = (S >> 13j) & 0x1FFF
    rng = np.random.default_rng(7)
    idx = rng.integers(0, 8192, size=64)
    S = 0
    for j, v in enumerate(idx):
        S |= int(v) << (13 * j)
    stream = np.frombuffer(S.to_bytes(64 * 13 // 8, "little"), np.uint8)
    assert [oracle.idx13(stream, j) for j in range(64)] == list(map(int, idx))


def _tiny_cfg(**kw):
    return synth.get_cfg("tiny_mxfp4", **kw)


def _blank_mx_layer(cfg):
    L = synth.Layer(cfg=cfg)
    for p in range(3):
        N, K = cfg.shape(p)
        L.codes[p] = np.zeros((cfg.E, N, K // 2), np.uint8)
        L.scales[p] = np.full((cfg.E, N, K // 32), 127, np.uint8)
    return L


def test_mxfp4_nibble_order_and_block_scale():
    # Row 0 of expert 0's gate: bytes 0x10 0x32 0x54 0x76 0x98 0xBA 0xDC 0xFE
    # repeated; low nibble = even element.  Scales: block 0 -> 2^0,
    # block 1 -> 2^3, others 2^-2.
    cfg = _tiny_cfg()
    L = _blank_mx_layer(cfg)
    pattern = np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], np.uint8)
    L.codes[GATE][0, 0, :] = np.tile(pattern, cfg.H // 16)
    L.scales[GATE][0, 0, :] = 125
    L.scales[GATE][0, 0, 0] = 127
    L.scales[GATE][0, 0, 1] = 130
    W = oracle.dequant(L, 0, GATE)
    mags = [0, .5, 1, 1.5, 2, 3, 4, 6]
    seq = np.array(mags + [-m for m in mags], np.float64)  # element k -> code k % 16
    want = np.concatenate([seq, seq, 8 * seq, 8 * seq] + [0.25 * seq] * (cfg.H // 16 - 4))
    assert np.array_equal(W[0].astype(np.float64), want)
    assert np.signbit(W[0, 8]) and not np.signbit(W[0, 0])   # code 8 is -0
    assert not W[1:].any()


def test_vq_dequant_hand_example():
    # base entry 1 = 1.0 ... ; residual entry 3 = 2^-30 (below half an ulp of
    # 1.0 in f32, so the f32 sum is 1.0); gain 3.0.  f32 order gives exactly
    # 3.0, an f64 evaluation would give 3 + 3*2^-30.
    cfg = synth.get_cfg("tiny_mxfp4", fmt="vq13r8", gains=True)
    L = synth.Layer(cfg=cfg)
    L.book13 = np.zeros((8192, 8), np.uint16)
    L.book8 = np.zeros((256, 8), np.uint16)
    L.book13[1] = [0x3F80, 0x4000, 0x4040, 0x4080, 0xBF80, 0x3F00, 0x0000, 0x3FC0]  # 1 2 3 4 -1 .5 0 1.5
    L.book13[8191] = 0x4120  # 10.0
    L.book8[3] = 0x3080      # 2^-30
    L.book8[255] = 0x3E80    # 0.25
    for p in range(3):
        N, K = cfg.shape(p)
        L.idx13[p] = np.zeros((cfg.E, N, synth.idx13_row_bytes(K)), np.uint8)
        L.idx8[p] = np.zeros((cfg.E, N, K // 8), np.uint8)
        L.gain[p] = np.full((cfg.E, N), 0x3C00, np.uint16)  # 1.0
    # expert 2, up row 5: group 0 -> base 1, residual 3, gain 3.0 (0x4200);
    # group 1 -> base 8191, residual 255.
    S = 1 | (8191 << 13)
    row = S.to_bytes(synth.idx13_row_bytes(cfg.H), "little")
    L.idx13[UP][2, 5] = np.frombuffer(row, np.uint8)
    L.idx8[UP][2, 5, 0] = 3
    L.idx8[UP][2, 5, 1] = 255
    L.gain[UP][2, 5] = 0x4200
    W = oracle.dequant(L, 2, UP)
    base = np.array([1, 2, 3, 4, -1, .5, 0, 1.5])
    # the residual 2^-30 vanishes in every f32 sum except 0 + 2^-30
    want = np.array([3, 6, 9, 12, -3, 1.5, 3 * 2.0 ** -30, 4.5], np.float32)
    assert np.array_equal(W[5, :8], want)
    assert np.array_equal(W[5, 8:16], np.full(8, 3.0 * 10.25, np.float32))
    # untouched rows decode entry 0 of both books (zeros) times gain 1
    assert not W[4].any()
    # without the residual stage the same bytes give the base stage alone
    L2 = L.without_residual()
    W2 = oracle.dequant(L2, 2, UP)
    assert np.array_equal(W2[5, :8], (3.0 * base).astype(np.float32))
    assert np.array_equal(W2[5, 8:16], np.full(8, 30.0, np.float32))


def test_residual_off_is_base_bitwise_and_zero_book_is_off():
    # the 13-bit stage is the same with or without the residual stage
    cfg = synth.get_cfg("tiny_mxfp4", fmt="vq13r8")
    L = synth.gen_layer(cfg, seed=3)
    L0 = L.without_residual()
    Lz = synth.gen_layer(cfg, seed=3)
    Lz.book8 = np.zeros_like(Lz.book8)
    for p in range(3):
        a = oracle.dequant(L0, 1, p)
        b = oracle.dequant(Lz, 1, p)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
        # and it equals a plain table lookup of the base book
        N, K = cfg.shape(p)
        idx = np.array([[oracle.idx13(L.idx13[p][1, n], j) for j in range(K // 8)] for n in range(N)])
        lut = synth.f32_from_bf16_bits(L.book13)
        assert np.array_equal(a, lut[idx].reshape(N, K))
        # with the residual: table lookups of both books added in f32
        r = oracle.dequant(L, 1, p)
        res = synth.f32_from_bf16_bits(L.book8)[L.idx8[p][1].astype(np.int64)].reshape(N, K)
        assert np.array_equal(r, (lut[idx].reshape(N, K) + res).astype(np.float32))


# ---------------------------------------------------------------- forward

def _silu(z):
    return z / (1.0 + math.exp(-z)) if z > -700 else -0.0


# the per-route C loop and the expert-by-expert leg (numpy f64 products of
# the same exact weights) must both satisfy every forward pin
FORWARDS = {"per_route": oracle.forward, "by_expert": oracle.forward_by_expert}


@pytest.mark.parametrize("impl", sorted(FORWARDS))
def test_forward_constant_weights_closed_form(impl):
    # every weight 1.0: g = u = S = sum(x), h = silu(S) S, y_m = I h,
    # out_t = sum_s w_s I silu(S_t) S_t
    cfg = _tiny_cfg()
    L = _blank_mx_layer(cfg)
    for p in range(3):
        L.codes[p][:] = 0x22
    x = synth.gen_activations(cfg, seed=1)
    ids, w = synth.gen_routing(cfg, seed=1)
    out, _ = FORWARDS[impl](L, x, ids, w)
    for t in range(cfg.T):
        S = float(np.sum(x[t].astype(np.float64)))
        want = float(np.sum(w[t].astype(np.float64))) * cfg.I * _silu(S) * S
        np.testing.assert_allclose(out[t], want, rtol=1e-12)


@pytest.mark.parametrize("impl", sorted(FORWARDS))
def test_forward_orientation_one_hot(impl):
    # W_gate[n][k] = [k == n], W_up[n][k] = 2 [k == n+1], W_down[m][n] =
    # [n == m mod I] * (1 if m < I else -0.5): g_n = x_n, u_n = 2 x_{n+1},
    # h_n = silu(x_n) 2 x_{n+1}, y_m = c_m h_{m mod I}.  A transposed matrix,
    # swapped gate/up or silu on the wrong branch breaks it.
    cfg = _tiny_cfg()
    H, I = cfg.H, cfg.I
    L = _blank_mx_layer(cfg)

    def put(p, e, n, k, code):
        b = L.codes[p][e, n, k // 2]
        L.codes[p][e, n, k // 2] = (b & 0xF0) | code if k % 2 == 0 else (b & 0x0F) | (code << 4)

    e = 5
    for n in range(I):
        put(GATE, e, n, n, 2)        # 1.0
        put(UP, e, n, n + 1, 4)      # 2.0
    for m in range(H):
        put(DOWN, e, m, m % I, 2 if m < I else 9)  # 1.0 or -0.5
    x = synth.gen_activations(cfg, seed=2)
    ids = np.full((cfg.T, cfg.k), -1, np.int32)
    ids[:, 1] = e
    w = np.full((cfg.T, cfg.k), 0.75, np.float32)
    if impl == "per_route":
        out, counts, invalid = oracle.forward(L, x, ids, w, want_counts=True)
        assert invalid == 0 and list(counts) == [cfg.T] * 3
    else:
        out, invalid = oracle.forward_by_expert(L, x, ids, w)
        assert invalid == 0
    for t in range(cfg.T):
        xt = x[t].astype(np.float64)
        h = np.array([_silu(xt[n]) * 2.0 * xt[n + 1] for n in range(I)])
        want = np.array([(1.0 if m < I else -0.5) * h[m % I] for m in range(H)]) * 0.75
        np.testing.assert_allclose(out[t], want, rtol=1e-13, atol=0)


def _dense_reference(L, x, ids, w):
    """Brute force: every expert's FFN on every token (numpy f64 matmuls on
    the oracle's dequantised weights), mixed by a dense [T][E] gate matrix
    that is zero for unrouted experts."""
    cfg = L.cfg
    xf = np.asarray(x, np.float64) if x.dtype != np.uint16 else synth.f32_from_bf16_bits(x).astype(np.float64)
    G = np.zeros((cfg.T, cfg.E))
    for t in range(cfg.T):
        for s in range(cfg.k):
            if 0 <= ids[t, s] < cfg.E:
                G[t, ids[t, s]] += w[t, s]
    out = np.zeros((cfg.T, cfg.H))
    for e in range(cfg.E):
        Wg = oracle.dequant(L, e, GATE).astype(np.float64)
        Wu = oracle.dequant(L, e, UP).astype(np.float64)
        Wd = oracle.dequant(L, e, DOWN).astype(np.float64)
        g = xf @ Wg.T
        u = xf @ Wu.T
        h = g / (1.0 + np.exp(-g)) * u
        out += G[:, e:e + 1] * (h @ Wd.T)
    return out


@pytest.mark.parametrize("fmt", ["mxfp4", "vq13", "vq13r8"])
def test_forward_matches_dense_brute_force(fmt):
    cfg = _tiny_cfg(fmt=fmt, gains=(fmt == "vq13r8"))
    L = synth.gen_layer(cfg, seed=0)
    x = synth.gen_activations(cfg, seed=0)
    ids, w = synth.gen_routing(cfg, seed=0)
    out, counts, invalid = oracle.forward(L, x, ids, w, want_counts=True)
    ref = _dense_reference(L, x, ids, w)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())
    assert invalid == 0 and list(counts) == [cfg.T * cfg.k] * 3
    out2, invalid2 = oracle.forward_by_expert(L, x, ids, w)
    np.testing.assert_allclose(out2, ref, rtol=1e-11, atol=1e-11 * np.abs(ref).max())
    assert invalid2 == 0


@pytest.mark.parametrize("fmt,act", [("mxfp4", "bf16"), ("mxfp4", "f32"), ("vq13", "bf16"), ("vq13r8", "bf16")])
def test_forward_by_expert_matches_per_route(fmt, act):
    # a medium layer with repeated experts inside a token, no-route and
    # out-of-range ids, and a token subset in a scrambled order: the
    # expert-by-expert leg agrees with the per-route C loop to f64 rounding
    cfg = synth.get_cfg("tiny_mxfp4", H=256, I=192, E=12, k=4, T=40, fmt=fmt, act=act,
                        gains=(fmt == "vq13r8"), scale_exp=(-9, -5))
    L = synth.gen_layer(cfg, seed=12)
    x = synth.gen_activations(cfg, seed=12)
    ids, w = synth.gen_routing(cfg, seed=12)
    ids[3, 1] = ids[3, 0]
    ids[7, :] = -1
    ids[9, 2] = cfg.E + 3
    ids[11, 0] = -9
    w[5] *= -3.0
    for tokens in (None, np.array([39, 3, 7, 0, 9, 22], np.int32)):
        ref, inv = oracle.forward(L, x, ids, w, tokens=tokens)
        got, inv2 = oracle.forward_by_expert(L, x, ids, w, tokens=tokens)
        assert inv == inv2 == (2 if tokens is None else 1)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13 * np.abs(ref).max())
    assert not got[2].any()     # token 7 has no route


def test_routes_per_token_and_invalid_ids():
    # eight routes per processed token, summed across projections; -1 is
    # "no route", any other id outside [0, E) is skipped and reported
    cfg = synth.get_cfg("tiny_mxfp4", k=8, T=3)
    L = synth.gen_layer(cfg)
    x = synth.gen_activations(cfg)
    ids, w = synth.gen_routing(cfg)
    _, counts, invalid = oracle.forward(L, x, ids, w, want_counts=True)
    assert list(counts) == [cfg.T * 8] * 3 and invalid == 0
    ids2 = ids.copy()
    ids2[0, 3] = -1
    ids2[1, 0] = cfg.E
    ids2[2, 7] = -5
    out2, counts2, invalid2 = oracle.forward(L, x, ids2, w, want_counts=True)
    assert list(counts2) == [cfg.T * 8 - 3] * 3 and invalid2 == 2
    w3 = w.copy()
    w3[0, 3] = w3[1, 0] = w3[2, 7] = 0.0
    out3, _ = oracle.forward(L, x, ids, w3)
    np.testing.assert_allclose(out2, out3, rtol=1e-13, atol=0)


def test_unrouted_experts_contribute_nothing():
    cfg = _tiny_cfg()
    L = synth.gen_layer(cfg, seed=4)
    x = synth.gen_activations(cfg, seed=4)
    ids, w = synth.gen_routing(cfg, seed=4)
    out, _ = oracle.forward(L, x, ids, w)
    used = set(ids.ravel().tolist())
    L2 = synth.gen_layer(cfg, seed=4)
    rng = np.random.default_rng(9)
    for e in range(cfg.E):
        if e not in used:
            for p in range(3):
                L2.codes[p][e] = rng.integers(0, 256, L2.codes[p][e].shape, dtype=np.uint8)
                L2.scales[p][e] = 140
    out2, _ = oracle.forward(L2, x, ids, w)
    assert np.array_equal(out, out2)


def test_linear_in_weights_and_slot_order():
    cfg = synth.get_cfg("tiny_mxfp4", fmt="vq13r8")
    L = synth.gen_layer(cfg, seed=5)
    x = synth.gen_activations(cfg, seed=5)
    ids, w = synth.gen_routing(cfg, seed=5)
    out, _ = oracle.forward(L, x, ids, w)
    out2, _ = oracle.forward(L, x, ids, 2 * w)
    assert np.array_equal(out2, 2 * out)   # doubling is exact in f64
    out3, _ = oracle.forward(L, x, ids[:, ::-1], w[:, ::-1])
    np.testing.assert_allclose(out3, out, rtol=1e-12, atol=1e-14)


def test_token_subset_matches_full():
    cfg = _tiny_cfg()
    L = synth.gen_layer(cfg, seed=6)
    x = synth.gen_activations(cfg, seed=6)
    ids, w = synth.gen_routing(cfg, seed=6)
    out, _ = oracle.forward(L, x, ids, w)
    sub, _ = oracle.forward(L, x, ids, w, tokens=[3, 1])
    assert np.array_equal(sub, out[[3, 1]])


# ---------------------------------------------------------------- page figures

def test_page_shape_figures(golden):
    g = {r[0]: int(r[1]) for r in golden("page_shapes.txt")}
    cfg = synth.get_cfg("decode_mxfp4")
    layers = 47
    H, I, E = cfg.H, cfg.I, cfg.E
    assert E == g["n_experts"] and cfg.k == g["top_k"]
    per_kind = layers * E * H * I                      # weights per projection kind
    assert round(3 * per_kind / 1e8) == g["routed_params_rounded_1e8"]
    # payloads are whole bytes per 256-weight super-block: 66 B (IQ2_XXS), 74 B (IQ2_XS)
    assert g["gateup_payload_bytes"] * 256 == 2 * per_kind * 66
    assert g["down_payload_bytes"] * 256 == per_kind * 74
    assert layers * E * 3 == g["expert_matrices"]
    assert layers * E == g["layer_expert_slots"]
    assert layers * 3 == g["projection_matrices"]
    # one-byte book entries: 8192x8 + 256x8 = 66 KiB, residual book 2 KiB,
    # which is also the gap between the two GB10 kernels' shared memory
    assert (8192 * 8 + 256 * 8) == g["books_kib_one_byte"] * 1024
    assert 256 * 8 == g["residual_book_kib"] * 1024 == g["gb10_smem_r13r8"] - g["gb10_smem_r13"]


# ---------------------------------------------------------------- overflow workload

@pytest.mark.slow
def test_overflow_workload_property_and_finite():
    # the prefill VQ overflow workload (base book x64 shared by gate/up/down,
    # x ~ N(0, 2^2)): some 32-value block sums of the SwiGLU intermediate pass
    # f16's 65504, and the f64 output is finite.  Same per-expert statistics
    # as the full layer, with 8 experts so it stays small.
    cfg = synth.get_cfg("prefill_vq_overflow", E=8, T=1)
    L = synth.gen_layer(cfg, seed=0)
    x = synth.gen_activations(cfg, seed=0)
    ids = np.arange(8, dtype=np.int32)[None, :]
    w = np.full((1, 8), 0.125, np.float32)
    out, h, _ = oracle.forward(L, x, ids, w, want_h=True)
    sums = np.abs(h.reshape(8, cfg.I // 32, 32).sum(-1))
    assert (sums > 65504).any()
    assert np.isfinite(out).all() and np.isfinite(h).all()


def test_route_bucket_hand_example():
    # 3 tokens x 2 slots over 4 experts; -1 = no route, 9 = invalid
    ids = np.array([[2, 0], [0, -1], [2, 9]], np.int32)
    offsets, perm, bad = oracle.route_bucket(ids, 4)
    assert list(offsets) == [0, 2, 2, 4, 4]
    assert list(perm) == [1, 2, 0, 4]
    assert bad == 1


def test_route_bucket_is_a_stable_sort():
    # the bucketed order is numpy's stable argsort of the expert ids
    cfg = synth.get_cfg("prefill_mxfp4_zipf")
    ids, _ = synth.gen_routing(cfg)
    offsets, perm, bad = oracle.route_bucket(ids, cfg.E)
    flat = ids.ravel()
    assert bad == 0 and np.array_equal(perm, np.argsort(flat, kind="stable"))
    assert np.array_equal(np.diff(offsets), np.bincount(flat, minlength=cfg.E))
    assert offsets[13] == offsets[14] and offsets[184] == offsets[185]   # never routed
