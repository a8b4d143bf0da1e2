"""moeq_vq_encode (the VQ encoder kernel) against the encoder oracle.

Which codeword is nearest is an integer decided by floating point: the kernel
evaluates the errors in f32 (expanded form), the oracle in float64.  So the
test checks that every index the kernel picks is optimal to within the f32
error bound of the expanded form, and equal to the oracle's wherever the
oracle's margin between the best and the second best candidate is larger
than twice that bound; exact codewords must come back to their own index."""
import numpy as np
import pytest

import oracle
import synth
from _gpu_util import torch_mod
from oracle.vq_encode import (assignment_errors, encode_rows, pack_idx13, residual_stage,
                              second_best_base_errors)

pytestmark = pytest.mark.gpu


def _dev(a, dtype=None):
    torch = torch_mod()
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def _unpack(idx13_bytes, G):
    return np.array([[oracle.idx13(row, j) for j in range(G)] for row in idx13_bytes])


def _encode(W, book13, book8=None, gain=None, cw=None):
    from bit_quantized_moe_routed_b200 import moeq
    torch = torch_mod()
    i13, i8 = moeq.vq_encode(_dev(W), _dev(book13), None if book8 is None else _dev(book8),
                             None if gain is None else _dev(gain),
                             None if cw is None else _dev(np.asarray(cw, np.float32)))
    torch.cuda.synchronize()
    return i13.cpu().numpy(), (None if i8 is None else i8.cpu().numpy())


def _bound(W, book13, gain, cw):
    # f32 error of g^2 sum cw b^2 - 2 g sum (cw w) b, generously: 2^-18 of
    # the sizes of the two terms
    N, K = W.shape
    B = synth.f32_from_bf16_bits(book13).reshape(-1, 8).astype(np.float64)
    g = np.ones(N) if gain is None else gain.view(np.float16).astype(np.float64)
    om = np.ones(K) if cw is None else np.asarray(cw, np.float64)
    wv = (W.astype(np.float64) ** 2 * om).reshape(N, -1, 8).sum(-1)
    nb = (B[None, :, :] ** 2 * om.reshape(-1, 8)[:, None, :]).sum(-1).max(axis=1)   # [G]
    return 2.0 ** -18 * (wv + (g ** 2)[:, None] * nb[None, :]) + 1e-30


@pytest.mark.parametrize("gains", [False, True])
def test_exact_codewords_come_back(gains):
    cfg = synth.get_cfg("tiny_mxfp4", fmt="vq13", gains=gains, H=512, I=256, E=1, k=1, T=1)
    L = synth.gen_layer(cfg, seed=101)
    W = oracle.dequant(L, 0, 0)[:200]          # 200 rows: a ragged 128-row block
    i13, _ = _encode(W, L.book13, gain=None if not gains else L.gain[0][0][:200])
    assert np.array_equal(i13, L.idx13[0][0][:200])


@pytest.mark.parametrize("r8,gains,weighted", [(False, False, False), (True, True, True), (True, False, False)])
def test_random_weights_against_the_oracle(r8, gains, weighted):
    rng = np.random.default_rng(102)
    cfg = synth.get_cfg("tiny_mxfp4", fmt="vq13r8" if r8 else "vq13", gains=gains, H=256, I=128, E=1, k=1, T=1)
    L = synth.gen_layer(cfg, seed=102)
    N, K = 72, 256          # 72 rows: a ragged 128-row block
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    gain = L.gain[0][0][:N] if gains else None
    cw = rng.uniform(0.02, 1.0, size=K) ** 0.75 if weighted else None
    i13b, i8 = _encode(W, L.book13, L.book8 if r8 else None, gain, cw)
    G = K // 8
    i13 = _unpack(i13b, G)
    o13, o8, e13, e = encode_rows(W, L.book13, L.book8 if r8 else None, gain, cw)
    eps = _bound(W, L.book13, gain, cw)
    # base stage: optimal within the bound, equal where the decision is clear
    got13 = assignment_errors(W, L.book13, i13, gain=gain, col_weight=cw)
    assert (got13 <= e13 + eps).all()
    clear = second_best_base_errors(W, L.book13, gain, cw) - e13 > 2 * eps
    assert clear.mean() > 0.9
    assert np.array_equal(i13[clear], o13[clear])
    if r8:
        # residual stage, for the kernel's own base choice: optimal within the bound
        _, e_for_kernel_base = residual_stage(W, L.book13, i13, L.book8, gain, cw)
        got = assignment_errors(W, L.book13, i13, L.book8, i8, gain, cw)
        assert (got <= e_for_kernel_base + eps).all()
        same = clear & (i13 == o13)
        assert (i8[same] == o8[same]).mean() > 0.97
        # the 13-bit stream does not depend on the residual stage
        j13b, _ = _encode(W, L.book13, None, gain, cw)
        assert np.array_equal(j13b, i13b)
    assert np.array_equal(pack_idx13(i13), i13b)


def test_mimo_sized_matrix_sampled_rows():
    # a 2048 x 4096 gate matrix of codebook-like weights: the kernel's rows
    # against the oracle on a sample of rows
    cfg = synth.get_cfg("decode_vq")
    L = synth.gen_layer(cfg.replace(E=1), seed=103)
    rng = np.random.default_rng(103)
    W = (oracle.dequant(L, 0, 0) + rng.normal(0, 0.004, size=(2048, 4096))).astype(np.float32)
    i13b, i8 = _encode(W, L.book13, L.book8)
    rows = np.array([0, 1, 777, 1500, 2047])
    i13 = _unpack(i13b[rows], 512)
    o13, o8, e13, _ = encode_rows(W[rows], L.book13, L.book8)
    eps = _bound(W[rows], L.book13, None, None)
    got13 = assignment_errors(W[rows], L.book13, i13)
    assert (got13 <= e13 + eps).all()
    clear = second_best_base_errors(W[rows], L.book13) - e13 > 2 * eps
    assert np.array_equal(i13[clear], o13[clear])
    same = clear & (i13 == o13)
    assert (i8[rows][same] == o8[same]).mean() > 0.97
