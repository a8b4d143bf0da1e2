"""VQ encoder: nearest-codeword assignment of 8-weight vectors to the layer's
13-bit base book, then of the remainder to the 8-bit residual book.

TEST INFRASTRUCTURE ONLY: a plain float64 brute force for the tests and the
benchmark's CPU baseline; the CUDA library never calls it.

Source ("MiMo-V2.6-Flash-RL UNCENSORED VQ GGUF", "Recipe"): each 8-weight
vector of an expert row is replaced by the index of a codebook entry, the
row scaled by an f16 gain; a second, 256-entry book encodes the remainder
the first stage leaves, without changing the first stage's indices; the
page's whole procedure (books, assignment, gains) minimises an error
weighted per column by importance.  Only
the assignment is restated here (the codebooks and gains are inputs; their
training needs calibration data and is not part of this path).  Readings:
  - the error of a candidate is sum_i omega_i (w_i - v_i)^2 over the vector's
    8 columns, where v is exactly the weight the format decodes for that
    candidate: v_i = f32(f32(B13[c][i]) * g) for the base stage and
    v_i = f32(f32(B13[c][i] + R8[r][i]) * g) with the residual, g the row's
    f16 gain (1 when absent), every operation f32 round-to-nearest-even;
  - the base index is chosen first, on the base-stage error alone (so the
    13-bit stream does not depend on the residual stage), then the residual
    index for that base index;
  - ties go to the lowest index; omega defaults to 1 for every column;
  - indices are packed as the format stores them: the 13-bit indices of a
    row as one little-endian bitstream (index j = bits 13j..13j+12), the
    residual indices one byte each.
"""
from __future__ import annotations

import numpy as np


def _bf16_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _f16_to_f32(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float32)


def _argmin_first(d):
    """Index of the smallest value along the last axis, lowest index on ties."""
    return np.argmin(d, axis=-1)   # numpy returns the first occurrence


def encode_rows(w, book13, book8=None, gain=None, col_weight=None, chunk=256):
    """Assign every 8-vector of w (float32 [N][K], K a multiple of 64).

    book13 uint16 bf16 [8192][8]; book8 uint16 bf16 [256][8] or None;
    gain uint16 f16 [N] or None; col_weight float [K] or None.
    Returns (idx13 int32 [N][K/8], idx8 int32 [N][K/8] or None,
    err13 float64 [N][K/8], err float64 [N][K/8]) -- the weighted squared
    errors of each vector after the base stage and after the last stage."""
    w = np.asarray(w, np.float32)
    N, K = w.shape
    assert K % 64 == 0
    G = K // 8
    B = _bf16_to_f32(book13).reshape(-1, 8)                    # [8192][8] f32
    R = None if book8 is None else _bf16_to_f32(book8).reshape(-1, 8)
    g = np.ones(N, np.float32) if gain is None else _f16_to_f32(gain)
    om = np.ones(K, np.float64) if col_weight is None else np.asarray(col_weight, np.float64)
    idx13 = np.empty((N, G), np.int32)
    idx8 = None if R is None else np.empty((N, G), np.int32)
    err13 = np.empty((N, G), np.float64)
    err = np.empty((N, G), np.float64)
    for n in range(N):
        V13 = (B * g[n]).astype(np.float32).astype(np.float64)   # decoded base candidates [8192][8]
        for j0 in range(0, G, chunk):
            j1 = min(G, j0 + chunk)
            wv = w[n, 8 * j0:8 * j1].reshape(-1, 8).astype(np.float64)     # [g][8]
            ov = om[8 * j0:8 * j1].reshape(-1, 8)                            # [g][8]
            d = (((wv[:, None, :] - V13[None, :, :]) ** 2) * ov[:, None, :]).sum(-1)   # [g][8192]
            c = _argmin_first(d)
            idx13[n, j0:j1] = c
            err13[n, j0:j1] = d[np.arange(j1 - j0), c]
            if R is None:
                err[n, j0:j1] = err13[n, j0:j1]
                continue
            # residual candidates for each vector's chosen base entry
            S = (B[c][:, None, :] + R[None, :, :]).astype(np.float32)        # [g][256][8] f32 sums
            VR = (S * g[n]).astype(np.float32).astype(np.float64)
            dr = (((wv[:, None, :] - VR) ** 2) * ov[:, None, :]).sum(-1)    # [g][256]
            r = _argmin_first(dr)
            idx8[n, j0:j1] = r
            err[n, j0:j1] = dr[np.arange(j1 - j0), r]
    return idx13, idx8, err13, err


def residual_stage(w, book13, idx13, book8, gain=None, col_weight=None):
    """The residual stage alone, for a given base assignment idx13 [N][K/8]:
    (idx8 int32 [N][K/8], err float64 [N][K/8]), as in encode_rows."""
    w = np.asarray(w, np.float32)
    N, K = w.shape
    G = K // 8
    B = _bf16_to_f32(book13).reshape(-1, 8)
    R = _bf16_to_f32(book8).reshape(-1, 8)
    g = np.ones(N, np.float32) if gain is None else _f16_to_f32(gain)
    om = np.ones(K, np.float64) if col_weight is None else np.asarray(col_weight, np.float64)
    idx8 = np.empty((N, G), np.int32)
    err = np.empty((N, G), np.float64)
    for n in range(N):
        S = (B[np.asarray(idx13[n])][:, None, :] + R[None, :, :]).astype(np.float32)   # [G][256][8]
        V = (S * g[n]).astype(np.float32).astype(np.float64)
        d = (((w[n].reshape(G, 1, 8).astype(np.float64) - V) ** 2) * om.reshape(G, 1, 8)).sum(-1)
        r = _argmin_first(d)
        idx8[n] = r
        err[n] = d[np.arange(G), r]
    return idx8, err


def assignment_errors(w, book13, idx13, book8=None, idx8=None, gain=None, col_weight=None):
    """The weighted squared error (float64 [N][K/8]) of a given assignment,
    with the same decoded values as encode_rows."""
    w = np.asarray(w, np.float32)
    N, K = w.shape
    B = _bf16_to_f32(book13).reshape(-1, 8)
    R = None if book8 is None else _bf16_to_f32(book8).reshape(-1, 8)
    g = np.ones(N, np.float32) if gain is None else _f16_to_f32(gain)
    om = np.ones(K, np.float64) if col_weight is None else np.asarray(col_weight, np.float64)
    S = B[np.asarray(idx13)]                                        # [N][G][8]
    if R is not None:
        S = (S + R[np.asarray(idx8)]).astype(np.float32)
    V = (S * g[:, None, None]).astype(np.float32).astype(np.float64)
    return (((w.reshape(N, -1, 8).astype(np.float64) - V) ** 2) * om.reshape(1, -1, 8)).sum(-1)


def second_best_base_errors(w, book13, gain=None, col_weight=None):
    """float64 [N][K/8]: the second smallest base-stage error of each vector
    (the margin of the base decision is this minus the smallest)."""
    w = np.asarray(w, np.float32)
    N, K = w.shape
    B = _bf16_to_f32(book13).reshape(-1, 8)
    g = np.ones(N, np.float32) if gain is None else _f16_to_f32(gain)
    om = np.ones(K, np.float64) if col_weight is None else np.asarray(col_weight, np.float64)
    out = np.empty((N, K // 8), np.float64)
    for n in range(N):
        V13 = (B * g[n]).astype(np.float32).astype(np.float64)
        wv = w[n].reshape(-1, 8).astype(np.float64)
        d = (((wv[:, None, :] - V13[None, :, :]) ** 2) * om.reshape(-1, 8)[:, None, :]).sum(-1)
        out[n] = np.partition(d, 1, axis=1)[:, 1]
    return out


def pack_idx13(idx13):
    """int [N][G] 13-bit indices -> uint8 [N][G*13/8] little-endian streams."""
    idx13 = np.asarray(idx13, np.int64)
    N, G = idx13.shape
    assert G % 8 == 0 and (idx13 >= 0).all() and (idx13 < 8192).all()
    out = np.zeros((N, G * 13 // 8), np.uint8)
    for j in range(G):
        for q in range(13):
            bit = (idx13[:, j] >> q) & 1
            p = 13 * j + q
            out[:, p >> 3] |= (bit << (p & 7)).astype(np.uint8)
    return out


def relative_mse(w, err):
    """Weighted squared error over the weights' energy: sum(err) / sum(w^2)."""
    return float(np.sum(err) / np.sum(np.asarray(w, np.float64) ** 2))
