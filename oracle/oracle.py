"""ctypes front end of ``moe_oracle.c`` (argument marshalling only).

TEST INFRASTRUCTURE ONLY: used by tests, the package smoke check and the
benchmark's CPU-baseline leg.  It shares no code with the CUDA library.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_FMT = {"mxfp4": 0, "vq13": 1, "vq13r8": 2, "gvq1": 3, "gvq1r8": 4}


class _Layer(C.Structure):
    _fields_ = [
        ("H", C.c_int32), ("I", C.c_int32), ("E", C.c_int32), ("k", C.c_int32), ("fmt", C.c_int32),
        ("codes", C.c_void_p * 3), ("scales", C.c_void_p * 3), ("idx13", C.c_void_p * 3),
        ("idx8", C.c_void_p * 3), ("gain", C.c_void_p * 3),
        ("book13", C.c_void_p), ("book8", C.c_void_p),
        ("code12", C.c_void_p * 3), ("hi1", C.c_void_p * 3), ("gbook13", C.c_void_p), ("gbook8", C.c_void_p),
        ("gscale13", C.c_float), ("gscale8", C.c_float),
    ]


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (skipped when it is newer than the source)."""
    with _lock:
        if (not force and os.path.exists(_SO)
                and os.path.getmtime(_SO) >= os.path.getmtime(_SRC)):
            return _SO
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
            "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
        return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_SO)
        L.orc_e2m1.restype = C.c_double
        L.orc_e2m1.argtypes = [C.c_uint32]
        L.orc_e8m0.restype = C.c_double
        L.orc_e8m0.argtypes = [C.c_uint32]
        L.orc_bf16_to_f32.restype = C.c_float
        L.orc_bf16_to_f32.argtypes = [C.c_uint16]
        L.orc_f16_to_f64.restype = C.c_double
        L.orc_f16_to_f64.argtypes = [C.c_uint16]
        L.orc_idx13.restype = C.c_uint32
        L.orc_idx13.argtypes = [C.c_void_p, C.c_int64]
        L.orc_e4m3.restype = C.c_double
        L.orc_e4m3.argtypes = [C.c_uint32]
        L.orc_gvq1_idx.restype = C.c_uint32
        L.orc_gvq1_idx.argtypes = [C.c_void_p, C.c_void_p, C.c_int64]
        L.orc_dequant.restype = None
        L.orc_dequant.argtypes = [C.POINTER(_Layer), C.c_int, C.c_int, C.c_void_p]
        L.orc_forward.restype = C.c_int64
        L.orc_forward.argtypes = [C.POINTER(_Layer), C.c_void_p, C.c_void_p, C.c_void_p,
                                  C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]
        L.orc_num_threads.restype = C.c_int
        L.orc_route_bucket.restype = C.c_int64
        L.orc_route_bucket.argtypes = [C.c_void_p, C.c_int64, C.c_int32, C.c_void_p, C.c_void_p]
        _lib = L
    return _lib


def e2m1(code: int) -> float:
    return lib().orc_e2m1(code)


def e8m0(b: int) -> float:
    return lib().orc_e8m0(b)


def e4m3(b: int) -> float:
    return lib().orc_e4m3(b)


def gvq1_idx(code12_row: np.ndarray, hi_row: np.ndarray, j: int) -> int:
    c = np.ascontiguousarray(code12_row, dtype=np.uint8)
    h = np.ascontiguousarray(hi_row, dtype=np.uint8)
    return int(lib().orc_gvq1_idx(c.ctypes.data, h.ctypes.data, j))


def bf16_to_f32(bits: int) -> float:
    return lib().orc_bf16_to_f32(bits)


def f16_to_f64(bits: int) -> float:
    return lib().orc_f16_to_f64(bits)


def idx13(stream: np.ndarray, j: int) -> int:
    s = np.ascontiguousarray(stream, dtype=np.uint8)
    return int(lib().orc_idx13(s.ctypes.data, j))


def route_bucket(topk_ids, E: int):
    """(offsets int32 [E+1], perm int32 [n_valid], n_invalid) of the routes."""
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32).ravel()
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(len(ids), np.int32)
    bad = lib().orc_route_bucket(ids.ctypes.data, len(ids), E, offsets.ctypes.data, perm.ctypes.data)
    return offsets, perm[: offsets[E]].copy(), int(bad)


def num_threads() -> int:
    return int(lib().orc_num_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data


def _layer_struct(layer):
    """Build the C view of a ``synth.Layer`` (arrays must stay alive)."""
    cfg = layer.cfg
    keep = []

    def c(a, dt):
        if a is None:
            return None
        a = np.ascontiguousarray(a, dtype=dt)
        keep.append(a)
        return a.ctypes.data

    s = _Layer()
    s.H, s.I, s.E, s.k, s.fmt = cfg.H, cfg.I, cfg.E, cfg.k, _FMT[cfg.fmt]
    for p in range(3):
        s.codes[p] = c(layer.codes[p], np.uint8)
        s.scales[p] = c(layer.scales[p], np.uint8)
        s.idx13[p] = c(layer.idx13[p], np.uint8)
        s.idx8[p] = c(layer.idx8[p], np.uint8)
        s.gain[p] = c(layer.gain[p], np.uint16)
    s.book13 = c(layer.book13, np.uint16)
    s.book8 = c(layer.book8, np.uint16)
    for p in range(3):
        s.code12[p] = c(layer.code12[p], np.uint8)
        s.hi1[p] = c(layer.hi1[p], np.uint8)
    s.gbook13 = c(layer.gbook13, np.uint8)
    s.gbook8 = c(layer.gbook8, np.uint8)
    s.gscale13 = float(layer.gscale[0]) if layer.gscale is not None else 0.0
    s.gscale8 = float(layer.gscale[1]) if layer.gscale is not None else 0.0
    return s, keep


def dequant(layer, expert: int, proj: int) -> np.ndarray:
    """Projection ``proj`` of ``expert`` as float32 [N][K] (the exact f32
    weights; the bit-exact contract of the library's dequant)."""
    cfg = layer.cfg
    N, K = cfg.shape(proj)
    out = np.empty((N, K), np.float32)
    s, keep = _layer_struct(layer)
    lib().orc_dequant(C.byref(s), expert, proj, out.ctypes.data)
    del keep
    return out


def _x_f64(layer, x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.uint16:   # bf16 bit patterns: exact widening
        x = (x.astype(np.uint32) << 16).view(np.float32)
    return np.ascontiguousarray(x, dtype=np.float64)


def forward(layer, x, topk_ids, topk_w, tokens=None, want_h=False, want_counts=False):
    """f64 layer output for the requested tokens (all when ``tokens`` is None).

    Returns ``out`` [n][H] float64, plus, when asked, ``h`` [n][k][I]
    float64 and ``counts`` (routes applied per projection), and always the
    number of invalid route ids as the last element."""
    cfg = layer.cfg
    xf = _x_f64(layer, x)
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    w = np.ascontiguousarray(topk_w, dtype=np.float32)
    T = ids.shape[0]
    assert ids.shape == (T, cfg.k) and w.shape == (T, cfg.k) and xf.shape[0] == T
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    n = T if tok is None else len(tok)
    out = np.empty((n, cfg.H), np.float64)
    h = np.empty((n, cfg.k, cfg.I), np.float64) if want_h else None
    counts = np.zeros(3, np.int64)
    s, keep = _layer_struct(layer)
    invalid = lib().orc_forward(C.byref(s), xf.ctypes.data, ids.ctypes.data, w.ctypes.data,
                                _ptr(tok), n, out.ctypes.data, counts.ctypes.data, _ptr(h))
    del keep
    res = [out]
    if want_h:
        res.append(h)
    if want_counts:
        res.append(counts)
    res.append(int(invalid))
    return tuple(res)


def _silu64(z):
    # silu(z) = z / (1 + e^-z); for very negative z, e^-z overflows to +inf
    # and the quotient is -0 (as in the C restatement), never NaN
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def forward_by_expert(layer, x, topk_ids, topk_w, tokens=None):
    """The layer output of ``forward`` computed expert by expert, for
    micro-batches the per-route C loop takes minutes on (a 2048-token layer).

    Same definition ("MiMo-V2.6-Flash-RL GGUF for a single DGX Spark",
    "Architecture notes": k routed experts per token, gate/up/down experts;
    "MiMo-V2.6-Flash-RL UNCENSORED VQ GGUF", "Recipe": the weight formats):
    for every expert e with routes, its three matrices are dequantised once
    to their exact f32 values by ``dequant`` (the C restatement), widened to
    f64, and applied to all of e's routed tokens with numpy f64 matrix
    products (the library matmul is the step; nothing is fused):
        G = X_e W_gate,e^T,  U = X_e W_up,e^T,  Hh = silu(G) * U,
        Y = Hh W_down,e^T,   out[t] += w[t][s] * Y[route (t, s)].
    Routes are added slot by slot in slot order.  Ids of -1 are no route;
    other ids outside [0, E) are skipped and counted (among the requested
    tokens).

    Returns (out [n][H] float64, number of invalid ids)."""
    cfg = layer.cfg
    xf = _x_f64(layer, x)
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    w = np.ascontiguousarray(topk_w, dtype=np.float32).astype(np.float64)
    T, k = ids.shape
    assert k == cfg.k and w.shape == ids.shape and xf.shape == (T, cfg.H)
    if tokens is None:
        tok = np.arange(T)
    else:
        tok = np.asarray(tokens, dtype=np.int64)
    row_of = np.full(T, -1, np.int64)          # output row of each requested token
    row_of[tok] = np.arange(len(tok))
    out = np.zeros((len(tok), cfg.H), np.float64)
    invalid = int(((ids[tok] != -1) & ((ids[tok] < 0) | (ids[tok] >= cfg.E))).sum())
    sel = (ids >= 0) & (ids < cfg.E) & (row_of[:, None] >= 0)
    for e in np.unique(ids[sel]):
        t_idx, s_idx = np.nonzero(sel & (ids == e))
        Wg = dequant(layer, int(e), 0).astype(np.float64)
        Wu = dequant(layer, int(e), 1).astype(np.float64)
        Wd = dequant(layer, int(e), 2).astype(np.float64)
        X = xf[t_idx]
        Hh = _silu64(X @ Wg.T) * (X @ Wu.T)
        Y = Hh @ Wd.T
        for s in np.unique(s_idx):
            m = s_idx == s           # one route per token in a slot: rows are distinct
            out[row_of[t_idx[m]]] += w[t_idx[m], s][:, None] * Y[m]
    return out, invalid
