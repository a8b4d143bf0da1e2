"""Python binding of libmoeq (ctypes; argument marshalling only).

Every step of the layer runs in the CUDA library; this module only turns
torch tensors / numpy arrays into pointers, sizes and the current CUDA
stream.  It raises at import time when ``libmoeq.so`` is missing: there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoeq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m bit_quantized_moe_routed_b200.build` "
        "(the layer has no non-CUDA implementation)")

_lib = C.CDLL(LIB_PATH)

OK, INVALID_ARGUMENT, UNSUPPORTED, OUT_OF_MEMORY, CUDA, NOT_UPLOADED, ROUTE_OUT_OF_RANGE, TIMEOUT = range(8)
FMT = {"mxfp4": 0, "vq13": 1, "vq13r8": 2, "gvq1": 3, "gvq1r8": 4}
ACT = {"f32": 0, "bf16": 1}
GATE, UP, DOWN = 0, 1, 2

# every symbol the header declares
EXPORTS = ("moeq_layer_create", "moeq_upload_weights", "moeq_forward", "moeq_forward_host",
           "moeq_forward_profiled", "moeq_route", "moeq_dequant", "moeq_layer_status",
           "moeq_status_string", "moeq_layer_destroy", "moeq_kernel_launches", "moeq_route_noalloc",
           "moeq_router_upload", "moeq_router", "moeq_forward_routed", "moeq_vq_encode")
SCORE = {"sigmoid": 0, "softmax": 1}


class LayerDesc(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("inter", C.c_int32), ("n_experts", C.c_int32),
                ("top_k", C.c_int32), ("max_tokens", C.c_int32), ("fmt", C.c_int32),
                ("act", C.c_int32), ("device", C.c_int32)]


class Weights(C.Structure):
    _fields_ = [("codes", C.c_void_p * 3), ("scales", C.c_void_p * 3), ("idx13", C.c_void_p * 3),
                ("idx8", C.c_void_p * 3), ("book13", C.c_void_p), ("book8", C.c_void_p),
                ("gain", C.c_void_p * 3), ("code12", C.c_void_p * 3), ("hi1", C.c_void_p * 3),
                ("gbook13", C.c_void_p), ("gbook8", C.c_void_p), ("gscale", C.c_float * 2)]


_lib.moeq_layer_create.argtypes = [C.POINTER(LayerDesc), C.POINTER(C.c_void_p)]
_lib.moeq_upload_weights.argtypes = [C.c_void_p, C.POINTER(Weights), C.c_void_p]
_lib.moeq_forward.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p]
_lib.moeq_forward_host.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p,
                                   C.c_void_p]
_lib.moeq_forward_profiled.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p,
                                       C.c_void_p, C.POINTER(C.c_void_p)]
_lib.moeq_route.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]
_lib.moeq_route_noalloc.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p]
_lib.moeq_dequant.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p]
_lib.moeq_router_upload.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p]
_lib.moeq_router.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
_lib.moeq_forward_routed.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_void_p]
_lib.moeq_vq_encode.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                C.c_void_p, C.c_void_p, C.c_void_p]
_lib.moeq_layer_status.argtypes = [C.c_void_p, C.c_int32]
_lib.moeq_status_string.argtypes = [C.c_int]
_lib.moeq_status_string.restype = C.c_char_p
_lib.moeq_layer_destroy.argtypes = [C.c_void_p]
_lib.moeq_layer_destroy.restype = None
_lib.moeq_kernel_launches.argtypes = [C.c_void_p]
_lib.moeq_kernel_launches.restype = C.c_int64
for _f in ("moeq_layer_create", "moeq_upload_weights", "moeq_forward", "moeq_forward_host", "moeq_dequant",
           "moeq_layer_status", "moeq_forward_profiled", "moeq_route", "moeq_route_noalloc",
           "moeq_router_upload", "moeq_router", "moeq_forward_routed", "moeq_vq_encode"):
    getattr(_lib, _f).restype = C.c_int


class MoeqError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


def status_string(code: int) -> str:
    return _lib.moeq_status_string(int(code)).decode()


def lib():
    return _lib


def _check(code: int, what: str):
    if code != OK:
        raise MoeqError(code, what)


def _stream_ptr(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _host(a, dtype):
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def route_noalloc(topk_ids, n_experts, offsets_out, perm_out, stream=None):
    """moeq_route_noalloc: the route/bucket step without a layer and without
    any device allocation.  topk_ids int32 cuda [T][k]; offsets_out int32
    cuda [n_experts+1] and perm_out int32 cuda [T*k] are the caller's and
    are filled as by Layer.route.  The library's fixed scratch is shared by
    every call on a device: calls that overlap on the GPU race."""
    T, k = topk_ids.shape
    _check(_lib.moeq_route_noalloc(C.c_void_p(topk_ids.data_ptr()), T, k, n_experts,
                                   C.c_void_p(offsets_out.data_ptr()), C.c_void_p(perm_out.data_ptr()),
                                   _stream_ptr(stream)), "moeq_route_noalloc")


def vq_encode(w, book13, book8=None, gain=None, col_weight=None, stream=None):
    """moeq_vq_encode on cuda tensors: w float32 [N][K]; book13 / book8
    bf16 bit patterns (int16 or uint16 tensors) [8192][8] / [256][8]; gain
    f16 bit patterns [N] or None; col_weight float32 [K] or None.  Returns
    (idx13 uint8 [N][K*13/64], idx8 uint8 [N][K/8] or None)."""
    import torch
    N, K = w.shape
    idx13 = torch.empty((N, K * 13 // 64), dtype=torch.uint8, device=w.device)
    idx8 = torch.empty((N, K // 8), dtype=torch.uint8, device=w.device) if book8 is not None else None

    def p(t):
        return C.c_void_p(t.data_ptr() if t is not None else 0)
    _check(_lib.moeq_vq_encode(p(w), N, K, p(gain), p(col_weight), p(book13), p(book8), p(idx13), p(idx8),
                               _stream_ptr(stream)), "moeq_vq_encode")
    return idx13, idx8


class Layer:
    """One compressed-expert MoE layer owned by libmoeq on one CUDA device."""

    def __init__(self, hidden, inter, n_experts, top_k, max_tokens, fmt="mxfp4", act="bf16", device=0):
        self.desc = LayerDesc(hidden, inter, n_experts, top_k, max_tokens, FMT[fmt], ACT[act], device)
        self.fmt, self.act, self.device = fmt, act, device
        self.H, self.I, self.E, self.k, self.max_tokens = hidden, inter, n_experts, top_k, max_tokens
        h = C.c_void_p()
        _check(_lib.moeq_layer_create(C.byref(self.desc), C.byref(h)), "moeq_layer_create")
        self._h = h

    @classmethod
    def for_cfg(cls, cfg, max_tokens=None, device=0):
        return cls(cfg.H, cfg.I, cfg.E, cfg.k, max_tokens or cfg.T, cfg.fmt, cfg.act, device)

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None) and self._h.value:
            _lib.moeq_layer_destroy(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def upload(self, w, stream=None):
        """``w``: host arrays with the attributes codes, scales, idx13, idx8,
        gain, code12, hi1 (per-projection lists), book13, book8 (bf16),
        gbook13, gbook8 (E4M3) and gscale, logical layout; missing
        attributes count as absent."""
        ws = Weights()
        keep = []
        for p in range(3):
            for name, dt in (("codes", np.uint8), ("scales", np.uint8), ("idx13", np.uint8),
                             ("idx8", np.uint8), ("gain", np.uint16), ("code12", np.uint8), ("hi1", np.uint8)):
                arrs = getattr(w, name, None)
                arr, ptr = _host(arrs[p] if arrs is not None else None, dt)
                keep.append(arr)
                getattr(ws, name)[p] = ptr
        for name, dt in (("book13", np.uint16), ("book8", np.uint16), ("gbook13", np.uint8), ("gbook8", np.uint8)):
            arr, ptr = _host(getattr(w, name, None), dt)
            keep.append(arr)
            setattr(ws, name, ptr)
        gs = getattr(w, "gscale", None)
        if gs is not None:
            ws.gscale[0], ws.gscale[1] = float(gs[0]), float(gs[1])
        _check(_lib.moeq_upload_weights(self._h, C.byref(ws), _stream_ptr(stream)), "moeq_upload_weights")
        del keep

    def forward(self, x, topk_ids, topk_w, out=None, stream=None):
        """x: cuda tensor [T][H] (float32 or bfloat16 per ``act``); topk_ids
        int32 [T][k]; topk_w float32 [T][k]; returns ``out`` [T][H]."""
        import torch
        T = x.shape[0]
        for t in (x, topk_ids, topk_w):
            assert t.is_cuda and t.is_contiguous()
        assert topk_ids.dtype == torch.int32 and topk_w.dtype == torch.float32
        if out is None:
            out = torch.empty_like(x)
        _check(_lib.moeq_forward(self._h, C.c_void_p(x.data_ptr()), C.c_void_p(topk_ids.data_ptr()),
                                 C.c_void_p(topk_w.data_ptr()), T, C.c_void_p(out.data_ptr()),
                                 _stream_ptr(stream)), "moeq_forward")
        return out

    def forward_profiled(self, x, topk_ids, topk_w, out, events, stream=None):
        """moeq_forward recording 5 torch.cuda.Event objects at its phase
        boundaries (before; after route; after gate/up; after down; end)."""
        assert len(events) == 5
        evs = (C.c_void_p * 5)(*[C.c_void_p(e.cuda_event) for e in events])
        _check(_lib.moeq_forward_profiled(self._h, C.c_void_p(x.data_ptr()), C.c_void_p(topk_ids.data_ptr()),
                                          C.c_void_p(topk_w.data_ptr()), x.shape[0], C.c_void_p(out.data_ptr()),
                                          _stream_ptr(stream), evs), "moeq_forward_profiled")
        return out

    def route(self, topk_ids, stream=None):
        """(offsets int32 [E+1], perm int32 [T*k]) cuda tensors; only the
        first offsets[E] entries of perm are defined."""
        import torch
        T = topk_ids.shape[0]
        offsets = torch.empty(self.E + 1, dtype=torch.int32, device=topk_ids.device)
        perm = torch.full((T * self.k,), -1, dtype=torch.int32, device=topk_ids.device)
        _check(_lib.moeq_route(self._h, C.c_void_p(topk_ids.data_ptr()), T, C.c_void_p(offsets.data_ptr()),
                               C.c_void_p(perm.data_ptr()), _stream_ptr(stream)), "moeq_route")
        return offsets, perm

    def forward_host(self, x, topk_ids, topk_w, out=None, stream=None):
        """Host (numpy / CPU tensor) buffers in and out; synchronous."""
        x = np.ascontiguousarray(x)
        ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
        w = np.ascontiguousarray(topk_w, dtype=np.float32)
        if out is None:
            out = np.empty_like(x)
        _check(_lib.moeq_forward_host(self._h, x.ctypes.data, ids.ctypes.data, w.ctypes.data, x.shape[0],
                                      out.ctypes.data, _stream_ptr(stream)), "moeq_forward_host")
        return out

    def forward_host_ptr(self, x_ptr, ids_ptr, w_ptr, T, out_ptr, stream=None):
        """moeq_forward_host on raw host pointers (pinned buffers)."""
        _check(_lib.moeq_forward_host(self._h, C.c_void_p(x_ptr), C.c_void_p(ids_ptr), C.c_void_p(w_ptr), T,
                                      C.c_void_p(out_ptr), _stream_ptr(stream)), "moeq_forward_host")

    def dequant(self, expert, proj, out=None, stream=None):
        import torch
        N, K = (self.I, self.H) if proj in (GATE, UP) else (self.H, self.I)
        if out is None:
            out = torch.empty((N, K), dtype=torch.float32, device=f"cuda:{self.device}")
        _check(_lib.moeq_dequant(self._h, expert, proj, C.c_void_p(out.data_ptr()), _stream_ptr(stream)),
               "moeq_dequant")
        return out

    def router_upload(self, wr, score="sigmoid", stream=None):
        """Router matrix ``wr``: host float32 [E][H]; ``score``: "sigmoid" or "softmax"."""
        wr = np.ascontiguousarray(wr, dtype=np.float32)
        assert wr.shape == (self.E, self.H)
        _check(_lib.moeq_router_upload(self._h, wr.ctypes.data, SCORE[score], _stream_ptr(stream)),
               "moeq_router_upload")

    def router(self, x, want_logits=False, stream=None):
        """(topk_ids int32 [T][k], topk_w float32 [T][k], logits float32 [T][E] or None), cuda tensors."""
        import torch
        assert x.is_cuda and x.is_contiguous()
        T = x.shape[0]
        ids = torch.empty((T, self.k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.k), dtype=torch.float32, device=x.device)
        z = torch.empty((T, self.E), dtype=torch.float32, device=x.device) if want_logits else None
        _check(_lib.moeq_router(self._h, C.c_void_p(x.data_ptr()), T, C.c_void_p(ids.data_ptr()),
                                C.c_void_p(w.data_ptr()), C.c_void_p(z.data_ptr() if z is not None else 0),
                                _stream_ptr(stream)), "moeq_router")
        return ids, w, z

    def forward_routed(self, x, out=None, stream=None):
        """Router + forward: (out [T][H], topk_ids [T][k], topk_w [T][k]), cuda tensors."""
        import torch
        assert x.is_cuda and x.is_contiguous()
        T = x.shape[0]
        ids = torch.empty((T, self.k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.k), dtype=torch.float32, device=x.device)
        if out is None:
            out = torch.empty_like(x)
        _check(_lib.moeq_forward_routed(self._h, C.c_void_p(x.data_ptr()), T, C.c_void_p(ids.data_ptr()),
                                        C.c_void_p(w.data_ptr()), C.c_void_p(out.data_ptr()), _stream_ptr(stream)),
               "moeq_forward_routed")
        return out, ids, w

    def kernel_launches(self) -> int:
        return int(_lib.moeq_kernel_launches(self._h))

    def status(self, clear=False) -> int:
        return int(_lib.moeq_layer_status(self._h, 1 if clear else 0))
