"""Seeded generators for every workload of the compressed-expert MoE layer.

Recipe (all draws come from numpy's PCG64 through ``SeedSequence(seed,
spawn_key=(component,))``, so each array is fixed by the seed and its
component number alone, whatever else is drawn):

* component 0  -- routing: ``topk_ids`` int32 [T][k] and ``topk_w`` f32 [T][k]
  - "uniform": per token, E logits ~ N(0,1); the k largest (ties: lower
    expert id first) in descending order; weights = softmax over those k
    logits (computed in float64, stored as float32).
  - "zipf": experts listed in ``unrouted`` are never drawn; the others get
    a seeded random rank r = 1..E-len(unrouted) and popularity
    p ~ r**-s; per token k distinct experts by Gumbel-top-k on log p;
    weights = softmax of k fresh N(0,1) logits.
* component 1  -- activations x [T][H] ~ N(0, sigma^2) in float32, then
  rounded to bf16 (round-to-nearest-even, by torch) when act == "bf16".
* component 2  -- base codebook [8192][8] bf16 ~ N(0, book13_sigma^2),
  then multiplied by ``book13_mult`` (a power of two, so exact in bf16).
* component 3  -- residual codebook [256][8] bf16 ~ N(0, book8_sigma^2).
* component 10+p -- projection p's packed codes: MXFP4 nibbles or the
  13-bit index stream, as uniform random bytes (every nibble / every
  13-bit field is then uniform over its range).
* component 20+p -- projection p's E8M0 scale bytes, uniform over
  127+scale_exp[0] .. 127+scale_exp[1], or its 8-bit residual indices as
  uniform random bytes.
* component 30+p -- projection p's optional f16 row gains, uniform in
  [0.5, 2) rounded to f16.
* component 40  -- router matrix Wr [E][H] float32 ~ N(0, 1/H), so that with
  N(0,1) activations the router logits are about N(0,1).
* GVQ1 layers ("gvq1" / "gvq1r8"): the base and residual books are N(0,1)
  draws (components 2 and 3) rounded to E4M3 bytes (by torch), with book
  scales book13_sigma * book13_mult and book8_sigma; component 10+p gives
  the 12-bit code stream as uniform random bytes, component 50+p the bit-12
  plane, component 20+p the residual indices.

Projections are p = 0 gate [I][H], 1 up [I][H], 2 down [H][I]; rows are
output features and K (the reduction axis) is contiguous.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

GATE, UP, DOWN = 0, 1, 2
PROJ_NAMES = ("gate", "up", "down")
BOOK13_ROWS = 8192
BOOK8_ROWS = 256
VEC = 8          # weights per VQ index
MX_BLOCK = 32    # weights per E8M0 scale


@dataclass(frozen=True)
class LayerCfg:
    name: str
    H: int                      # hidden size
    I: int                      # expert intermediate size
    E: int                      # experts
    k: int                      # routes per token
    T: int                      # tokens
    fmt: str                    # "mxfp4" | "vq13" | "vq13r8"
    act: str                    # "f32" | "bf16"
    scale_exp: tuple = (-9, -5)  # E8M0 exponent range (MXFP4)
    x_sigma: float = 1.0
    routing: str = "uniform"    # "uniform" | "zipf"
    zipf_s: float = 1.1
    unrouted: tuple = ()
    book13_sigma: float = 0.02
    book8_sigma: float = 0.005
    book13_mult: float = 1.0
    gains: bool = False

    def shape(self, p: int) -> tuple:
        """(N, K) of projection p."""
        return (self.I, self.H) if p in (GATE, UP) else (self.H, self.I)

    def replace(self, **kw) -> "LayerCfg":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    # Tiny MXFP4 layer, f32 activations, scales 2^-8..2^-4.
    "tiny_mxfp4": LayerCfg("tiny_mxfp4", H=256, I=128, E=16, k=2, T=4,
                           fmt="mxfp4", act="f32", scale_exp=(-8, -4)),
    # MiMo-shaped layer, one decode token, MXFP4, scales 2^-9..2^-5.
    "decode_mxfp4": LayerCfg("decode_mxfp4", H=4096, I=2048, E=256, k=8, T=1,
                             fmt="mxfp4", act="bf16"),
    # MiMo-shaped layer, decode with 1/4/8 tokens, VQ13 with the residual on.
    "decode_vq": LayerCfg("decode_vq", H=4096, I=2048, E=256, k=8, T=1,
                          fmt="vq13r8", act="bf16"),
    # Prefill micro-batch of 2048, MXFP4, Zipf(1.1) popularity, two
    # experts never routed.
    "prefill_mxfp4_zipf": LayerCfg("prefill_mxfp4_zipf", H=4096, I=2048,
                                   E=256, k=8, T=2048, fmt="mxfp4",
                                   act="bf16", routing="zipf",
                                   unrouted=(13, 184)),
    # Prefill micro-batch of 2048, VQ13+R8, base book x64, x ~ N(0, 2^2).
    "prefill_vq_overflow": LayerCfg("prefill_vq_overflow", H=4096, I=2048,
                                    E=256, k=8, T=2048, fmt="vq13r8",
                                    act="bf16", x_sigma=2.0,
                                    book13_mult=64.0),
}


def get_cfg(name: str, **overrides) -> LayerCfg:
    return CONFIGS[name].replace(**overrides) if overrides else CONFIGS[name]


def _rng(seed: int, component: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(component,)))


def _random_bytes(rng: np.random.Generator, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return np.frombuffer(rng.bytes(n), dtype=np.uint8).reshape(shape).copy()


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round-to-nearest-even via torch."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact: a bf16 is the top half of an f32)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _f16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def e4m3_bytes_from_f32(a: np.ndarray) -> np.ndarray:
    """float -> E4M3 bytes (uint8), round-to-nearest-even via torch's float8_e4m3fn."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy().copy()


def gvq1_code_row_bytes(K: int) -> int:
    """Bytes of one row's GVQ1 12-bit code stream: K/8 codes of 12 bits."""
    assert K % 64 == 0
    return (K // VEC) * 12 // 8


def idx13_row_bytes(K: int) -> int:
    """Bytes of one row's 13-bit index stream: K/8 indices of 13 bits."""
    assert K % 64 == 0, "K must be a multiple of 64 for whole bytes per row"
    return (K // VEC) * 13 // 8


@dataclass
class Layer:
    """Host copy of one layer's compressed expert weights (logical layout)."""
    cfg: LayerCfg
    codes: list = field(default_factory=lambda: [None] * 3)    # MXFP4 [E][N][K/2]
    scales: list = field(default_factory=lambda: [None] * 3)   # MXFP4 [E][N][K/32]
    idx13: list = field(default_factory=lambda: [None] * 3)    # VQ [E][N][K*13/64]
    idx8: list = field(default_factory=lambda: [None] * 3)     # VQ [E][N][K/8]
    book13: Optional[np.ndarray] = None                          # uint16 [8192][8]
    book8: Optional[np.ndarray] = None                           # uint16 [256][8]
    gain: list = field(default_factory=lambda: [None] * 3)     # uint16 f16 [E][N]
    code12: list = field(default_factory=lambda: [None] * 3)   # GVQ1 12-bit streams [E][N][K*3/16]
    hi1: list = field(default_factory=lambda: [None] * 3)      # GVQ1 bit-12 planes [E][N][K/64]
    gbook13: Optional[np.ndarray] = None                         # uint8 e4m3 [8192][8]
    gbook8: Optional[np.ndarray] = None                          # uint8 e4m3 [256][8]
    gscale: Optional[tuple] = None                               # (scale of gbook13, scale of gbook8) f32

    @property
    def fmt(self) -> str:
        return self.cfg.fmt

    def without_residual(self) -> "Layer":
        """The same layer with the residual stage switched off (the base
        stage arrays are shared, byte for byte)."""
        if self.cfg.fmt.startswith("gvq1"):
            return Layer(cfg=self.cfg.replace(fmt="gvq1"), code12=list(self.code12), hi1=list(self.hi1),
                         gbook13=self.gbook13, gscale=self.gscale, gain=list(self.gain))
        return Layer(cfg=self.cfg.replace(fmt="vq13"), idx13=list(self.idx13),
                     book13=self.book13, gain=list(self.gain))

    def weight_bytes_per_expert(self) -> int:
        tot = 0
        for p in range(3):
            for arr in (self.codes[p], self.scales[p], self.idx13[p], self.idx8[p], self.gain[p], self.code12[p],
                        self.hi1[p]):
                if arr is not None:
                    tot += arr[0].nbytes
        return tot


def gen_layer(cfg: LayerCfg, seed: int = 0, experts: Optional[range] = None) -> Layer:
    """Draw a layer's compressed weights.  ``experts`` is ignored for the
    draw itself (all E experts are always drawn, so a sub-range never
    changes the bytes); it exists so callers can document intent."""
    L = Layer(cfg=cfg)
    E = cfg.E
    if cfg.fmt == "mxfp4":
        lo, hi = 127 + cfg.scale_exp[0], 127 + cfg.scale_exp[1]
        for p in range(3):
            N, K = cfg.shape(p)
            assert K % MX_BLOCK == 0
            L.codes[p] = _random_bytes(_rng(seed, 10 + p), (E, N, K // 2))
            L.scales[p] = _rng(seed, 20 + p).integers(lo, hi + 1, size=(E, N, K // MX_BLOCK),
                                                      dtype=np.uint8)
    elif cfg.fmt in ("vq13", "vq13r8"):
        b13 = _rng(seed, 2).normal(0.0, cfg.book13_sigma, size=(BOOK13_ROWS, VEC)).astype(np.float32)
        b13 = f32_from_bf16_bits(bf16_bits_from_f32(b13)) * np.float32(cfg.book13_mult)
        L.book13 = bf16_bits_from_f32(b13)
        for p in range(3):
            N, K = cfg.shape(p)
            L.idx13[p] = _random_bytes(_rng(seed, 10 + p), (E, N, idx13_row_bytes(K)))
        if cfg.fmt == "vq13r8":
            b8 = _rng(seed, 3).normal(0.0, cfg.book8_sigma, size=(BOOK8_ROWS, VEC)).astype(np.float32)
            L.book8 = bf16_bits_from_f32(b8)
            for p in range(3):
                N, K = cfg.shape(p)
                L.idx8[p] = _random_bytes(_rng(seed, 20 + p), (E, N, K // VEC))
    elif cfg.fmt in ("gvq1", "gvq1r8"):
        L.gbook13 = e4m3_bytes_from_f32(_rng(seed, 2).normal(0.0, 1.0, size=(BOOK13_ROWS, VEC)))
        s8 = 0.0
        for p in range(3):
            N, K = cfg.shape(p)
            L.code12[p] = _random_bytes(_rng(seed, 10 + p), (E, N, gvq1_code_row_bytes(K)))
            L.hi1[p] = _random_bytes(_rng(seed, 50 + p), (E, N, K // 64))
        if cfg.fmt == "gvq1r8":
            L.gbook8 = e4m3_bytes_from_f32(_rng(seed, 3).normal(0.0, 1.0, size=(BOOK8_ROWS, VEC)))
            s8 = cfg.book8_sigma
            for p in range(3):
                N, K = cfg.shape(p)
                L.idx8[p] = _random_bytes(_rng(seed, 20 + p), (E, N, K // VEC))
        L.gscale = (float(np.float32(cfg.book13_sigma * cfg.book13_mult)), float(np.float32(s8)))
    else:
        raise ValueError(cfg.fmt)
    if cfg.gains:
        for p in range(3):
            N, _ = cfg.shape(p)
            g = _rng(seed, 30 + p).uniform(0.5, 2.0, size=(E, N)).astype(np.float32)
            L.gain[p] = _f16_bits_from_f32(g)
    return L


def _softmax64(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.float64)
    z = z - z.max(axis=-1, keepdims=True)
    ez = np.exp(z)
    return (ez / ez.sum(axis=-1, keepdims=True)).astype(np.float32)


def _topk_desc(v: np.ndarray, k: int) -> np.ndarray:
    # stable sort of -v: equal values keep ascending expert id
    return np.argsort(-v, axis=-1, kind="stable")[..., :k]


def gen_routing(cfg: LayerCfg, seed: int = 0, T: Optional[int] = None):
    """(topk_ids int32 [T][k], topk_w float32 [T][k]) for the config."""
    T = cfg.T if T is None else T
    rng = _rng(seed, 0)
    if cfg.routing == "uniform":
        logits = rng.normal(0.0, 1.0, size=(T, cfg.E))
        ids = _topk_desc(logits, cfg.k)
        w = _softmax64(np.take_along_axis(logits, ids, axis=-1))
    elif cfg.routing == "zipf":
        routed = np.array([e for e in range(cfg.E) if e not in cfg.unrouted])
        ranks = rng.permutation(len(routed)) + 1
        logp = np.full(cfg.E, -np.inf)
        logp[routed] = -cfg.zipf_s * np.log(ranks.astype(np.float64))
        gumbel = rng.gumbel(size=(T, cfg.E))
        ids = _topk_desc(logp[None, :] + gumbel, cfg.k)
        w = _softmax64(rng.normal(0.0, 1.0, size=(T, cfg.k)))
    else:
        raise ValueError(cfg.routing)
    return ids.astype(np.int32), w.astype(np.float32)


def gen_disjoint_routing_schedule(cfg: LayerCfg, n_steps: int, seed: int = 0):
    """Routings for ``n_steps`` consecutive single-token decode steps in which
    consecutive steps share no expert: a seeded permutation of the experts is
    cut into E//k disjoint sets of k, used round-robin (step i takes set
    i mod E//k), so an expert's weights come back only after E//k - 1 other
    sets have streamed through.  Each set is a uniform random k-subset.  The
    weights are the softmax of the top-k of E fresh N(0,1) logits per step.
    Returns ids int32 [n_steps][T][k] and w float32 [n_steps][T][k]."""
    assert cfg.T == 1
    rng = _rng(seed, 4)
    perm = rng.permutation(cfg.E)
    n_sets = cfg.E // cfg.k
    sets = perm[: n_sets * cfg.k].reshape(n_sets, cfg.k)
    ids = np.empty((n_steps, 1, cfg.k), np.int32)
    w = np.empty((n_steps, 1, cfg.k), np.float32)
    for i in range(n_steps):
        logits = rng.normal(0.0, 1.0, size=cfg.E)
        top = np.sort(logits)[::-1][: cfg.k]
        ids[i, 0] = sets[i % n_sets]
        w[i, 0] = _softmax64(top)
    return ids, w


def gen_router(cfg: LayerCfg, seed: int = 0) -> np.ndarray:
    """Router matrix Wr float32 [E][H] (component 40)."""
    return _rng(seed, 40).normal(0.0, 1.0 / np.sqrt(cfg.H), size=(cfg.E, cfg.H)).astype(np.float32)


def gen_activations(cfg: LayerCfg, seed: int = 0, T: Optional[int] = None) -> np.ndarray:
    """x [T][H]: float32 for act f32, bf16 bit patterns (uint16) for act bf16."""
    T = cfg.T if T is None else T
    x = _rng(seed, 1).normal(0.0, cfg.x_sigma, size=(T, cfg.H)).astype(np.float32)
    return x if cfg.act == "f32" else bf16_bits_from_f32(x)
