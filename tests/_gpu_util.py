"""Helpers shared by the GPU parity tests: upload a synthetic layer through
the C ABI, run it, and compare with the oracle under the stated tolerance."""
import numpy as np

import oracle
import synth

# max_m |out[t][m] - ref[t][m]| / ||ref[t]||_2 per token
TOL = {"f32": 1e-5, "bf16": 2e-3}


def torch_mod():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("GPU tests need a CUDA device")
    return torch


def dev_layer(L, max_tokens=None):
    """Create + upload a libmoeq layer holding the synthetic layer L."""
    from bit_quantized_moe_routed_b200 import moeq
    cfg = L.cfg
    lay = moeq.Layer(cfg.H, cfg.I, cfg.E, cfg.k, max_tokens or cfg.T, cfg.fmt, cfg.act, device=0)
    lay.upload(L)
    return lay


def to_dev_inputs(cfg, x, ids, w):
    torch = torch_mod()
    if cfg.act == "bf16":
        xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        xt = torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    return xt, torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda(), \
        torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda()


def out_to_f64(out):
    torch = torch_mod()
    return out.float().cpu().numpy().astype(np.float64) if out.dtype == torch.bfloat16 \
        else out.cpu().numpy().astype(np.float64)


def run(lay, cfg, x, ids, w):
    torch = torch_mod()
    xt, it, wt = to_dev_inputs(cfg, x, ids, w)
    out = lay.forward(xt, it, wt)
    torch.cuda.synchronize()
    return out_to_f64(out)


def rel_err_per_token(out, ref):
    """max_m |out - ref| / ||ref||_2 per row; rows with ||ref|| = 0 give 0 if
    out is exactly 0 there, else inf."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    nrm = np.linalg.norm(ref, axis=1)
    err = np.abs(out - ref).max(axis=1)
    res = np.where(nrm > 0, err / np.where(nrm > 0, nrm, 1.0), np.where(err == 0, 0.0, np.inf))
    return res


def assert_close(out, ref, act, what=""):
    r = rel_err_per_token(out, ref)
    tol = TOL[act]
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    assert r.max() <= tol, f"{what}: max rel err {r.max():.3e} > {tol:.0e} (token {int(r.argmax())})"
    return float(r.max())


def oracle_ref(L, x, ids, w, tokens=None):
    out, _ = oracle.forward(L, x, ids, w, tokens=tokens)
    return out


def sample_tokens(T, n, seed=0):
    """n distinct tokens including the first and last."""
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, T - 1), size=max(0, min(n, T) - 2), replace=False)
    return np.unique(np.concatenate([[0, T - 1], mid])).astype(np.int32)


__all__ = ["TOL", "torch_mod", "dev_layer", "to_dev_inputs", "out_to_f64", "run", "rel_err_per_token",
           "assert_close", "oracle_ref", "sample_tokens", "synth", "oracle"]
