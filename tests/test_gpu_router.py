"""The router kernel (moeq_router) against the router oracle.

The logits must match the oracle's float64 logits within the f32 error bound
of a K = H sum; the selection is an integer decided by floating point, so it
is checked in the kernel's own precision -- the ids must be exactly the
oracle's selection applied to the kernel's f32 logits -- and against the
float64 selection wherever the oracle's margin between the k-th and the
(k+1)-th logit is larger than twice that bound.  The weights must match the
oracle's weighting of the kernel's logits."""
import numpy as np
import pytest

from _gpu_util import assert_close, dev_layer, oracle, synth, to_dev_inputs, torch_mod
from oracle.router import router_logits, topk_from_logits

pytestmark = pytest.mark.gpu


def _x64(cfg, x):
    return synth.f32_from_bf16_bits(x).astype(np.float64) if cfg.act == "bf16" else x.astype(np.float64)


def _check_router(cfg, x, wr, ids, w, z, score):
    xf = _x64(cfg, x)
    zref = router_logits(xf, wr)
    # |error| of an f32 sum of K exact products: <= K 2^-24 sum |x w|, and the
    # three bf16 terms of wr carry it to 2^-24 relative
    bound = (cfg.H * 2.0 ** -24 + 2.0 ** -22) * (np.abs(xf) @ np.abs(wr.astype(np.float64)).T) + 1e-30
    assert (np.abs(z.astype(np.float64) - zref) <= bound).all(), float((np.abs(z - zref) / bound).max())
    # the kernel's decisions on its own logits
    ids_k, w_k = topk_from_logits(z, cfg.k, score)
    assert np.array_equal(ids, ids_k)
    np.testing.assert_allclose(w, w_k, rtol=4e-6, atol=1e-7)
    # and the float64 decisions where they are unambiguous
    ids_o, _ = topk_from_logits(zref, cfg.k, score)
    zs = -np.sort(-zref, axis=1)
    margin = zs[:, cfg.k - 1] - zs[:, cfg.k]
    clear = margin > 2 * bound.max(axis=1)
    assert clear.mean() > 0.5
    assert np.array_equal(ids[clear], ids_o[clear])
    # the selected sets are always valid top-k sets under the float64 logits
    # up to the bound
    for t in range(cfg.T):
        sel = set(ids[t].tolist())
        worst_in = min(zref[t, e] for e in sel)
        best_out = max(zref[t, e] for e in range(cfg.E) if e not in sel)
        assert worst_in >= best_out - 2 * bound[t].max()


def _router_layer(cfg, score, seed):
    from bit_quantized_moe_routed_b200 import moeq
    lay = moeq.Layer(cfg.H, cfg.I, cfg.E, cfg.k, cfg.T, cfg.fmt, cfg.act)
    wr = synth.gen_router(cfg, seed=seed)
    lay.router_upload(wr, score)
    return lay, wr


@pytest.mark.parametrize("T", [1, 5, 8, 37, 300])
@pytest.mark.parametrize("score", ["sigmoid", "softmax"])
def test_router_mimo_shape(T, score):
    torch = torch_mod()
    cfg = synth.get_cfg("decode_mxfp4", T=T)         # H 4096, E 256, k 8, bf16
    lay, wr = _router_layer(cfg, score, seed=81 + T)
    x = synth.gen_activations(cfg, seed=81 + T)
    xt, _, _ = to_dev_inputs(cfg, x, np.zeros((T, cfg.k), np.int32), np.zeros((T, cfg.k), np.float32))
    n0 = lay.kernel_launches()
    ids, w, z = lay.router(xt, want_logits=True)
    torch.cuda.synchronize()
    assert lay.kernel_launches() - n0 == 1
    _check_router(cfg, x, wr, ids.cpu().numpy(), w.cpu().numpy(), z.cpu().numpy(), score)
    # a second call gives the same bits (fixed slice order, counters reset)
    ids2, w2, z2 = lay.router(xt, want_logits=True)
    torch.cuda.synchronize()
    assert torch.equal(ids, ids2) and torch.equal(w, w2) and torch.equal(z, z2)


def test_router_prefill_micro_batch():
    cfg = synth.get_cfg("prefill_mxfp4_zipf", T=2048)
    lay, wr = _router_layer(cfg.replace(routing="uniform"), "sigmoid", seed=90)
    x = synth.gen_activations(cfg, seed=90)
    xt, _, _ = to_dev_inputs(cfg, x, np.zeros((1, 8), np.int32), np.zeros((1, 8), np.float32))
    ids, w, z = lay.router(xt, want_logits=True)
    # logits and decisions on every 16th token (the float64 oracle loops in Python)
    sub = np.arange(0, cfg.T, 16)
    cs = cfg.replace(T=len(sub))
    _check_router(cs, x[sub], wr, ids.cpu().numpy()[sub], w.cpu().numpy()[sub], z.cpu().numpy()[sub], "sigmoid")
    # every token's decisions on its own logits
    ids_k, w_k = topk_from_logits(z.cpu().numpy(), cfg.k, "sigmoid")
    assert np.array_equal(ids.cpu().numpy(), ids_k)
    np.testing.assert_allclose(w.cpu().numpy(), w_k, rtol=4e-6, atol=1e-7)


@pytest.mark.parametrize("T", [5, 45])          # the GEMV (T <= 8) and the tiled path
@pytest.mark.parametrize("act", ["f32", "bf16"])
def test_router_small_and_ragged_expert_count(act, T):
    # E = 24 (not a whole number of 16-expert tiles), H = 256, k = 3
    cfg = synth.get_cfg("tiny_mxfp4", act=act, E=24, k=3, T=T)
    lay, wr = _router_layer(cfg, "sigmoid", seed=91)
    x = synth.gen_activations(cfg, seed=91)
    xt, _, _ = to_dev_inputs(cfg, x, np.zeros((1, 3), np.int32), np.zeros((1, 3), np.float32))
    ids, w, z = lay.router(xt, want_logits=True)
    _check_router(cfg, x, wr, ids.cpu().numpy(), w.cpu().numpy(), z.cpu().numpy(), "sigmoid")


@pytest.mark.parametrize("act", ["f32", "bf16"])
def test_router_all_ties_take_the_lowest_ids(act):
    torch = torch_mod()
    cfg = synth.get_cfg("tiny_mxfp4", act=act, E=40, k=5, T=3)
    lay, _ = _router_layer(cfg, "sigmoid", seed=92)
    x = torch.zeros((cfg.T, cfg.H), dtype=torch.float32 if act == "f32" else torch.bfloat16, device="cuda")
    ids, w, z = lay.router(x, want_logits=True)
    assert (ids.cpu().numpy() == np.arange(5)).all()
    assert (w.cpu().numpy() == np.float32(0.2)).all()
    assert not z.cpu().numpy().any()


def test_forward_routed_decode():
    # router + the decode kernels in one call; the layer part against the
    # oracle on the routing the router chose
    torch = torch_mod()
    cfg = synth.get_cfg("decode_mxfp4", H=2048, I=2048, E=16, k=8, T=4)
    L = synth.gen_layer(cfg, seed=93)
    x = synth.gen_activations(cfg, seed=93)
    lay = dev_layer(L)
    wr = synth.gen_router(cfg, seed=93)
    lay.router_upload(wr, "sigmoid")
    xt, _, _ = to_dev_inputs(cfg, x, np.zeros((1, 8), np.int32), np.zeros((1, 8), np.float32))
    out, ids, w = lay.forward_routed(xt)
    torch.cuda.synchronize()
    ids_h, w_h = ids.cpu().numpy(), w.cpu().numpy()
    ref, _ = oracle.forward(L, x, ids_h, w_h)
    assert_close(out.float().cpu().numpy().astype(np.float64), ref, "bf16", "forward_routed")
    _, _, z = lay.router(xt, want_logits=True)
    ids_k, _ = topk_from_logits(z.cpu().numpy(), cfg.k, "sigmoid")
    assert np.array_equal(ids_h, ids_k)
