"""The route/bucket step (moeq_route) is bit-exact against the oracle."""
import numpy as np
import pytest

from _gpu_util import dev_layer, oracle, synth, torch_mod

pytestmark = pytest.mark.gpu


def _check(lay, ids, E):
    torch = torch_mod()
    it = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()
    offs, perm = lay.route(it)
    torch.cuda.synchronize()
    want_off, want_perm, bad = oracle.route_bucket(ids, E)
    offs = offs.cpu().numpy()
    perm = perm.cpu().numpy()
    assert np.array_equal(offs, want_off)
    assert np.array_equal(perm[: offs[E]], want_perm)
    # eight routes per token, summed over experts
    assert offs[E] == int(((ids >= 0) & (ids < E)).sum())
    return bad


def test_route_prefill_zipf_exact():
    cfg = synth.get_cfg("prefill_mxfp4_zipf", H=64, I=64)   # routing does not depend on H, I
    ids, _ = synth.gen_routing(cfg)
    from bit_quantized_moe_routed_b200 import moeq
    lay = moeq.Layer(128, 128, cfg.E, cfg.k, cfg.T, "mxfp4", "bf16")
    assert _check(lay, ids, cfg.E) == 0
    assert lay.status() == moeq.OK


@pytest.mark.parametrize("T,E,k", [(1, 256, 8), (3, 16, 2), (1023, 64, 4), (129, 1024, 64), (2048, 256, 8)])
def test_route_random_with_invalid_ids(T, E, k):
    from bit_quantized_moe_routed_b200 import moeq
    rng = np.random.default_rng(T * 7 + E)
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)   # duplicates allowed
    mask = rng.random(ids.shape)
    ids[mask < 0.05] = -1
    ids[(mask >= 0.05) & (mask < 0.07)] = E + 3
    ids[(mask >= 0.07) & (mask < 0.08)] = -7
    lay = moeq.Layer(128, 128, E, k, T, "mxfp4", "bf16")
    bad = _check(lay, ids, E)
    assert (lay.status(clear=True) == moeq.ROUTE_OUT_OF_RANGE) == (bad > 0)
    assert lay.status() == moeq.OK


def test_route_all_no_route():
    from bit_quantized_moe_routed_b200 import moeq
    ids = np.full((5, 2), -1, np.int32)
    lay = moeq.Layer(128, 128, 16, 2, 5, "mxfp4", "bf16")
    assert _check(lay, ids, 16) == 0
    assert lay.status() == moeq.OK
