"""moeq_route_noalloc, the route/bucket step with its scratch in a fixed
in-library array (no device allocation), for callers that cannot allocate
device memory.  It must give exactly the oracle's buckets, and exactly those
of moeq_route (the entry point that uses a layer's workspace), call after
call.  Collected last so that it also runs after every other test has used
the device."""
import ctypes as C

import numpy as np
import pytest

from _gpu_util import oracle, torch_mod

pytestmark = pytest.mark.gpu


def _noalloc(lib, ids_dev, T, k, E, offs, perm, stream):
    return lib.moeq_route_noalloc(C.c_void_p(ids_dev.data_ptr()), T, k, E, C.c_void_p(offs.data_ptr()),
                                  C.c_void_p(perm.data_ptr()), C.c_void_p(stream.cuda_stream))


def test_route_noalloc_matches_route_on_consecutive_calls():
    torch = torch_mod()
    from bit_quantized_moe_routed_b200 import moeq
    lib = moeq.lib()
    E, k, Tmax = 256, 8, 2048
    lay = moeq.Layer(128, 128, E, k, Tmax, "mxfp4", "bf16")
    stream = torch.cuda.current_stream()
    rng = np.random.default_rng(2026)
    # a large call, then a smaller one with out-of-range ids: the second must
    # not see anything the first left in the shared scratch
    for T, p_bad in ((Tmax, 0.0), (37, 0.05)):
        ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
        u = rng.random(ids.shape)
        ids[u < 0.04] = -1
        ids[(u >= 0.04) & (u < 0.04 + p_bad)] = E + 5
        ids_dev = torch.from_numpy(ids).cuda()
        orc_off, orc_perm, orc_bad = oracle.route_bucket(ids, E)
        want_off, want_perm = lay.route(ids_dev)
        offs = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
        perm = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
        assert _noalloc(lib, ids_dev, T, k, E, offs, perm, stream) == moeq.OK
        torch.cuda.synchronize()
        n = int(orc_off[E])
        assert n == int(((ids >= 0) & (ids < E)).sum())
        assert orc_bad == int(((ids != -1) & ((ids < 0) | (ids >= E))).sum())
        # against the oracle, bit for bit
        assert np.array_equal(offs.cpu().numpy(), orc_off)
        assert np.array_equal(perm[:n].cpu().numpy(), orc_perm)
        assert bool((perm[n:] == -7).all())   # nothing written past the valid routes
        # and against moeq_route
        assert torch.equal(offs, want_off)
        assert torch.equal(perm[:n], want_perm[:n])
        lay.status(clear=True)


def test_route_noalloc_rejects_beyond_its_scratch():
    torch = torch_mod()
    from bit_quantized_moe_routed_b200 import moeq
    lib = moeq.lib()
    stream = torch.cuda.current_stream()
    ids_dev = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    offs = torch.full((1026,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((8,), -7, dtype=torch.int32, device="cuda")
    assert _noalloc(lib, ids_dev, 4, 2, 1025, offs, perm, stream) == moeq.UNSUPPORTED
    assert _noalloc(lib, ids_dev, 4, 65, 16, offs, perm, stream) == moeq.INVALID_ARGUMENT
    assert _noalloc(lib, ids_dev, 0, 2, 16, offs, perm, stream) == moeq.INVALID_ARGUMENT
    torch.cuda.synchronize()
    assert bool((offs == -7).all()) and bool((perm == -7).all())   # nothing launched
    # the largest expert count it takes
    ids_dev = torch.full((4, 2), 1023, dtype=torch.int32, device="cuda")
    assert _noalloc(lib, ids_dev, 4, 2, 1024, offs, perm, stream) == moeq.OK
    torch.cuda.synchronize()
    assert int(offs[1023]) == 0 and int(offs[1024]) == 8
    assert perm.tolist() == list(range(8))
