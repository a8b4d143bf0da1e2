import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")


def read_golden(name):
    """Rows of a golden text fixture: '#' lines are comments, fields split on whitespace."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def golden():
    return read_golden


class _MimoLayers(dict):
    """MiMo-shaped layers (hidden 4096, inter 2048, 256 experts, top-8),
    generated and uploaded on first use, shared by every GPU test:
      decode_mxfp4         MXFP4, max 2048 tokens (the prefill Zipf workload
                           has the same weights)
      decode_vq            VQ13+R8, base book N(0, 0.02^2)
      decode_vq_off        the same bytes with the residual stage off
      prefill_vq_overflow  VQ13+R8 with the base book x64, max 2048 tokens"""

    def __missing__(self, name):
        import synth
        from _gpu_util import dev_layer
        if name == "decode_mxfp4":
            L = synth.gen_layer(synth.get_cfg("decode_mxfp4"))
            val = (L, dev_layer(L, max_tokens=2048))
        elif name == "decode_vq":
            L = synth.gen_layer(synth.get_cfg("decode_vq"))
            val = (L, dev_layer(L, max_tokens=8))
        elif name == "decode_vq_off":
            L = self["decode_vq"][0].without_residual()
            val = (L, dev_layer(L, max_tokens=8))
        elif name == "prefill_vq_overflow":
            L = synth.gen_layer(synth.get_cfg("prefill_vq_overflow"))
            val = (L, dev_layer(L, max_tokens=2048))
        else:
            raise KeyError(name)
        self[name] = val
        return val


@pytest.fixture(scope="session")
def mimo_layers():
    layers = _MimoLayers()
    yield layers
    for _, lay in layers.values():
        lay.close()
