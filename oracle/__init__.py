"""The oracle: a plain f64 CPU restatement of the compressed-expert MoE layer.

TEST INFRASTRUCTURE ONLY.  Imported by the tests, by the package smoke
check and by the benchmark's CPU-baseline leg; never by the library.
"""
from .oracle import (  # noqa: F401
    build,
    lib,
    e2m1,
    e8m0,
    idx13,
    e4m3,
    gvq1_idx,
    bf16_to_f32,
    f16_to_f64,
    dequant,
    forward,
    forward_by_expert,
    num_threads,
    route_bucket,
)
