"""Host logic of the multi-process bench on CPU: the timed durations are the
maximum over ranks (gloo, world size 2) and the reported value is the whole
job's throughput over that slowest rank."""
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms, e2e = bench.reduce_times(10.0 + 5.0 * rank, 1.0 + rank * 0.25, world, torch.device("cpu"))
    results[rank] = (ms, e2e)
    dist.barrier()
    dist.destroy_process_group()


def test_times_are_max_over_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs)
        assert results[0] == results[1] == (15.0, 1.25)


def test_single_rank_times_pass_through_and_job_value():
    import bench
    assert bench.reduce_times(3.0, 4.0, 1, None) == (3.0, 4.0)
    # 2 ranks x 1 token x 200 steps over 8 ms -> 50,000 tokens/s
    assert bench.job_tokens_per_s(2, 1, 200, 8.0) == pytest.approx(50000.0)


def test_traffic_record_follows_the_profiled_source(tmp_path, monkeypatch):
    import bench
    t, src = bench.ncu_traffic("decode_mxfp4")
    assert t is None or (t > 7e7 and src.startswith("profiles/"))
    assert bench.ncu_traffic("prefill_mxfp4_zipf") == (None, None)
    # a different source hash means no traffic figure
    path, sha, traffic, summary = bench.NCU_TRAFFIC["decode_mxfp4"]
    monkeypatch.setitem(bench.NCU_TRAFFIC, "decode_mxfp4", (path, "0" * 64, traffic, summary))
    assert bench.ncu_traffic("decode_mxfp4") == (None, None)


def test_gather_roofline_of_the_vq_decode_kernels():
    # VQ13+R8 at one token: 8 experts x gate and up x 2048 rows x 512 vectors,
    # two 16-byte entries per vector; GVQ1+R8 gathers 8-byte entries
    import bench
    import synth
    cfg = synth.get_cfg("decode_vq", T=1)
    g = bench.gather_roofline(cfg, 8.0, 0.05, {"sm_max_mhz": 1965.0})
    assert g["per_launch_bytes"] == 8 * 2 * 2048 * 512 * 32
    assert g["achieved"] == pytest.approx(g["per_launch_bytes"] / 50e-6 / 1e9)
    assert g["peak"] == pytest.approx(148 * 128 * 1.965)
    g1 = bench.gather_roofline(cfg.replace(fmt="gvq1r8"), 8.0, 0.05, {"sm_max_mhz": 1965.0})
    assert g1["per_launch_bytes"] * 2 == g["per_launch_bytes"]
    g0 = bench.gather_roofline(cfg.replace(fmt="vq13"), 8.0, 0.05, {"sm_max_mhz": 1965.0})
    assert g0["per_launch_bytes"] * 2 == g["per_launch_bytes"]
