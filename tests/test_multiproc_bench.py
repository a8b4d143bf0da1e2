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


def test_a_failing_extra_workload_keeps_the_headline_line(monkeypatch, capsys):
    # main() with the GPU-facing steps stubbed: one extra workload raises,
    # the JSON line still prints, with the error in that workload's entry
    import json
    import sys

    import torch

    import bench
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda *a, **k: None)
    monkeypatch.setattr(bench, "load_peaks", lambda: ({"hbm_gbs": 1.0, "bf16_tflops": 1.0}, "test"))
    monkeypatch.setattr(bench, "reduce_times", lambda ms, e2e, world, dev: (ms, e2e))

    def fake_measure(name, *a, **k):
        if name == "prefill_vq_overflow":
            raise RuntimeError("injected failure")
        return {"ms": 1.0, "e2e_s": 1.0, "name": name}

    monkeypatch.setattr(bench, "measure", fake_measure)
    monkeypatch.setattr(bench, "summarize", lambda args, name, r, *a, **k: {"workload": name, "value": 1.0})
    monkeypatch.setattr(bench, "measure_router", lambda T, *a, **k: {"workload": f"router_t{T}"})
    monkeypatch.setattr(bench, "measure_encoder", lambda *a, **k: {"workload": "vq_encode_expert"})
    monkeypatch.setattr(sys, "argv", ["bench.py", "--no-cpu-baseline"])
    assert bench.main() == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["workload"] == "decode_mxfp4"
    w = line["workloads"]
    assert "injected failure" in w["prefill_vq_overflow"]["error"]
    assert w["prefill_mxfp4_zipf"]["workload"] == "prefill_mxfp4_zipf"
    assert set(w) == set(bench.EXTRA_WORKLOADS) | {"router_t1", "router_t2048", "vq_encode_expert"}
