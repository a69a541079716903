"""Host-side logic of bench.py that needs no GPU: the reference arm (the oracle on the host cores)
prints one JSON line with the GPU arm's config, metric and unit; the traffic table is keyed by the
workload's shape."""
import io
import json
import types
from contextlib import redirect_stdout

import pytest

import bench


def _args(workload, **kw):
    a = types.SimpleNamespace(workload=workload, M=0, proj="up", steps=1, warmup=0, cpu_budget=0.2,
                              gpus=1, world=1)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("workload,kw", [("w8a8_channel", {"M": 16}), ("w8a16", {"M": 4, "proj": "down"}),
                                         ("w8a8_block", {"M": 1, "proj": "down"})])
def test_reference_line_matches_gpu_arm_config(workload, kw):
    args = _args(workload, **kw)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC
    assert line["config"] == bench.describe(workload, args)["config"]
    assert line["unit"] == bench.WORKLOADS[workload].unit
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    from oracle import ref_cpp
    assert line["cpu_baseline"]["cores"] == ref_cpp.num_threads() >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_describe_shapes():
    d = bench.describe("w8a8_block", _args("w8a8_block", M=16384))
    assert (d["M"], d["N"], d["K"]) == (16384, 18432, 7168) and d["R"] >= 1
    d = bench.describe("w8a8_block", _args("w8a8_block", proj="down"))
    assert (d["M"], d["N"], d["K"]) == (16384, 7168, 18432)
    d = bench.describe("w8a16", _args("w8a16"))
    assert (d["M"], d["N"], d["K"]) == (16, 12288, 4096)
    assert bench.describe("w8a8_channel", _args("w8a8_channel", world=4))["config"]["global_batch"] == 4 * 4096


def test_measured_traffic_lookup():
    traffic, src = bench.measured_traffic("w8a16", {"M": 16, "N": 12288, "K": 4096})
    assert traffic and src.endswith(".md")
    assert bench.measured_traffic("w8a8_channel", {"M": 7, "N": 7168, "K": 2048}) == (None, None)


def test_default_is_the_block_wise_prefill_layer():
    import sys
    argv = sys.argv
    try:
        sys.argv = ["bench.py"]
        ap_args = None
        import argparse
        orig = argparse.ArgumentParser.parse_args

        def grab(self, *a, **k):
            nonlocal ap_args
            ap_args = orig(self, *a, **k)
            raise SystemExit(0)
        argparse.ArgumentParser.parse_args = grab
        try:
            bench.main()
        except SystemExit:
            pass
        finally:
            argparse.ArgumentParser.parse_args = orig
    finally:
        sys.argv = argv
    assert ap_args.workload == "w8a8_block" and ap_args.proj == "up"
    d = bench.describe(ap_args.workload, ap_args)
    assert (d["M"], d["N"], d["K"]) == (16384, 18432, 7168)


def test_traffic_sources_exist():
    import os
    root = os.path.dirname(os.path.abspath(bench.__file__))
    for key, (traffic, src) in bench.MEASURED_TRAFFIC.items():
        assert traffic > 0, key
        assert os.path.exists(os.path.join(root, "profiles", src)), (key, src)


def test_gpus_flag_spawns_one_process_per_gpu(monkeypatch):
    """`bench.py --gpus N` without torchrun spawns N ranks itself, each with the rank environment
    torchrun would give it (loopback rendezvous); under torchrun (WORLD_SIZE set) it spawns nothing."""
    import sys
    import torch.multiprocessing as mp
    calls, envs = [], []

    def fake_spawn(fn, args=(), nprocs=1, join=True):
        calls.append(nprocs)
        for r in range(nprocs):
            fn(r, *args)

    def fake_run(args):
        import os
        envs.append({k: os.environ[k] for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR", "MASTER_PORT")})

    monkeypatch.setattr(mp, "spawn", fake_spawn)
    monkeypatch.setattr(bench, "run_ours", fake_run)
    for k in ("RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):   # restored after the test
        monkeypatch.setenv(k, "x")
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "3"])
    bench.main()
    assert calls == [3]
    assert [e["RANK"] for e in envs] == ["0", "1", "2"] and all(e["WORLD_SIZE"] == "3" for e in envs)
    assert all(e["MASTER_ADDR"] == "127.0.0.1" and e["LOCAL_RANK"] == e["RANK"] for e in envs)
    calls.clear()
    envs.clear()
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main()
    assert calls == [] and len(envs) == 1
