"""Host-side logic of bench.py on the CPU: the multi-rank reduction (gloo,
world size 2), replica sizing against L2, clock-log parsing, the guard
that drops profiled DRAM traffic once the kernel source changes, and the
reference arm (the oracle on the host cores), which needs no GPU: its one
JSON line at one rank and under torchrun at two."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [12.5, 20.0][rank]
    ms = bench.max_over_ranks(local_ms, world, "cpu")
    value = bench.job_throughput(world, 32776, 100, ms)
    with open("%s.%d" % (out_path, rank), "w") as f:
        json.dump({"ms": ms, "value": value}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo(tmp_path):
    out = str(tmp_path / "r")
    mp.spawn(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    res = [json.load(open("%s.%d" % (out, r))) for r in range(2)]
    for r in res:
        assert r["ms"] == 20.0                           # slowest rank
        assert r["value"] == pytest.approx(2 * 32776 * 100 / 0.020)


def test_single_rank_passthrough():
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
    assert bench.job_throughput(1, 10, 5, 1000.0) == 50.0


def test_replicas_exceed_twice_l2():
    l2 = 126 * 1024 * 1024
    for per in (37_761_024, 75_497_472, 10_000, 10 ** 9):
        R = bench.replicas_for(per, l2)
        assert R >= 2 and (R * per >= 2 * l2 or per > l2)


def test_kv_bytes_per_token():
    # K and V, 8 heads, 64 code bytes + 8 scale bytes each = 1152 bytes
    assert bench.kv_bytes_per_token(8, 128) == 1152


def test_clock_summary_parsing():
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.samples = [
        (10.0, "0, 1965, 1965, 500.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"),
        (10.1, "0, 1950, 1965, 510.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active"),
        (10.2, "0, 1800, 1965, 520.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"),
        (20.0, "0, 345, 1965, 90.0, 0x0000000000000000, Active, Not Active, Not Active, Not Active"),
    ]
    s = c.summary(9.9, 10.25)
    assert s["samples"] == 3 and s["sm_mhz"] == 1950 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    assert c.summary(30.0, 31.0)["samples"] == 0


def test_traffic_dropped_when_source_changes(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    for p in bench.ATTN_SOURCES:
        os.makedirs(os.path.dirname(tmp_path / p), exist_ok=True)
        (tmp_path / p).write_text("kernel v1")
    os.makedirs(tmp_path / "profiles")
    digest = bench.source_digest(bench.ATTN_SOURCES)
    (tmp_path / "profiles" / "t.json").write_text(json.dumps(
        {"source_digest": digest, "dram_bytes_per_launch": 123}))
    assert bench.profiled_traffic("t.json") == (123, None)
    (tmp_path / bench.ATTN_SOURCES[0]).write_text("kernel v2")
    traffic, why = bench.profiled_traffic("t.json")
    assert traffic is None and "changed since the capture" in why
    assert bench.profiled_traffic("missing.json")[0] is None


REF_KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _check_reference_line(line, n):
    d = json.loads(line)
    assert REF_KEYS <= set(d), REF_KEYS - set(d)
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["n_gpus"] == n and d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["vs_baseline"] is None
    assert d["config"]["workload"].startswith(bench.DEFAULT_WORKLOAD)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def _run(cmd):
    r = subprocess.run(cmd, cwd=bench.ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return lines


@pytest.mark.slow
def test_reference_arm_one_rank_prints_its_line():
    lines = _run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert len(lines) == 1
    _check_reference_line(lines[0], 1)


@pytest.mark.slow
def test_reference_arm_under_torchrun_rank0_alone_prints():
    lines = _run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                  "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
                  "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"])
    assert len(lines) == 1
    _check_reference_line(lines[0], 2)
