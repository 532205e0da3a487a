"""Host-side logic of bench.py, on the CPU: the cross-rank reduction and the whole-job
throughput of the N-GPU replica run (world size 2 over gloo), the nvidia-smi clock
sampler (against a fake nvidia-smi), and the reference arm's JSON line."""
import importlib.util
import json
import os
import socket
import stat
import subprocess
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("fv_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, per_rank, out_dir):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        b = load_bench()
        step_ms = b.max_over_ranks(per_rank[rank]["step_ms"], world, "cpu")
        e2e_ms = b.max_over_ranks(per_rank[rank]["e2e_ms"], world, "cpu")
        res = {"step_ms": step_ms, "e2e_ms": e2e_ms,
               "value": b.whole_job_tflops(per_rank[rank]["eff"], world, step_ms)}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_replica_timing_is_max_over_ranks_gloo_world2(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    # rank 1 is the slow one for the layer, rank 0 for the end-to-end leg
    per_rank = [{"step_ms": 3.9, "e2e_ms": 12.0, "eff": 3.4e12},
                {"step_ms": 4.2, "e2e_ms": 11.0, "eff": 3.4e12}]
    ctx = mp.get_context("spawn")
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, per_rank, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["step_ms"] == 4.2 and r["e2e_ms"] == 12.0
        # two replicas of 3.4e12 effective FLOPs each, per 4.2 ms
        assert r["value"] == pytest.approx(2 * 3.4e12 / 4.2e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    b = load_bench()
    assert b.max_over_ranks(3.25, 1) == 3.25
    assert b.whole_job_tflops(2e12, 1, 2.0) == pytest.approx(1000.0)
    assert b.whole_job_tflops(2e12, 4, 2.0) == pytest.approx(4000.0)


FAKE_SMI = """#!/bin/bash
# fake nvidia-smi: only --id={ok_id} answers; samples every 20 ms after a slow start
case "$1" in --id={ok_id}) ;; *) exit 6;; esac
sleep 0.3
while true; do echo "{line}"; sleep 0.02; done
"""


def fake_smi(tmp_path, ok_id, line):
    d = tmp_path / "bin"
    d.mkdir(exist_ok=True)
    p = d / "nvidia-smi"
    p.write_text(FAKE_SMI.format(ok_id=ok_id, line=line))
    p.chmod(p.stat().st_mode | stat.S_IXUSR)
    return str(d)


def test_clock_sampler_waits_for_first_sample_and_keeps_the_timed_region(tmp_path, monkeypatch):
    b = load_bench()
    line = "1700, 1965, 950.5, 0x4, Not Active, Not Active, Not Active, Active"
    monkeypatch.setenv("PATH", fake_smi(tmp_path, 0, line) + os.pathsep + os.environ["PATH"])
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    s = b.ClockSampler(0)
    t0 = time.monotonic()
    s.start()
    assert s.lines, "start() returns only once a sample has arrived"
    assert time.monotonic() - t0 >= 0.25
    s.begin()
    time.sleep(0.15)
    s.end()
    c = s.stop()
    assert c["sm_mhz"] == 1700.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    assert c["samples_inside_timed_region"] >= 1
    assert c["samples"] == c["samples_inside_timed_region"] + 1


def test_clock_sampler_maps_visible_devices_and_falls_back_to_local_rank(tmp_path, monkeypatch):
    b = load_bench()
    line = "1965, 1965, 300.0, 0x0, Active, Not Active, Not Active, Not Active"
    monkeypatch.setenv("PATH", fake_smi(tmp_path, 0, line) + os.pathsep + os.environ["PATH"])
    # the rank's device is physical GPU 5, which this fake refuses: the sampler falls back
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "5,6")
    s = b.ClockSampler(0)
    assert s.ids == ["5", "0"]
    s.start()
    assert s.index == "0"
    s.begin()
    time.sleep(0.1)
    s.end()
    c = s.stop()
    assert c["reasons"] == ["hw_slowdown"]
    assert b.ClockSampler(1).ids == ["6", "1"]


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    b = load_bench()
    monkeypatch.setenv("PATH", str(tmp_path))
    s = b.ClockSampler(0)
    s.start()
    s.begin()
    s.end()
    assert s.stop()["reasons"] == ["nvidia-smi unavailable"]


def run_bench(args, env_extra, timeout=300):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_only_rank0_prints():
    r = run_bench(["--impl", "reference", "--steps", "1", "--warmup", "3"],
                  {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_json_line():
    r = run_bench(["--impl", "reference", "--steps", "1", "--warmup", "3"], {})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True and d["dtype"] == "f64"
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "wan21_1.3b_480p_h12_21x30x52"


def test_attention_traffic_only_for_its_workload_and_source():
    bench = load_bench()
    w480 = bench.W.WAN21_480P.name
    assert bench.ATTN_NCU_TRAFFIC["workload"] == w480
    got = bench.attn_traffic(w480)
    # the recorded bytes when the kernel source is the one they were taken from, else null
    assert got in (bench.ATTN_NCU_TRAFFIC["bytes"], None)
    for wl in (bench.W.TINY, bench.W.WAN22_720P, bench.W.WAN21_6X):
        assert bench.attn_traffic(wl.name) is None


def test_e2e_chunks_default_divides_the_slices():
    bench = load_bench()
    assert bench.e2e_chunks(0, 12) == 6
    assert bench.e2e_chunks(0, 40) == 5
    assert bench.e2e_chunks(0, 2) == 2
    assert bench.e2e_chunks(0, 7) == 4
    assert bench.e2e_chunks(0, 1) == 1
    assert bench.e2e_chunks(8, 12) == 8
    assert bench.e2e_chunks(16, 12) == 12
