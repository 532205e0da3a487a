"""bench.py's GPU arm run end to end on the CPU (tests/_fake_cuda_bench.py stands in for
CUDA and the library), at world size 1 and as two torchrun ranks over gloo: it exits 0,
rank 0 alone prints one JSON line, and the line has every key of the bench contract
with consistent values.  Device timings are constant stand-ins; only the bookkeeping
is under test."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HARNESS = os.path.join(ROOT, "tests", "_fake_cuda_bench.py")

TOP_KEYS = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"]


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def json_lines(out: str):
    return [json.loads(ln) for ln in out.splitlines() if ln.startswith("{")]


def check_line(d, n):
    for key in TOP_KEYS:
        assert key in d, key
    assert d["n_gpus"] == n and d["steps"] == 3 and d["warmup"] == 3
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["dtype"] == "bf16" and d["data"] == "synthetic" and d["vs_baseline"] is None
    assert d["config"]["workload"] == "wan21_1.3b_480p_h12_21x30x52" and "l2" in d["config"]
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    e = d["e2e"]
    assert set(["value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"]) <= set(e)
    assert e["h2d_bytes_per_step"] == 3 * 12 * 32760 * 128 * 2          # Q, K, V in
    assert e["d2h_bytes_per_step"] == 12 * 32760 * 128 * 2 + 12 * 32760 * 4   # out and lse back
    # six kernels a layer step (pool, logits, selection, prep_cost, prep_order,
    # attention), three steps
    assert d["gpu_launches"] == 6 * 3
    assert set(["sm_mhz", "sm_max_mhz", "reasons"]) <= set(d["clocks"])
    # the stand-in route keeps every block: the layer's effective FLOPs are the dense count,
    # n replicas of it every 4 ms
    dense = 4.0 * 128 * 32760 * 32760 * 12
    assert abs(d["value"] - n * dense / 4e-3 / 1e12) < 1e-2


def test_single_rank_line():
    r = subprocess.run([sys.executable, HARNESS, "--steps", "3", "--warmup", "3", "--no-cpu-baseline"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    check_line(lines[0], 1)


def test_two_ranks_over_gloo():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), HARNESS, "--gpus", "2",
           "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1                       # rank 0 only
    check_line(lines[0], 2)
    assert "cpu_baseline" not in lines[0] or lines[0]["cpu_baseline"] is None   # N = 1 only


def test_sweep_lines_world_size_1():
    """--sweep prints the headline line, then one line per p x k point, each timed by graph
    replay with the direct call beside it."""
    env = dict(os.environ, PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, HARNESS, "--steps", "3", "--warmup", "3", "--sweep",
                          "--no-cpu-baseline"], capture_output=True, text=True, env=env, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = json_lines(out.stdout)
    assert "metric" in lines[0]
    pts = [d for d in lines[1:] if "sweep_point" in d]
    assert len(pts) == 15
    for d in pts:
        for key in ("p", "k_floor", "kept_block_frac", "attn_ms", "attn_ms_direct_call", "speedup_vs_dense",
                    "effective_tflops", "frac_of_bf16_peak", "timing"):
            assert key in d, key
        assert d["kept_block_frac"] == 1.0          # the stand-in route keeps every block


def test_workload_flag_prints_one_line_for_that_workload():
    """--workload runs one workload only (the profiler runs use it): one line, named for it,
    not the headline, and the ncu traffic of the 480p kernel is not reported on it."""
    r = subprocess.run([sys.executable, HARNESS, "--steps", "3", "--warmup", "3", "--no-cpu-baseline",
                        "--workload", "tiny_h2_d64_4x8x8"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["config"]["workload"] == "tiny_h2_d64_4x8x8"
    assert "not the headline" in d["metric"]
    assert d["roofline"]["traffic"] is None
