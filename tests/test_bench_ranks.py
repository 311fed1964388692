"""The multi-rank plumbing of bench.py on CPU: two gloo ranks run the same
helpers bench.py's timed path uses under torchrun (max over ranks, whole-job
rate, per-replica inputs), and the reference arm does no work off rank 0."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_env_defaults(monkeypatch):
    for v in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(v, raising=False)
    assert bench.dist_env() == (1, 0, 0)
    monkeypatch.setenv("WORLD_SIZE", "4")
    monkeypatch.setenv("RANK", "3")
    monkeypatch.setenv("LOCAL_RANK", "3")
    assert bench.dist_env() == (4, 3, 3)


def test_whole_job_rate_counts_every_rank_over_the_slowest():
    # 8 tokens per step per rank, 100 steps, 2 ranks, slowest rank 50 ms -> 32000 tokens/s
    assert bench.whole_job_rate(8, 100, 2, 50.0) == pytest.approx(32000.0)
    assert bench.whole_job_rate(8, 100, 1, 50.0) == pytest.approx(16000.0)


def test_replicas_draw_distinct_inputs():
    seeds = {bench.replica_input_seed(0, r, b) for r in range(8) for b in range(16)}
    assert len(seeds) == 8 * 16


def test_single_rank_max_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_WORKER = r"""
import json, os, sys
sys.path.insert(0, sys.argv[1])
import torch.distributed as dist
import bench
world, rank, _ = bench.dist_env()
dist.init_process_group("gloo", init_method="env://", world_size=world, rank=rank)
ms = 10.0 + 5.0 * rank           # rank 1 is the slower one
ms_max = bench.max_over_ranks(ms, world)
dist.barrier()
rate = bench.whole_job_rate(8, 100, world, ms_max)
dist.destroy_process_group()
print(json.dumps({"rank": rank, "ms_max": ms_max, "rate": rate}))
"""


def test_two_gloo_ranks_agree_on_the_max(tmp_path):
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, WORLD_SIZE="2", RANK=str(r), LOCAL_RANK=str(r), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", _WORKER, ROOT], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["ms_max"] == 15.0
        assert o["rate"] == pytest.approx(8 * 100 * 2 / 0.015)


def test_reference_arm_does_no_work_off_rank_zero():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""


def test_bench_parses_its_arguments():
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"], capture_output=True, text=True,
                       timeout=120)
    assert p.returncode == 0, p.stderr
    assert "--steps" in p.stdout


def test_launch_count_follows_the_dispatch():
    # verify8: front kernel, two E2M1-term stages, combine; verify256: hybrid; zipf1024: hybrid + multi-block
    # grouping; prefill8192: large-token FFN + multi-block grouping
    assert [bench.kernels_per_step(T, 8, 384, 6144) for T in (8, 256, 1024, 8192)] == [4, 12, 14, 11]
    # below 128 tokens with more than 384 experts: the chained launches
    assert bench.kernels_per_step(8, 8, 512, 6144) == 1 + 2 + 3 + 1
    assert bench.kernels_per_step(127, 32, 384, 6144) == 4  # 4064 pairs: still the front path
    assert bench.kernels_per_step(4, 2, 16, 256) == 4  # tiny


def test_verify_workload_reference_arm_prints_the_contract_line():
    # the verification workload's reference arm: the float64 oracle on host
    # cores, one block per step, printed as one JSON line with the base keys
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "verify_block", "--impl",
                        "reference", "--steps", "2", "--warmup", "1", "--vocab", "3000"], capture_output=True,
                       text=True, timeout=300, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    line = json.loads(p.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "blocks/s" and line["value"] > 0
    assert line["config"]["vocab"] == 3000 and line["config"]["block_size"] == 8
    # off rank 0 the arm does nothing
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    q = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "verify_block", "--impl",
                        "reference", "--steps", "2", "--warmup", "1", "--vocab", "3000"], capture_output=True,
                       text=True, timeout=300, cwd=ROOT, env=env)
    assert q.returncode == 0 and q.stdout.strip() == ""


def test_clock_summary_reads_the_timed_windows():
    cs = bench.ClockSampler("GPU-x")
    t = 1000.0

    def sample(dt, sm, pcap="Not Active"):
        return dict(t=t + dt, sm=sm, max=1965.0, hw="Not Active", hwt="Not Active", swt="Not Active", pcap=pcap)

    cs.samples = [sample(0.0, 1965.0), sample(0.5, 1500.0, "Active"), sample(0.55, 1400.0, "Active"),
                  sample(2.0, 1965.0)]
    out = cs.summary([(t + 0.45, t + 0.6)])
    assert out["samples"] == 2 and out["sm_mhz"] == 1450.0 and out["reasons"] == ["sw_power_cap"]
    # two windows: the union of their samples
    out = cs.summary([(t - 0.01, t + 0.01), (t + 1.99, t + 2.01)])
    assert out["samples"] == 2 and out["sm_mhz"] == 1965.0 and out["reasons"] == []
    # a window between samples falls back to the nearest ones, and says so
    out = cs.summary([(t + 1.0, t + 1.01)])
    assert out["samples"] == 2 and out.get("nearest_to_window")
    assert bench.ClockSampler("GPU-y").summary([(t, t + 1)])["reasons"] == ["unsampled"]


def test_host_cpu_names_cores_and_model():
    cores, model = bench.host_cpu()
    assert cores >= 1 and isinstance(model, str) and model


def test_layer_reference_arm_prints_the_contract_line():
    # the layer's reference arm on the tiny workload: the float64 oracle on
    # host cores, one seeded token per step
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    line = json.loads(p.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["host_cores"] >= 1 and line["cpu_baseline"]["cpu_model"]
    assert line["config"]["workload"].startswith("tiny:")


def test_headline_is_the_largest_single_gpu_workload():
    assert bench.HEADLINE == max(datagen_configs(), key=lambda c: c.T).name


def datagen_configs():
    import datagen

    return datagen.CONFIGS
