"""bench.py host logic on the CPU: work formulas, clock parsing, the ncu
traffic guard, the reference arm's JSON line, and the N > 1 replica path's
rank logic and max-over-ranks reduction on 2 gloo ranks."""
import json
import os
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from moe_inputs import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_expert_stage_work_counts_only_active_experts():
    cfg = CONFIGS["builder_bf16"]
    counts = [0] * 64
    counts[3] = 8000
    counts[9] = 192
    b, f = bench.expert_stage_work(cfg, counts)
    N, H, I = 8192, 4096, 1408
    assert f == 2 * N * 3 * H * I
    # weights, x_packed read, h written and read, bf16 y_packed written, routing weights
    assert b == 2 * 3 * H * I * 2 + N * H * 2 + 2 * N * I * 2 + N * H * 2 + N * 4


def test_gemm_roofline_counts_only_activated_weights():
    cfg = CONFIGS["builder_bf16"]
    counts = [0] * 64
    counts[3] = 8000
    counts[9] = 192
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}
    H, I, N = 4096, 1408, 8192
    wb, fl = bench.expert_weight_work(cfg, counts)
    assert wb == 2 * 3 * H * I * 2 and fl == 2 * N * 3 * H * I
    r = bench.gemm_roofline(cfg, counts, 0.5, peaks)
    # flops / weight bytes = 2*8192/2 = 8192 > ridge 250: tensor bound
    assert r["bound"] == "tensor"
    assert abs(r["achieved"] - fl / 0.5e-3 / 1e12) < 1e-9
    assert abs(r["frac"] - r["achieved"] / 1500.0) < 1e-12
    assert abs(r["frac_nominal"] - r["achieved"] / 2250.0) < 1e-12
    assert r["bytes_incl_packed"] == bench.expert_stage_work(cfg, counts)[0]
    # every expert active at uniform load: weight-bound
    r = bench.gemm_roofline(cfg, [128] * 64, 0.4, peaks)
    assert r["bound"] == "hbm"
    assert abs(r["achieved"] - 64 * 3 * H * I * 2 / 0.4e-3 / 1e9) < 1e-6
    assert r["frac_incl_packed"] > r["frac"]


def test_layer_roofline_against_measured_and_nominal_peaks():
    cfg = CONFIGS["decode_t1"]
    counts = [0, 1, 0, 0, 0, 0, 1, 0]
    lb, lf = bench.layer_work(cfg, counts)
    r = bench.layer_roofline(cfg, counts, 0.2, {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0})
    assert r["bound"] == r["bound_nominal"] == "hbm"
    assert abs(r["frac"] - lb / 6000e9 / 0.2e-3) < 1e-12
    assert abs(r["frac_nominal"] - lb / 8000e9 / 0.2e-3) < 1e-12


def test_zipf_slope_of_an_exact_power_law():
    counts = [int(round(1e6 * r ** -1.1)) for r in range(1, 121)] + [0] * 8
    assert abs(bench.zipf_slope(counts) + 1.1) < 1e-3
    assert bench.zipf_slope([5, 0, 0]) is None


def test_layer_work_includes_router_and_shared_expert():
    cfg = CONFIGS["qwen15_t32"]
    counts = [1] * 60
    b, f = bench.layer_work(cfg, counts)
    H, I, Is, E, T, k = 2048, 1408, 5632, 60, 32, 4
    assert f == 2 * T * k * 3 * H * I + 2 * T * H * E + 2 * T * 3 * H * Is + 2 * T * H
    assert b == 60 * 3 * H * I * 2 + E * H * 2 + 2 * T * H * 2 + 3 * H * Is * 2 + H * 2


def test_clock_parsing():
    rows = ("0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Active\n"
            "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Not Active\n"
            "garbage line\n")
    c = bench.parse_clock_samples(rows)
    assert c == {"sm_mhz": 1882.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2}


def test_ncu_traffic_is_dropped_when_the_kernel_changed(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "grouped_gemm_traffic.json").write_text(json.dumps(
        {"kernel_source_sha": "not-the-current-hash", "per_step_bytes": {"builder_bf16": 1}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.ncu_traffic("builder_bf16") is None
    (prof / "grouped_gemm_traffic.json").write_text(json.dumps(
        {"kernel_source_sha": "abc", "per_step_bytes": {"builder_bf16": 123}}))
    assert bench.ncu_traffic("builder_bf16") == 123


def test_kernel_hash_ignores_comments_but_not_code():
    a = "int f(int x) {  // doubles\n  return 2 * x; /* fast */ }"
    b = "int f(int x) {\n  return 2 * x;\n}"
    c = "int f(int x) { return 3 * x; }"
    assert bench.strip_comments(a) == bench.strip_comments(b)
    assert bench.strip_comments(a) != bench.strip_comments(c)


def test_reference_arm_prints_one_json_line_and_other_ranks_exit_quietly():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--workload", "tiny_f32", "--steps", "2", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == "tiny_f32"
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def _replica_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = CONFIGS["tiny_f32"]
        p = bench.rank_inputs(cfg, rank)
        m = bench.max_over_ranks(1.5 + rank, torch.device("cpu"))
        q.put((rank, m, float(p["w13"].sum()), float(p["x"].sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_weights_differ_in_tokens_and_reduce_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_replica_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res[0][1] == res[1][1] == 2.5                       # max over ranks
    assert res[0][2] == res[1][2]                              # same layer weights
    assert res[0][3] != res[1][3]                              # different token batches


def test_max_over_ranks_without_a_process_group_is_the_identity():
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25
