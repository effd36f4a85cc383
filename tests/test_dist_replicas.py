"""The multi-GPU path of bench.py is N independent replicas (no data-path
collective): whole-job throughput = every rank's tokens / the slowest rank's
device time.  Checked here with two gloo ranks on the CPU."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_WORKER = r"""
import importlib.util, json, os, sys
from datetime import timedelta
import torch.distributed as dist
spec = importlib.util.spec_from_file_location("bench", os.path.join(sys.argv[1], "bench.py"))
bench = importlib.util.module_from_spec(spec)
spec.loader.exec_module(bench)
ws, rank, local = bench.dist_env()
dist.init_process_group("gloo", timeout=timedelta(seconds=60))
ms, value = bench.job_throughput(10.0 + 5.0 * rank, 100, ws, device="cpu")
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "ms": ms, "value": value}))
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_replicas_take_the_slowest_rank_and_all_tokens():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                   LOCAL_RANK=str(rank), WORLD_SIZE="2", CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", _WORKER, ROOT], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["ms"] == 15.0                          # max over ranks
        assert abs(o["value"] - 200 / 0.015) < 1e-6     # both ranks' tokens / the slowest time


def test_single_rank_needs_no_process_group():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    ms, value = bench.job_throughput(20.0, 64, 1, device="cpu")
    assert ms == 20.0 and abs(value - 3200.0) < 1e-9


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the other ranks of the reference arm exit without work."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--config", "tiny", "--steps", "3", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_reference_arm_prints_the_contract_line():
    """Rank 0 of the reference arm prints one JSON line with every key of the
    bench contract, on the same workload config as the GPU arm."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "3", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3
    assert d["unit"] == "tok/s" and d["higher_is_better"] is True and d["value"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    from token_decode_b200 import synth
    assert d["config"] == bench.workload_config(synth.CONFIGS["tiny"], 1)


def test_clock_summary_keeps_the_timed_region():
    """Clock samples are summarised over the ones inside the timed region (by
    their nvidia-smi timestamps), or over all of them when none falls inside."""
    import datetime
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    c = bench.ClockSampler(0)
    c.t0 = datetime.datetime(2026, 1, 2, 3, 4, 5, 100000)
    c.t1 = datetime.datetime(2026, 1, 2, 3, 4, 5, 400000)
    idle = "2026/01/02 03:04:05.050, 1100, 1965, 120.0, Not Active, Not Active, Not Active, Not Active"
    busy1 = "2026/01/02 03:04:05.150, 1965, 1965, 700.5, Not Active, Not Active, Not Active, Active"
    busy2 = "2026/01/02 03:04:05.350, 1950, 1965, 720.0, Not Active, Not Active, Not Active, Not Active"
    after = "2026/01/02 03:04:05.450, 1000, 1965, 90.0, Active, Not Active, Not Active, Not Active"
    c.out = "\n".join([idle, busy1, busy2, after])
    s = c.summary()
    assert s["sm_mhz"] == 1957.5 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples_in_timed_region"] == 2
    c.t0 = c.t1 = datetime.datetime(2025, 1, 1)        # no sample inside: all of them
    s = c.summary()
    assert s["samples"] == 4 and s["samples_in_timed_region"] == 0
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    c.out = "not a sample\n"
    assert c.summary()["reasons"] == ["unavailable"]


def test_launch_count_claim_matches_the_committed_launch_lists():
    """bench.py's gpu_launches per step agrees with the ncu launch lists under
    profiles/: 142 launches for one 7B Q4_0 step at B = 1, and six launches per
    MoE block."""
    import importlib.util
    import re
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    from token_decode_b200 import synth
    text = open(os.path.join(ROOT, "profiles", "launches_decode_step_7b_q4_0.md")).read()
    n_listed = int(re.search(r"^(\d+) launches", text, flags=re.M).group(1))
    assert bench.step_launches(synth.CONFIGS["7b"]) == n_listed == 142
    moe = synth.CONFIGS["moe"]
    # a MoE layer replaces the dense FFN's two projections (each an activation
    # pack + a tensor-core GEMM at 32 rows) with the six launches of the block
    dense = moe.with_(n_experts=0, F=512)
    assert bench.step_launches(moe) - bench.step_launches(dense) == moe.L * (6 - 2 * 2)
    text = open(os.path.join(ROOT, "profiles", "launches_moe_layer_b32.md")).read()
    assert re.search(r"^12 launches", text, flags=re.M)
    # at 32 rows every NVFP4 projection is an activation pack plus a tensor-core GEMM
    text = open(os.path.join(ROOT, "profiles", "launches_decode_step_9b_b32.md")).read()
    n_listed = int(re.search(r"^(\d+) launches", text, flags=re.M).group(1))
    assert bench.step_launches(synth.CONFIGS["9b_b32"]) == n_listed == 1 + 36 * 9 + 2


def test_roofline_traffic_only_from_a_summary_of_the_current_sources(tmp_path, monkeypatch):
    """roofline.traffic comes from a committed ncu summary only while the
    kernel sources it lists still hash to the value it records."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    srcs = ["gemv.cu", "bw_common.cuh"]
    sha = bench.kernel_sources_sha(srcs)
    prof = tmp_path / "profiles"
    prof.mkdir()
    good = "- kernel_sources: `%s`\n- kernel_sources_sha: `%s`\n- traffic_bytes_per_launch: `1234`\n" % (
        " ".join(srcs), sha)
    (prof / "good.md").write_text(good)
    (prof / "stale.md").write_text(good.replace(sha, "0" * 16))
    (prof / "nosrc.md").write_text("- traffic_bytes_per_launch: `99`\n")
    monkeypatch.setattr(bench, "_PROFILE_FILES", {("a", "c"): "good.md", ("b", "c"): "stale.md",
                                                  ("d", "c"): "nosrc.md", ("e", "c"): "missing.md"})
    # summaries looked up under tmp_path; the hash of the real sources as computed above
    monkeypatch.setattr(bench, "__file__", str(tmp_path / "bench.py"))
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda files: sha if files == srcs else "-")
    assert bench._ncu_traffic("a", "c") == 1234
    assert bench._ncu_traffic("b", "c") is None
    assert bench._ncu_traffic("d", "c") is None
    assert bench._ncu_traffic("e", "c") is None
    assert bench._ncu_traffic("zz", "c") is None


def test_step_bytes_counts_weights_kv_and_routed_experts():
    """The roofline's algorithmic bytes per step: every dense weight matrix and
    norm once, K + V over the context and the new rows, and per MoE layer the
    bytes its launch touches (router, shared expert, selected experts)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    from token_decode_b200 import synth
    cfg = synth.CONFIGS["tiny"]
    model = synth.make_model(cfg, "cpu", seed=0)
    H, F, V, L = cfg.H, cfg.F, cfg.V, cfg.L
    w = (cfg.nqkv * H + H * cfg.nq * cfg.hd + 3 * F * H + V * H) * 9 // 16 + (2 * L + 1) * H * 4
    kv = 2 * L * cfg.nkv * cfg.hd * 2 * cfg.B
    assert bench.step_bytes(cfg, model, 100.0) == w + kv * 100 + kv
    moe = cfg.with_(fmt=synth.FMT_NVFP4, F=0, n_experts=8, topk=2, F_exp=64, B=2)
    mm = synth.make_model(moe, "cpu", seed=0)
    dense = bench.step_bytes(moe, mm, 10.0)
    assert bench.step_bytes(moe, mm, 10.0, moe_layer_bytes=12345) == dense + moe.L * 12345
