"""Host-side pieces of bench.py that need no GPU: the units of the metric, the bytes a step moves, and the
reference arm's bounded oracle sample."""

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import flashnorm_inputs as I  # noqa: E402


def test_metric_units_prefill_and_decode():
    pre = [I.WORKLOADS[n] for n in bench.BENCH_WORKLOADS["smollm2_prefill_m8192"]]
    assert not bench._is_decode(pre)
    assert bench._units(pre) == sum(w.flops for w in pre)
    dec = [I.WORKLOADS["llama7b_qkv_m4"]]
    assert bench._is_decode(dec) and bench._units(dec) == 2 * 4096 * 12288
    fp8 = [I.WORKLOADS["llama7b_qkv_fp8_m4"]]
    assert bench._units(fp8) == 4096 * 12288 + 4 * 12288  # one byte per weight plus the channel scales
    nv4 = [I.WORKLOADS["llama7b_qkv_nvfp4_m4"]]
    # half a byte per weight, one E4M3 scale per 16 weights, a fp32 scale per channel
    assert bench._units(nv4) == 12288 * (4096 // 2 + 4096 // 16 + 4)


def test_step_bytes_follow_the_weight_format():
    w16, w8 = I.WORKLOADS["llama7b_qkv_m4"], I.WORKLOADS["llama7b_qkv_fp8_m4"]
    assert bench._set_bytes(w16) - bench._set_bytes(w8) == 4096 * 12288 - 4 * 12288
    assert w8.bytes == 2 * (4 * 4096 + 4 * 12288) + 4096 * 12288 + 4 * 12288
    w4 = I.WORKLOADS["llama7b_qkv_nvfp4_m4"]
    assert w4.bytes == 2 * (4 * 4096 + 4 * 12288) + 12288 * (2048 + 256 + 4)
    assert bench._set_bytes(w8) - bench._set_bytes(w4) == 12288 * (4096 - 2048 - 256)


def test_reference_sample_shrinks_and_still_runs_the_oracle():
    wl = "smollm2_qkv_m64"
    bench._ORACLE_CACHE.pop(wl, None)
    _, _, projs = bench._oracle_setup(wl)
    assert len(projs[0]["rows"]) == 64
    rate, cores, desc, el = bench.time_oracle(wl, 0.0)  # one pass
    assert rate > 0 and cores >= 1 and "64 of 64 rows" in desc
    bench._shrink_sample(wl, 0.25)
    assert len(projs[0]["rows"]) == 16
    rate2, _, desc2, _ = bench.time_oracle(wl, 0.0)
    assert rate2 > 0 and "16 of 64 rows" in desc2
    # the sampled rows are the oracle's own output for those rows
    y = projs[0]["call"](projs[0]["rows"], projs[0]["chans"])
    assert y.shape == (16, 960) and np.isfinite(y).all()
    bench._ORACLE_CACHE.pop(wl, None)


def test_decode_sample_shrinks_channels():
    wl = "llama7b_qkv_fp8_m1"
    bench._ORACLE_CACHE.pop(wl, None)
    _, decode, projs = bench._oracle_setup(wl)
    assert decode and projs[0]["chans"] == 1024
    bench._shrink_sample(wl, 0.1)
    assert projs[0]["chans"] == 96 and bench._pass_units(projs[0], True) == 96 * (4096 + 4)
    bench._ORACLE_CACHE.pop(wl, None)


def test_gpu_count_must_match_the_ranks():
    # --gpus N without N ranks would print a line for fewer GPUs than asked; bench.py refuses instead
    import subprocess

    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference"],
                       capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode == 2 and "WORLD_SIZE=1" in r.stderr


def test_nvfp4_sample_runs_the_oracle():
    """The NVFP4 decode workload's CPU baseline decodes a bounded channel sample with the oracle."""
    wl = "llama7b_qkv_nvfp4_m1"
    bench._ORACLE_CACHE.pop(wl, None)
    _, decode, projs = bench._oracle_setup(wl)
    assert decode and projs[0]["chans"] == 1024
    bench._shrink_sample(wl, 1 / 16)
    assert projs[0]["chans"] == 64 and bench._pass_units(projs[0], True) == 64 * (2048 + 256 + 4)
    y = projs[0]["call"](projs[0]["rows"], projs[0]["chans"])
    assert y.shape == (1, 64) and np.isfinite(y).all()
    bench._ORACLE_CACHE.pop(wl, None)


def test_reference_arm_on_a_quantized_workload():
    """bench.py --impl reference on the NVFP4 decode workload: one JSON line, the oracle on the host cores,
    in the GPU arm's metric and unit."""
    import json
    import subprocess

    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "llama7b_qkv_nvfp4_m4"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["config"]["workload"] == "llama7b_qkv_nvfp4_m4"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
