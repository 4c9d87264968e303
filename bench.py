"""Benchmark of the FlashNorm fused RMSNorm -> linear path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload (one "step"): the SmolLM2-135M-shaped prefill of 8192 tokens, d = 576: the fused
QKV projection (W [576, 960]) and the fused SwiGLU up-projection (W [576, 2 x 1536]), both with the
RMSNorm gain folded into the weights and the 1/rms scale deferred into the kernels' epilogues.
Weights are folded once, outside the timed region (folding is an offline step).

Timing: W untimed warm-up steps, then exactly K steps. Between steps a 256 MiB buffer is written to
flush the 126 MB L2, outside the per-step CUDA events; each step is bracketed by events on the
launching stream and the step times are summed. Multi-GPU (torchrun): every rank runs its own
batch (weak scaling, no collective on the data path); the time is the max over ranks.

One JSON line is printed by rank 0. `value` is TFLOP/s of the contraction (2 M d N per projection)
for prefill workloads and weight GB/s for decode workloads. `roofline` describes the dominant kernel
against MEASURED_PEAKS.json; `e2e` is the same metric through the same C-ABI calls with host
buffers (pinned H2D copy of x and D2H copy of the outputs inside the timed region); `cpu_baseline`
is the fp64 oracle timed on this host's cores on a bounded sample of the workload.

--impl reference times the oracle itself (the only reference implementation there is: the pages
ship no code) on the host cores, on the same workload, metric and unit.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import flashnorm_inputs as I  # noqa: E402

# ----------------------------------------------------------------------------------------------
# Workloads the bench knows. A workload is a list of projections run back to back in one step.
# ----------------------------------------------------------------------------------------------
BENCH_WORKLOADS = {
    "smollm2_prefill_m8192": ["smollm2_qkv_m8192", "smollm2_ffn_m8192"],
    "smollm2_qkv_m64": ["smollm2_qkv_m64"],
    "llama7b_qkv_m1": ["llama7b_qkv_m1"],
    "llama7b_qkv_m4": ["llama7b_qkv_m4"],
    "llama7b_qkv_m16": ["llama7b_qkv_m16"],
    "llama7b_qkv_m2048": ["llama7b_qkv_m2048"],
    "llama7b_ffn_m2048": ["llama7b_ffn_m2048"],
    "mla_latent_m2048": ["mla_latent_m2048"],
}
DEFAULT_WORKLOAD = "smollm2_prefill_m8192"

# DRAM traffic of the dominant kernel per launch, from the ncu capture summarised in profiles/
# (dram__bytes_read.sum + dram__bytes_write.sum). Valid only for the kernel source it was taken on:
# if the CUDA sources hash differently now, traffic is reported as null.
NCU_TRAFFIC = {
    # workload: (bytes per launch, sha256[:16] of the csrc/*.cu* sources at capture time, profile file)
}

L2_FLUSH_BYTES = 256 << 20


def _sources_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "rmsnorm_linear_projection_fold_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()[:16]


def _peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


def _is_decode(wls) -> bool:
    return all(w.M <= 16 for w in wls)


def _metric(wls):
    if _is_decode(wls):
        return "fused RMSNorm+linear weight GB/s (decode)", "GB/s"
    return "fused RMSNorm+linear TFLOP/s (prefill)", "TFLOP/s"


def _units(wls) -> float:
    """Work per step in the metric's numerator: FLOPs (prefill) or weight bytes (decode)."""
    if _is_decode(wls):
        return float(sum(2 * w.d * w.w_cols for w in wls))
    return float(sum(w.flops for w in wls))


def _scale(wls) -> float:
    return 1e-12 if not _is_decode(wls) else 1e-9


# ----------------------------------------------------------------------------------------------
# Clock sampling during the timed region (NVML, the library nvidia-smi reads).
# ----------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        0x0000000000000004: "sw_power_cap",
        0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False

    def _sample(self):
        try:
            self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
            self.reasons |= int(self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self) -> dict:
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(np.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------------------------
# Our implementation on the GPU
# ----------------------------------------------------------------------------------------------
def _to_dev(bits, torch):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


class Projection:
    """One workload's projection with its inputs resident in HBM and its weights folded."""

    def __init__(self, wl, fn, torch):
        self.wl, self.fn, self.torch = wl, fn, torch
        b = wl.draw()
        self.x = _to_dev(b["x"], torch)
        self.g = _to_dev(b["g"], torch)
        W = _to_dev(b["w"], torch)
        self.ws = fn.flashnorm_fold_weights(W, self.g, glu=(wl.kind == "glu"))
        ones = torch.ones(wl.d, dtype=torch.bfloat16, device="cuda")
        self.wk = fn.flashnorm_fold_weights(W, ones, glu=(wl.kind == "glu"))  # unfolded, K-major
        del W
        self.g2 = _to_dev(b["g2"], torch) if wl.kind == "postnorm" else None
        self.y = torch.empty(wl.M, wl.N, dtype=torch.bfloat16, device="cuda")
        self.xn = torch.empty(wl.M, wl.d, dtype=torch.bfloat16, device="cuda")
        self.x_host = torch.from_numpy(np.ascontiguousarray(b["x"]).view(np.int16)).view(torch.bfloat16).pin_memory()
        self.y_host = torch.empty(wl.M, wl.N, dtype=torch.bfloat16).pin_memory()

    def run(self, x=None):
        wl, fn = self.wl, self.fn
        x = self.x if x is None else x
        if wl.kind == "linear":
            fn.flashnorm_linear(x, self.ws, wl.eps, out=self.y)
        elif wl.kind == "glu":
            fn.flashnorm_glu(x, self.ws, wl.eps, out=self.y)
        else:
            fn.flashnorm_linear_postnorm(x, self.ws, self.g2, wl.head_dim, wl.eps2, out=self.y)

    def run_unfused(self):
        wl, fn = self.wl, self.fn
        if wl.kind == "linear":
            fn.flashnorm_linear_unfused(self.x, self.g, self.wk, wl.eps, xn_ws=self.xn, out=self.y)
        elif wl.kind == "glu":
            fn.flashnorm_glu_unfused(self.x, self.g, self.wk, wl.eps, xn_ws=self.xn, out=self.y)
        else:
            return False
        return True

    def launches(self) -> int:
        return 1


def _time_steps(torch, steps, body, flush):
    """Sum of per-step CUDA-event times (ms) over `steps` steps; L2 flushed between steps."""
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    marks = []
    for i in range(steps):
        flush()
        evs[i][0].record(stream)
        m = body()
        evs[i][1].record(stream)
        marks.append(m)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs), marks


def run_ours(args, rank, world, device_index):
    import torch

    import rmsnorm_linear_projection_fold_b200 as fn

    fn.load_library()
    torch.cuda.set_device(device_index)
    names = BENCH_WORKLOADS[args.workload]
    wls = [I.WORKLOADS[n] for n in names]
    projs = [Projection(w, fn, torch) for w in wls]
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def flush():
        flush_buf.fill_(1)

    # the dominant kernel: the projection with the most work
    dom = max(range(len(projs)), key=lambda i: wls[i].flops if not _is_decode(wls) else wls[i].bytes)
    stream = torch.cuda.current_stream()

    def step():
        ev = None
        for i, p in enumerate(projs):
            if i == dom:
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            p.run()
            if i == dom:
                e1 = torch.cuda.Event(enable_timing=True)
                e1.record(stream)
                ev = (e0, e1)
        return ev

    for _ in range(args.warmup):
        flush()
        step()
    fn.flashnorm_check_device_error()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(device_index)
    with sampler:
        t0 = time.perf_counter()
        total_ms, marks = _time_steps(torch, args.steps, step, flush)
        wall = time.perf_counter() - t0
    fn.flashnorm_check_device_error()
    dom_ms = sum(a.elapsed_time(b) for a, b in marks) / len(marks)
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
        torch.distributed.barrier()
    ms_per_step = total_ms / args.steps

    # unfused two-kernel baseline (same workload, same timing), for what folding + deferral buy
    unfused = None
    if all(w.kind in ("linear", "glu") for w in wls) and not _is_decode(wls):
        for _ in range(args.warmup):
            flush()
            [p.run_unfused() for p in projs]
        torch.cuda.synchronize()
        k_unf = max(3, min(args.steps, 200))
        unf_ms, _ = _time_steps(torch, k_unf, lambda: [p.run_unfused() for p in projs], flush)
        unfused = {"ms_per_step": unf_ms / k_unf, "fused_speedup": (unf_ms / k_unf) / ms_per_step,
                   "kernels_per_step": 2 * len(projs)}

    # end to end through the same calls with host buffers: H2D of x, the kernels, D2H of the outputs
    k_e2e = max(3, min(args.steps, 100))
    x_dev = [torch.empty_like(p.x) for p in projs]

    def e2e_step():
        for p, xd in zip(projs, x_dev):
            xd.copy_(p.x_host, non_blocking=True)
            p.run(xd)
            p.y_host.copy_(p.y, non_blocking=True)
        return None

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e2e_ms, _ = _time_steps(torch, k_e2e, e2e_step, flush)
    if world > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())
    h2d = sum(p.x.numel() * 2 for p in projs)
    d2h = sum(p.y.numel() * 2 for p in projs)

    units = _units(wls)
    scale = _scale(wls)
    metric, unit = _metric(wls)
    value = units * world / (ms_per_step * 1e-3) * scale
    peaks = _peaks()
    w_dom = wls[dom]
    if _is_decode(wls):
        achieved = w_dom.bytes / (dom_ms * 1e-3) * 1e-9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_kind": f"hbm copy ({peaks['source']})"}
    else:
        achieved = w_dom.flops / (dom_ms * 1e-3) * 1e-12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "peak_kind": f"bf16 burst ({peaks['source']})"}
    tr = NCU_TRAFFIC.get(args.workload)
    roof["traffic"] = tr[0] if tr and tr[1] == _sources_hash() else None
    roof["kernel"] = f"{w_dom.kind} {w_dom.name}"
    roof["kernel_ms"] = dom_ms
    roof["algorithmic_bytes"] = w_dom.bytes
    roof["algorithmic_flops"] = w_dom.flops

    out = {
        "metric": metric,
        "value": value,
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; x ~ N(0,1) x log-uniform[0.1,10] row scale, g ~ U(0.5,1.5), W ~ N(0,1/d))",
        "config": {
            "workload": args.workload,
            "projections": [{"name": w.name, "kind": w.kind, "M": w.M, "d": w.d, "N": w.N, "eps": w.eps}
                            for w in wls],
            "tokens_per_rank": wls[0].M,
            "l2": "flushed between steps (256 MiB write, outside the timed events)",
            "parallelism": f"dp{world} (independent batches per GPU)",
        },
        "roofline": roof,
        "e2e": {"value": units * world / (e2e_ms / k_e2e * 1e-3) * scale, "unit": unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": k_e2e},
        "gpu_launches": args.steps * sum(p.launches() for p in projs),
        "clocks": sampler.summary(),
        "wall_s_timed_region": wall,
    }
    if unfused is not None:
        out["unfused"] = unfused
    return out


# ----------------------------------------------------------------------------------------------
# The oracle on the host cores (cpu_baseline, and the --impl reference arm)
# ----------------------------------------------------------------------------------------------
def _cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle(workload: str, budget_s: float):
    """Run the oracle (as it stands) on sampled rows of each projection until budget_s is used.

    Returns (units per second scaled to the metric, cores, sample description, seconds)."""
    from oracle import flashnorm_oracle as O

    wls = [I.WORKLOADS[n] for n in BENCH_WORKLOADS[workload]]
    draws = [w.draw() for w in wls]
    # a bounded row sample: at most 1024 rows per projection per pass (all rows for small M)
    rows = [np.arange(min(w.M, 1024)) for w in wls]
    O.reference_output(wls[0].kind, draws[0], wls[0].eps, eps2=wls[0].eps2, head_dim=wls[0].head_dim,
                       rows=rows[0][:8])  # warm-up
    done_units, passes = 0.0, 0
    t0 = time.perf_counter()
    while True:
        for w, b, r in zip(wls, draws, rows):
            O.reference_output(w.kind, b, w.eps, eps2=w.eps2, head_dim=w.head_dim, rows=r)
            if _is_decode(wls):
                done_units += 2 * w.d * w.w_cols
            else:
                done_units += 2.0 * len(r) * w.d * w.w_cols
        passes += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    rate = done_units / el * _scale(wls)
    desc = (f"{passes} passes over " + ", ".join(f"{len(r)} of {w.M} rows of {w.name}" for w, r in zip(wls, rows))
            + f" in {el:.1f} s (fp64 numpy)")
    return rate, _cpu_threads(), desc, el


def run_reference(args, rank, world):
    if rank != 0:
        return None
    wls = [I.WORKLOADS[n] for n in BENCH_WORKLOADS[args.workload]]
    metric, unit = _metric(wls)
    per_step = []
    for _ in range(args.warmup):
        time_oracle(args.workload, 0.05)
    for _ in range(args.steps):
        rate, cores, desc, el = time_oracle(args.workload, 1.0)
        per_step.append((rate, el))
    value = float(np.mean([r for r, _ in per_step]))
    ms_per_step = float(np.mean([e for _, e in per_step])) * 1e3
    return {
        "impl": "reference",
        "metric": metric,
        "value": value,
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded, same inputs as the GPU arm)",
        "config": {"workload": args.workload,
                   "projections": [{"name": w.name, "kind": w.kind, "M": w.M, "d": w.d, "N": w.N} for w in wls]},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(BENCH_WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    import torch

    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    out = run_ours(args, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            rate, cores, desc, _ = time_oracle(args.workload, args.cpu_budget)
            out["cpu_baseline"] = {"value": rate, "unit": out["unit"], "cores": cores, "kind": "oracle",
                                   "sample": desc}
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
