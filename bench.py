#!/usr/bin/env python3
"""Benchmark of the SharQ sparse-dense FP4 linear layer on B200.

One step = the whole hot path on one batch: fused prep (device tensor amax,
RMSNorm, online 4:8-pair mask, backbone + residual NVFP4) and the fused
sparse+dense FP4 GEMM, on the Llama-3.1-8B q_proj shape (X 2048 x 4096 bf16,
W 4096 x 4096), synthetic seeded data.  The weight is quantized once, outside
the timed region (it is an offline step of the layer).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sharq|reference]

Prints ONE JSON line (rank 0).  value = effective TFLOP/s = 2*T*N*K per step
summed over ranks / max-over-ranks time; L2 is flushed (256 MB write) before
every timed step, outside the step's CUDA events.  Multi-GPU runs are
independent replicas (the layer has no exchange step): weak scaling.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "effective TFLOP/s of sparse+dense FP4 linear (1 B200) + prep GB/s vs roofline"
T, K, N = 2048, 4096, 4096
WORKLOAD = "Llama-3.1-8B q_proj: X 2048x4096 bf16 (0.5*t3 + 8 outlier channels x100), RMSNorm, W 4096x4096; NVFP4, 4:8 pair"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
FP4_OVER_BF16 = 9.0 / 2.25          # nominal dense FP4 / dense BF16 ratio
PREP_BYTES_PER_ELEM = 2.0 + 0.25 + 1 / 16 + 1 / 32 + 0.5 + 1 / 16  # bf16 in; bb codes, meta, bb sf, res codes, res sf


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


class ClockSampler:
    """SM clock and throttle reasons sampled (read-only NVML queries, every 2 ms
    in a background thread) during the timed region."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, torch_index: int):
        self.torch_index = torch_index
        self.samples = []
        self.max_mhz = None
        self._stop = False
        self._thread = None
        self.handle = None

    def _open(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = None
        try:
            uuid = str(torch.cuda.get_device_properties(self.torch_index).uuid)
        except Exception:
            pass
        if uuid:
            u = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(u.encode() if isinstance(u, str) else u)
        else:
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.torch_index)
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        return pynvml

    def _run(self, nv):
        while not self._stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.0002)

    def __enter__(self):
        import threading
        try:
            nv = self._open()
            self._thread = threading.Thread(target=self._run, args=(nv,), daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *a):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        reasons = set()
        for _, rs in self.samples:
            for name, bit in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml"}


def kernel_hash() -> str:
    h = hashlib.sha256()
    for name in ("gemm.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "activation_sparsity_fp4_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_hash") != kernel_hash():
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- CPU oracle
_ORACLE_SETUP = {}


def _oracle_setup():
    """Workload and the offline weight quantization for the oracle (untimed, once)."""
    if not _ORACLE_SETUP:
        import oracle
        from activation_sparsity_fp4_b200 import workloads
        cfg = workloads.q_proj()
        wq = oracle.quantize_weight(cfg["w"], "nvfp4")
        _ORACLE_SETUP.update(cfg=cfg, wq=wq, wu=oracle.decode_weight(wq))
    return _ORACLE_SETUP


def cpu_baseline(rows: int = T):
    """The oracle, as it stands, on the host cores: tensor amax over all rows,
    prep of the first `rows` rows and the fp64 reference GEMM of those rows;
    scaled to effective TFLOP/s (2 * rows * N * K / time)."""
    import numpy as np

    import oracle

    st = _oracle_setup()
    cfg, wq, wu = st["cfg"], st["wq"], st["wu"]
    cores = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    amax = oracle.rows_amax(cfg["x"], cfg["gamma"], cfg["eps"])
    prep = oracle.prepare(cfg["x"][:rows], "nvfp4", "4:8pair", gamma=cfg["gamma"], eps=cfg["eps"], act_amax=amax,
                          threads=cores)
    y = oracle.linear_ref(prep, wq, wu=wu)
    dt = time.perf_counter() - t0
    assert np.isfinite(y).all()
    value = 2.0 * rows * N * K / dt / 1e12
    return {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{rows} of {T} rows: tensor amax over all rows, prep of those rows with {cores} threads, "
                      f"fp64 numpy GEMM of those rows ({dt:.2f} s)"}, dt


# --------------------------------------------------------------------- GPU
def run_sharq(args):
    import numpy as np
    import torch

    from activation_sparsity_fp4_b200 import sharq, workloads

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist

    cfg = workloads.q_proj()
    x_host = torch.from_numpy(cfg["x"]).to(torch.bfloat16).pin_memory()
    x = x_host.to(dev)
    gamma = torch.from_numpy(cfg["gamma"]).to(torch.bfloat16).to(dev)
    w = torch.from_numpy(cfg["w"]).to(torch.bfloat16).to(dev)
    wq = sharq.FP4Weight.quantize(w, "nvfp4")
    prep = sharq.Prepared(T, K, "nvfp4", "4:8pair", dev)
    y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
    y_host = torch.empty((T, N), dtype=torch.bfloat16).pin_memory()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sharq.sharq_sync_status()

    def step():
        sharq.prepare(x, "nvfp4", "4:8pair", gamma, cfg["eps"], out=prep)
        sharq.linear(prep, wq, out=y)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    sharq.sharq_sync_status()

    # the step as two CUDA graphs (prep, GEMM): no host launch overhead, and the
    # GEMM can still be timed on its own with events between the replays
    g_prep, g_gemm = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    sharq.sharq_launch_count(reset=True)
    with torch.cuda.graph(g_prep):
        sharq.prepare(x, "nvfp4", "4:8pair", gamma, cfg["eps"], out=prep)
    with torch.cuda.graph(g_gemm):
        sharq.linear(prep, wq, out=y)
    launches_per_step = sharq.sharq_launch_count()
    for _ in range(args.warmup):
        flush.fill_(1)
        g_prep.replay()
        g_gemm.replay()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            flush.fill_(1)
            e0, e1, e2, e3 = ev[i]
            e0.record(stream)
            g_prep.replay()
            e1.record(stream)
            e2.record(stream)
            g_gemm.replay()
            e3.record(stream)
        torch.cuda.synchronize()
    launches = launches_per_step * args.steps
    if pg:
        pg.barrier()
    sharq.sharq_sync_status()
    step_ms = [e[0].elapsed_time(e[3]) for e in ev]
    prep_ms = [e[0].elapsed_time(e[1]) for e in ev]
    gemm_ms = [e[2].elapsed_time(e[3]) for e in ev]
    total_ms = sum(step_ms)

    # caller-given amax variant of prep (no extra read of x), for the prep roofline
    pev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    amax = float(prep.tensor[0].item())
    for i in range(args.steps):
        flush.fill_(1)
        pev[i][0].record(stream)
        sharq.prepare(x, "nvfp4", "4:8pair", gamma, cfg["eps"], act_amax=amax, out=prep)
        pev[i][1].record(stream)
    torch.cuda.synchronize()
    prep_given_ms = statistics.mean(a.elapsed_time(b) for a, b in pev)

    # end to end through the public API from pinned host buffers
    eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(1)
        eev[i][0].record(stream)
        x.copy_(x_host, non_blocking=True)
        step()
        y_host.copy_(y, non_blocking=True)
        eev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in eev)
    sharq.sharq_sync_status()

    times = torch.tensor([total_ms, e2e_ms], dtype=torch.float64, device=dev)
    if pg:
        pg.all_reduce(times, op=pg.ReduceOp.MAX)
    total_ms, e2e_ms = times.tolist()

    if rank == 0:
        pk, src = peaks()
        flops = 2.0 * T * N * K
        value = world * flops * args.steps / (total_ms / 1e3) / 1e12
        gemm_avg = statistics.mean(gemm_ms) / 1e3
        fp4_peak = pk["bf16_tflops"] * FP4_OVER_BF16
        achieved = 3.0 * T * N * K / gemm_avg / 1e12   # FP4-dense-equivalent work of the pair
        prep_bytes = PREP_BYTES_PER_ELEM * T * K
        prep_gbs = prep_bytes / (statistics.mean(prep_ms) / 1e3) / 1e9
        prep_given_gbs = prep_bytes / (prep_given_ms / 1e3) / 1e9
        clocks = clk.summary()
        out = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "nvfp4 (e2m1 x e4m3 block-16 scales, fp32 accumulate)",
            "data": "synthetic (seeded, shaped like the pages' Llama-3.1-8B q_proj layer)",
            "config": {"workload": WORKLOAD, "t": T, "k": K, "n": N, "fmt": "nvfp4", "pattern": "4:8 pair",
                       "norm": "rmsnorm", "y_dtype": "bf16", "parallelism": f"replicas x{world}",
                       "l2": "flushed (256 MB write) before every timed step"},
            "roofline": {"bound": "tensor", "kernel": "gemm_kernel<NVF4, sparse>",
                         "achieved": round(achieved, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                         "frac": round(achieved / fp4_peak, 4), "traffic": committed_traffic(),
                         "peak_source": f"{src}: bf16 burst x {FP4_OVER_BF16:g} (nominal FP4/BF16)",
                         "work": "3*T*N*K FP4-dense-equivalent flops per launch (sparse 2TNK at 2x rate + dense 2TNK)",
                         "avg_launch_us": round(gemm_avg * 1e6, 2)},
            "prep": {"gbs_device_amax": round(prep_gbs, 1), "gbs_given_amax": round(prep_given_gbs, 1),
                     "peak_gbs": pk["hbm_gbs"], "frac_given_amax": round(prep_given_gbs / pk["hbm_gbs"], 4),
                     "frac_device_amax": round(prep_gbs / pk["hbm_gbs"], 4),
                     "bytes_per_elem": PREP_BYTES_PER_ELEM, "avg_us": round(statistics.mean(prep_ms) * 1e3, 2),
                     "avg_us_given_amax": round(prep_given_ms * 1e3, 2)},
            "e2e": {"value": round(world * flops * args.steps / (e2e_ms / 1e3) / 1e12, 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(x_host.numel() * 2), "d2h_bytes_per_step": int(y_host.numel() * 2)},
            "gpu_launches": int(launches),
            "launch_mode": "CUDA graphs (prep graph + GEMM graph per step); e2e uses direct API calls",
            "clocks": clocks,
        }
        if not args.no_cpu_baseline and world == 1:
            out["cpu_baseline"], _ = cpu_baseline()
        print(json.dumps(out), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def run_reference(args):
    """Reference arm: the CPU oracle as it stands, on the host cores, each step a
    bounded sample of the same workload (rank 0 only)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    rows = 256
    for _ in range(args.warmup):
        cpu_baseline(rows)
    times = []
    base = None
    for _ in range(args.steps):
        base, dt = cpu_baseline(rows)
        times.append(dt)
    total = sum(times)
    value = 2.0 * rows * N * K * args.steps / total / 1e12
    base["value"] = value
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 prep / f64 GEMM (CPU oracle)",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "t": T, "k": K, "n": N, "sample_rows_per_step": rows},
        "cpu_baseline": base,
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["sharq", "reference"], default="sharq")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_sharq(args)


if __name__ == "__main__":
    main()
