#!/usr/bin/env python3
"""Benchmark of the SharQ sparse-dense FP4 linear layer on B200.

One step = the whole hot path on one batch: fused prep (device tensor amax,
RMSNorm, online 4:8-pair mask, backbone + residual NVFP4) and the fused
sparse+dense FP4 GEMM, on the Llama-3.1-8B q_proj shape (X 2048 x 4096 bf16,
W 4096 x 4096), synthetic seeded data.  The weight is quantized once, outside
the timed region (it is an offline step of the layer).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sharq|reference]
                  [--workload NAME] [--tokens T] [--extra all|none]

The headline line measures --workload (default q_proj) and, with --extra all
(the default), carries a "workloads" object with the same measurements for
every other layer shape the pages evaluate: Tiny, down_proj at 2048 rows and
the 1/16/64/256-row sweep, Wan2.2 (4:8 pair and 8:16), and the Qwen3-30B-A3B
MoE gate/up (tokens prepared once, prepared rows gathered) and down
projections.  --tokens sets the row count of the q_proj / down_proj shapes.

Timing.  Each workload holds R sets of inputs, weights and outputs whose
total is at least three times the 126 MB L2 (R = 1 once one set is that
large); consecutive steps use consecutive sets, so every step reads data that
has left L2.  The K timed steps run back to back as ONE CUDA graph (kernels
chained by programmatic dependent launch) between two CUDA events; prep and
GEMM are then timed alone the same way (a graph of back-to-back launches over
the sets), which gives each kernel's average launch duration for the roofline
fields.

Prints ONE JSON line (rank 0).  value = effective TFLOP/s = 2*T*N*K per step
summed over ranks / max-over-ranks time.  Multi-GPU runs are independent
replicas (the layer has no exchange step): weak scaling.
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
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
FP4_OVER_BF16 = 9.0 / 2.25          # nominal dense FP4 / dense BF16 ratio
FP8_OVER_BF16 = 4.5 / 2.25          # nominal dense FP8 / dense BF16 ratio

WORKLOADS = {
    "tiny": "Tiny: X 16x256 fp32 ~N(0,1), channels 3 and 77 x40, W 256x256 ~N(0,0.02^2) fp32; no norm; MXFP4, 2:4",
    "q_proj": "Llama-3.1-8B q_proj: X 2048x4096 bf16 (0.5*t3 + 8 outlier channels x100), RMSNorm, W 4096x4096; "
              "NVFP4, 4:8 pair",
    "down_proj": "Llama-3.1-8B down_proj: X 2048x14336 bf16 = SiLU(a)*b, a,b ~N(0,1); W 4096x14336 ~N(0,0.01^2); "
                 "MXFP4, 2:4",
    "wan": "Wan2.2-14B DiT linear: X 32768x5120 bf16 ~N(0,1) + 16 outlier channels x50, RMSNorm; W 5120x5120; "
           "NVFP4, 4:8 pair",
    "wan_816": "Wan2.2-14B DiT linear: X 32768x5120 bf16 ~N(0,1) + 16 outlier channels x50, RMSNorm; W 5120x5120; "
               "NVFP4, 8:16",
    "wan_816pair": "Wan2.2-14B DiT linear: X 32768x5120 bf16 ~N(0,1) + 16 outlier channels x50, RMSNorm; W 5120x5120; "
                   "NVFP4, 8:16 selection re-packed into the 4:8 pair layout (sparse tensor cores)",
    "down_proj_swiglu": "Llama-3.1-8B down_proj from its gate and up inputs: gate, up 2048x14336 bf16 ~N(0,1), "
                        "h = SiLU(gate)*up formed inside the prep kernel; W 4096x14336 ~N(0,0.01^2); MXFP4, 2:4",
    "qwen_moe_gate_up": "Qwen3-30B-A3B MoE gate/up: 4096 tokens top-8 of 128 experts -> 32768 routed rows (each expert "
                        "padded to 128 rows), hidden 2048; per expert W 1536x2048; NVFP4, 4:8 pair, no norm; grouped",
    "qwen_moe_gate_up_gather": "Qwen3-30B-A3B MoE gate/up as qwen_moe_gate_up, but each of the 4096 tokens prepared "
                               "once and its prepared row gathered into the 32768 routed rows; grouped",
    "qwen_moe_gate_up_gemm_gather": "Qwen3-30B-A3B MoE gate/up as qwen_moe_gate_up, the 4096 tokens prepared once "
                                    "and the grouped GEMM reading each routed row by index from them (no routed "
                                    "copy); grouped",
    "qwen_moe_down": "Qwen3-30B-A3B MoE down: 32768 routed rows (expert order, each expert padded to 128 rows) x 768 "
                     "bf16 0.5*t3; per expert W 2048x768; NVFP4, 4:8 pair, no norm; grouped",
}

# the shapes the headline line also reports (name, rows or None)
EXTRA = [("tiny", None), ("down_proj", None), ("down_proj", 1), ("down_proj", 16), ("down_proj", 64),
         ("down_proj", 256), ("wan", None), ("wan_816", None), ("wan_816pair", None), ("qwen_moe_gate_up_gather", None),
         ("qwen_moe_gate_up_gemm_gather", None), ("qwen_moe_down", None)]

L2_BYTES = 126 * 1024 * 1024
ROTATE_BYTES = 3 * L2_BYTES  # the rotating sets of a workload cover at least this much


def prep_bytes_per_elem(fmt: str, pat: str, x_bytes: int = 2) -> float:
    """Algorithmic bytes of sharq_prepare per element of X: X read, then backbone codes, metadata,
    backbone scales, residual codes and residual scales written (layouts of sharq.h)."""
    b = 16 if fmt == "nvfp4" else 32
    meta = 1 / 16 if pat in ("4:8pair", "8:16pair") else 1 / 8
    bb_codes = 0.5 if pat == "8:16" else 0.25
    bb_sf = 1 / b if pat == "8:16" else 1 / (2 * b)  # 8:16 keeps the dense view (each scale twice)
    return x_bytes + bb_codes + meta + bb_sf + 0.5 + 1 / b


_CONFIG_CACHE = {}


def _config(fn, **kw) -> dict:
    """Seeded inputs of a config generator, built once per process (the MoE config
    serves two workloads)."""
    key = (fn.__name__, tuple(sorted(kw.items())))
    if key not in _CONFIG_CACHE:
        _CONFIG_CACHE[key] = fn(**kw)
    return _CONFIG_CACHE[key]


def make_workload(name: str, tokens: int | None = None) -> dict:
    """Inputs and roofline terms of one bench workload (host arrays; nothing of the method here).
    tokens: row count of the q_proj / down_proj shapes (the down_proj token sweep)."""
    from activation_sparsity_fp4_b200 import workloads
    if name.startswith("qwen_moe"):
        c = _config(workloads.qwen_moe)
        down = name == "qwen_moe_down"
        x, w = (c["x_down"], c["w_d"]) if down else (c["x"], c["w_gu"])
        t, k = x.shape
        n = w.shape[1]
        wl = dict(name=name, desc=WORKLOADS[name], x=x, x_dtype="bf16", gamma=None, eps=1e-6, w=w, fmt="nvfp4",
                  pat="4:8pair", offsets=c["offsets"], t=t, k=k, n=n, real_rows=int(c["counts"].sum()),
                  first_group=(int(c["offsets"][0]), int(c["offsets"][1])), gate=None, up=None)
        if name.endswith("_gather"):
            wl.update(tokens=c["x_tok"], gather=c["gather"], gemm_gather=name.endswith("_gemm_gather"))
        return wl
    kw = {"t": tokens} if tokens and name in ("q_proj", "down_proj", "down_proj_swiglu") else {}
    desc = WORKLOADS[name].replace("2048x", f"{tokens}x") if kw else WORKLOADS[name]
    gen = {"tiny": workloads.tiny, "q_proj": workloads.q_proj, "down_proj": workloads.down_proj,
           "down_proj_swiglu": workloads.down_proj, "wan": workloads.wan, "wan_816": workloads.wan,
           "wan_816pair": workloads.wan}[name]
    if name in ("wan_816", "wan_816pair"):
        kw = {"pat": "8:16" if name == "wan_816" else "8:16pair"}
    c = _config(gen, **kw)
    t, k = c["x"].shape
    wl = dict(name=name, desc=desc, x=c["x"], x_dtype=c.get("x_dtype", "bf16"), gamma=c["gamma"], eps=c["eps"], w=c["w"],
              fmt=c["fmt"], pat=c["pat"], offsets=None, t=t, k=k, n=c["w"].shape[0], real_rows=t,
              first_group=None, gate=None, up=None)
    if name == "down_proj_swiglu":
        wl.update(x=None, gate=c["gate"], up=c["up"])
    return wl


def gemm_roofline(wl: dict):
    """(work per launch in FP4- or FP8-dense-equivalent flops, peak kind, description)."""
    rows, n, k = wl["real_rows"], wl["n"], wl["k"]
    if wl["pat"] == "8:16":
        return 4.0 * rows * n * k, "fp4", "4*T*N*K: dense backbone 2TNK + dense residual 2TNK (kind::mxf4nvf4)"
    if wl["fmt"] == "mxfp4" and wl["pat"] == "2:4":
        return (3.0 * rows * n * k, "fp8",
                "3*T*N*K FP8-dense-equivalent: sparse 2TNK at 2x + dense 2TNK, both kind::mxf8f6f4")
    return 3.0 * rows * n * k, "fp4", "3*T*N*K FP4-dense-equivalent (sparse 2TNK at 2x rate + dense 2TNK)"


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of per-rank timings (one all_reduce(MAX)); the plain
    values when there is no process group."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def replica_throughput(world: int, work_per_step: float, steps: int, ms: float) -> float:
    """Whole-job throughput of N replicas in units of 1e12 per second: every rank
    did work_per_step per step; ms is the max-over-ranks time of the steps."""
    return world * work_per_step * steps / (ms / 1e3) / 1e12


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
    for name in ("gemm.cuh", "gemm_pair.cuh", "ptx.cuh"):
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


def _oracle_setup(name: str, tokens: int | None = None):
    """Workload and the offline weight quantization for the oracle (untimed, once)."""
    if _ORACLE_SETUP.get("name") != (name, tokens):
        import oracle
        wl = make_workload(name, tokens)
        w = wl["w"][0] if wl["offsets"] is not None else wl["w"]  # grouped: the first expert's weight
        wq = oracle.quantize_weight(w, wl["fmt"])
        _ORACLE_SETUP.clear()
        _ORACLE_SETUP.update(name=(name, tokens), wl=wl, wq=wq, wu=oracle.decode_weight(wq))
    return _ORACLE_SETUP


def cpu_baseline(name: str = "q_proj", rows: int = 2048, tokens: int | None = None):
    """The oracle, as it stands, on the host cores: the tensor amax over all rows
    (NVFP4), prep of `rows` rows (grouped: rows of the first expert) and the fp64
    reference GEMM of those rows; scaled to effective TFLOP/s (2 * rows * N * K / time)."""
    import numpy as np

    import oracle

    st = _oracle_setup(name, tokens)
    wl, wq, wu = st["wl"], st["wq"], st["wu"]
    x = wl["x"]
    r0 = wl["first_group"][0] if wl["first_group"] else 0
    rows = min(rows, (wl["first_group"][1] - r0) if wl["first_group"] else wl["t"])
    cores = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    if wl["gate"] is not None:  # SwiGLU form (MXFP4: no tensor amax)
        prep = oracle.prepare_swiglu(wl["gate"][:rows], wl["up"][:rows], wl["fmt"], wl["pat"], threads=cores)
    else:
        amax = oracle.rows_amax(x, wl["gamma"], wl["eps"]) if wl["fmt"] == "nvfp4" else 0.0
        prep = oracle.prepare(x[r0:r0 + rows], wl["fmt"], wl["pat"], gamma=wl["gamma"], eps=wl["eps"],
                              act_amax=amax, threads=cores)
    y = oracle.linear_ref(prep, wq, wu=wu)
    dt = time.perf_counter() - t0
    assert np.isfinite(y).all()
    value = 2.0 * rows * wl["n"] * wl["k"] / dt / 1e12
    _ORACLE_SETUP["rows_used"] = rows
    return {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{rows} of {wl['t']} rows: tensor amax over all rows, prep of those rows with {cores} threads, "
                      f"fp64 numpy GEMM of those rows ({dt:.2f} s)"}, dt


# --------------------------------------------------------------------- GPU
class LayerSets:
    """Device state of one workload: R sets of inputs, quantized weight, prepared
    activations and outputs, used in turn by consecutive steps so that together
    they cover at least ROTATE_BYTES (a step never finds its data in L2)."""

    def __init__(self, wl: dict, dev, max_sets: int = 16):
        import torch

        from activation_sparsity_fp4_b200 import sharq
        self.wl = wl
        T, K, N, fmt, pat = wl["t"], wl["k"], wl["n"], wl["fmt"], wl["pat"]
        self.swiglu = wl["gate"] is not None
        self.gathered = wl.get("gather") is not None
        self.gemm_gather = bool(wl.get("gemm_gather"))  # rows read by index inside the GEMM
        x_src = wl["gate"] if self.swiglu else (wl["tokens"] if self.gathered else wl["x"])
        self.x_dt = torch.float32 if wl.get("x_dtype") == "f32" else torch.bfloat16
        self.x_host = torch.from_numpy(x_src).to(self.x_dt).pin_memory()
        self.up_host = torch.from_numpy(wl["up"]).to(torch.bfloat16).pin_memory() if self.swiglu else None
        self.gamma = torch.from_numpy(wl["gamma"]).to(torch.bfloat16).to(dev) if wl["gamma"] is not None else None
        self.offsets = torch.from_numpy(wl["offsets"]).to(torch.int32).to(dev) if wl["offsets"] is not None else None
        self.rows_host = torch.from_numpy(wl["gather"]).to(torch.int32).pin_memory() if self.gathered else None
        self.rows = self.rows_host.to(dev) if self.gathered else None
        w = torch.from_numpy(wl["w"]).to(self.x_dt).to(dev)
        experts = int(wl["w"].shape[0]) if wl["offsets"] is not None else 1
        b = 16 if fmt == "nvfp4" else 32
        tp = (T + 127) // 128 * 128
        self.set_bytes = (self.x_host.numel() * self.x_host.element_size() * (2 if self.swiglu else 1)
                          + experts * (N * K // 2 + 2 * N * K // b) + tp * K + T * N * 2)
        self.R = max(1, min(max_sets, -(-ROTATE_BYTES // self.set_bytes)))
        self.x, self.up, self.prep, self.prep_tok, self.y, self.wq, self.ws = [], [], [], [], [], [], []
        for i in range(self.R):
            self.x.append(self.x_host.to(dev))
            self.up.append(self.up_host.to(dev) if self.swiglu else None)
            self.prep.append(None if self.gemm_gather else sharq.Prepared(T, K, fmt, pat, dev))
            self.prep_tok.append(sharq.Prepared(self.x_host.shape[0], K, fmt, pat, dev) if self.gathered else None)
            self.y.append(torch.zeros((T, N), dtype=torch.bfloat16, device=dev))
            self.wq.append(sharq.FP4Weight.quantize(w, fmt))  # the same codes in every set
            self.ws.append(sharq.linear_workspace(dev))  # lets few-tile shapes split their K loops
        del w

    def do_prep(self, i: int, act_amax: float = 0.0, stream=None):
        from activation_sparsity_fp4_b200 import sharq
        wl = self.wl
        if self.swiglu:
            sharq.prepare_swiglu(self.x[i], self.up[i], wl["fmt"], wl["pat"], act_amax=act_amax, out=self.prep[i],
                                 stream=stream)
        elif self.gathered:
            sharq.prepare(self.x[i], wl["fmt"], wl["pat"], self.gamma, wl["eps"], act_amax=act_amax,
                          out=self.prep_tok[i], stream=stream)
            if not self.gemm_gather:
                sharq.gather_prepared(self.prep_tok[i], self.rows, out=self.prep[i], stream=stream)
        else:
            sharq.prepare(self.x[i], wl["fmt"], wl["pat"], self.gamma, wl["eps"], act_amax=act_amax,
                          out=self.prep[i], stream=stream)

    def do_gemm(self, i: int, stream=None):
        from activation_sparsity_fp4_b200 import sharq
        if self.offsets is None:
            sharq.linear(self.prep[i], self.wq[i], out=self.y[i], workspace=self.ws[i], stream=stream)
        elif self.gemm_gather:
            sharq.linear_grouped_gather(self.prep_tok[i], self.rows, self.wq[i], self.offsets, out=self.y[i],
                                        stream=stream)
        else:
            sharq.linear_grouped(self.prep[i], self.wq[i], self.offsets, out=self.y[i], stream=stream)

    def step(self, i: int):
        self.do_prep(i)
        self.do_gemm(i)


def graph_of(fn, count: int, R: int):
    """One CUDA graph of `count` back-to-back calls fn(i % R)."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(count):
            fn(i % R)
    return g


def timed_replay_ms(g, stream) -> float:
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def measure(name: str, tokens, steps: int, warmup: int, e2e_steps: int, dev, pg, world: int) -> dict:
    """Timings of one workload (max over ranks) and its JSON fields."""
    import torch

    from activation_sparsity_fp4_b200 import sharq

    wl = make_workload(name, tokens)
    T, K, N, fmt, pat = wl["t"], wl["k"], wl["n"], wl["fmt"], wl["pat"]
    L = LayerSets(wl, dev)
    R = L.R
    stream = torch.cuda.current_stream()
    sharq.sharq_sync_status()
    for i in range(warmup):
        L.step(i % R)
    sharq.sharq_sync_status()

    # the K steps as ONE graph, back to back over the rotating sets; launches counted at capture
    sharq.sharq_launch_count(reset=True)
    g_steps = graph_of(L.step, steps, R)
    launches = sharq.sharq_launch_count()
    g_warm = graph_of(L.step, warmup, R)
    m = R * max(1, -(-16 // R))  # kernel-alone graphs: >= 16 launches, whole rounds of the sets
    g_prep = graph_of(L.do_prep, m, R)
    g_gemm = graph_of(L.do_gemm, m, R)
    g_warm.replay()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    with ClockSampler(torch.cuda.current_device()) as clk:
        total_ms = timed_replay_ms(g_steps, stream)
        if pg:
            pg.barrier()
        prep_ms = timed_replay_ms(g_prep, stream) / m
        gemm_ms = timed_replay_ms(g_gemm, stream) / m
    sharq.sharq_sync_status()
    # caller-given amax variant of prep (no extra read of x), for the prep roofline
    amax = float((L.prep_tok[0] if L.gemm_gather else L.prep[0]).tensor[0].item())
    g_given = graph_of(lambda i: L.do_prep(i, amax if fmt == "nvfp4" else 0.0), m, R)
    given_ms = timed_replay_ms(g_given, stream) / m
    sharq.sharq_sync_status()
    del g_steps, g_warm, g_prep, g_gemm, g_given

    # end to end through the public API from pinned host buffers: every step copies
    # its input in, runs prep + GEMM and copies y out; the steps run as a pipeline on
    # three streams (input copies, compute, output copies) with two sets of device
    # buffers (sets 0 and 1 when there are two), so step i+1's input copy and step
    # i-1's output copy overlap step i's compute.  Timed from the first input copy to
    # the last output copy (device events).
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    nb = min(R, 2)
    y_host = [torch.empty((T, N), dtype=torch.bfloat16).pin_memory() for _ in range(nb)]
    ev_in = [torch.cuda.Event() for _ in range(nb)]
    ev_cmp = [torch.cuda.Event() for _ in range(nb)]
    ev_out = [torch.cuda.Event() for _ in range(nb)]
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    for i in range(warmup + e2e_steps):
        b = i % nb
        if i == warmup:
            torch.cuda.synchronize()
            e_start.record(s_in)
        with torch.cuda.stream(s_in):
            if i >= nb:
                s_in.wait_event(ev_cmp[b])  # the compute that read these inputs is done
            L.x[b].copy_(L.x_host, non_blocking=True)
            if L.swiglu:
                L.up[b].copy_(L.up_host, non_blocking=True)
            if L.gathered:
                L.rows.copy_(L.rows_host, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b])
            if i >= nb:
                s_cmp.wait_event(ev_out[b])  # y of this buffer has been copied out
            L.do_prep(b, stream=s_cmp)
            L.do_gemm(b, stream=s_cmp)
            ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            y_host[b].copy_(L.y[b], non_blocking=True)
            ev_out[b].record(s_out)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    e_end.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_end)
    sharq.sharq_sync_status()

    total_ms, e2e_ms, prep_ms, given_ms, gemm_ms = max_over_ranks([total_ms, e2e_ms, prep_ms, given_ms, gemm_ms],
                                                                   pg, dev)
    pk, src = peaks()
    flops = 2.0 * wl["real_rows"] * N * K
    value = replica_throughput(world, flops, steps, total_ms)
    gemm_s = gemm_ms / 1e3
    work, kind, work_desc = gemm_roofline(wl)
    b_blk = 16 if fmt == "nvfp4" else 32
    experts = wl["w"].shape[0] if wl["offsets"] is not None else 1
    # algorithmic bytes of one launch: every expert's weight codes and sparse-view
    # scales once, the prepared rows (codes, scales, metadata) once, y (bf16) once
    wbytes = (experts * (N * K / 2 + N * K / (2 * b_blk) * (2 if pat == "8:16" else 1))
              + prep_bytes_per_elem(fmt, pat, 0) * T * K + 2 * T * N)
    ratio = FP4_OVER_BF16 if kind == "fp4" else FP8_OVER_BF16
    peak = pk["bf16_tflops"] * ratio
    achieved = work / gemm_s / 1e12
    # roofline time = max(compute at the tensor peak, bytes at the HBM peak)
    t_compute_us = work / (peak * 1e12) * 1e6
    t_bytes_us = wbytes / (pk["hbm_gbs"] * 1e9) * 1e6
    hbm_bound = t_bytes_us > t_compute_us
    bpe = prep_bytes_per_elem(fmt, pat, 4 if (L.swiglu or L.x_dt == torch.float32) else 2)
    prep_bytes = bpe * T * K
    if L.gemm_gather:  # prep of the tokens only (the GEMM reads the routed rows by index)
        prep_bytes = bpe * L.x_host.shape[0] * K
    elif L.gathered:  # prep of the tokens, then each routed row's prepared bytes read and written once
        prep_bytes = bpe * L.x_host.shape[0] * K + 2 * (bpe - 2) * T * K + 4 * T
    prep_gbs = prep_bytes / (prep_ms / 1e3) / 1e9
    given_gbs = prep_bytes / (given_ms / 1e3) / 1e9
    grouped = wl["offsets"] is not None
    kernel = {"4:8pair": "sparse", "8:16pair": "sparse", "2:4": "sparse", "8:16": "dense backbone"}[pat]
    kname = ("gemv_kernel" if (not grouped and T == 1) else
             "gemm_swap_kernel" if (not grouped and 2 <= T <= 64) else
             "gemm_pair_kernel" if (not grouped and pat in ("4:8pair", "8:16pair")
                                    and ((T + 127) // 128 * 128) % 256 == 0)
             else "gemm_kernel")
    kkind = "MXF8" if (fmt == "mxfp4" and pat == "2:4") else ("NVF4" if fmt == "nvfp4" else "MXF4")
    klabel = (f"gemv_kernel<{'MX' if fmt == 'mxfp4' else 'NV'}, {pat}, {T} rows>" if kname == "gemv_kernel"
              else f"gemm_swap_kernel<{'NVF4' if fmt == 'nvfp4' else 'MXF4'}, {pat} expanded, N={32 if T <= 32 else 64}>"
              if kname == "gemm_swap_kernel" else f"{kname}<{kkind}, {kernel}>")
    set_mb = L.set_bytes / 2 ** 20
    res = {
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "ms_per_step": round(total_ms / steps, 5),
        "steps": steps,
        "config": {"workload": wl["desc"], "t": T, "k": K, "n": N, "fmt": fmt, "pattern": pat,
                   "norm": "rmsnorm" if wl["gamma"] is not None else "none", "y_dtype": "bf16",
                   "l2": (f"{R} rotating sets of inputs, weight and outputs ({set_mb:.0f} MiB each, "
                          f"{R * set_mb:.0f} MiB in all, L2 126 MB), steps back to back; each set is touched "
                          f"once every {R} steps")},
        "roofline": ({"bound": "tensor", "kernel": klabel,
                      "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                      "frac": round(achieved / peak, 4), "traffic": None,
                      "peak_source": f"{src}: bf16 burst x {ratio:g} (nominal {kind.upper()}/BF16)",
                      "work": work_desc, "avg_launch_us": round(gemm_s * 1e6, 2),
                      "t_compute_us": round(t_compute_us, 2), "t_bytes_us": round(t_bytes_us, 2)}
                     if not hbm_bound else
                     # the bytes take longer than the arithmetic at peak (decode-size rows,
                     # short-K layers with many experts' weights): HBM bound
                     {"bound": "hbm", "kernel": klabel,
                      "achieved": round(wbytes / gemm_s / 1e9, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                      "frac": round(wbytes / gemm_s / 1e9 / pk["hbm_gbs"], 4), "traffic": None,
                      "peak_source": src,
                      "work": ("weight codes E*N*K/2 + sparse-view scales E*N*K/(2b) (E experts) + prepared X "
                               "+ y bytes"),
                      "avg_launch_us": round(gemm_s * 1e6, 2),
                      "t_compute_us": round(t_compute_us, 2), "t_bytes_us": round(t_bytes_us, 2)}),
        "prep": {"gbs_device_amax": round(prep_gbs, 1), "gbs_given_amax": round(given_gbs, 1),
                 "peak_gbs": pk["hbm_gbs"], "frac_given_amax": round(given_gbs / pk["hbm_gbs"], 4),
                 "frac_device_amax": round(prep_gbs / pk["hbm_gbs"], 4),
                 "bytes_per_elem": bpe, "avg_us": round(prep_ms * 1e3, 2), "avg_us_given_amax": round(given_ms * 1e3, 2)},
        "e2e": {"value": round(replica_throughput(world, flops, e2e_steps, e2e_ms), 3), "unit": "TFLOP/s",
                "steps": e2e_steps,
                "mode": "public API per step (pinned host x in, y out), steps pipelined on copy-in / compute / "
                        "copy-out streams with double buffers",
                "h2d_bytes_per_step": int(L.x_host.numel() * L.x_host.element_size() * (2 if L.swiglu else 1)
                                          + (L.rows_host.numel() * 4 if L.gathered else 0)),
                "d2h_bytes_per_step": int(T * N * 2)},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if grouped:
        res["config"]["routed_rows"] = wl["real_rows"]
        res["config"]["experts"] = int(wl["w"].shape[0])
    del L
    torch.cuda.empty_cache()
    return res


def run_sharq(args):
    import torch

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist

    head = measure(args.workload, args.tokens, args.steps, args.warmup, args.steps, dev, pg, world)
    extras = {}
    if args.extra == "all" and args.workload == "q_proj" and not args.tokens:
        for name, tokens in EXTRA:
            key = name if tokens is None else f"{name}_t{tokens}"
            big = name.startswith(("wan", "qwen"))
            extras[key] = measure(name, tokens, min(args.steps, 10 if big else 20), 3,
                                  min(args.steps, 4 if big else 10), dev, pg, world)

    if rank == 0:
        wl = make_workload(args.workload, args.tokens)
        fmt = wl["fmt"]
        traffic = committed_traffic() if args.workload == "q_proj" and not args.tokens else None
        head["roofline"]["traffic"] = traffic
        out = {
            "metric": METRIC,
            "value": head["value"],
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": head["ms_per_step"],
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": (f"{fmt} (e2m1 x {'e4m3 block-16' if fmt == 'nvfp4' else 'e8m0 block-32'} scales, "
                      "fp32 accumulate)"),
            "data": f"synthetic (seeded, shaped like the pages' {args.workload} layer)",
            "config": dict(head["config"], parallelism=f"replicas x{world}"),
            "roofline": head["roofline"],
            "prep": head["prep"],
            "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"],
            "launch_mode": ("the K steps as one CUDA graph (amax, prep, GEMM per step, chained by programmatic "
                            "dependent launch) over rotating sets; prep and GEMM timed alone as graphs of "
                            "back-to-back launches over the same sets; e2e uses direct API calls"),
            "clocks": head["clocks"],
        }
        if extras:
            out["workloads"] = extras
        if not args.no_cpu_baseline and world == 1:
            out["cpu_baseline"], _ = cpu_baseline(args.workload, tokens=args.tokens)
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
        cpu_baseline(args.workload, rows, args.tokens)
    times = []
    base = None
    for _ in range(args.steps):
        base, dt = cpu_baseline(args.workload, rows, args.tokens)
        times.append(dt)
    wl = _ORACLE_SETUP["wl"]
    rows = _ORACLE_SETUP["rows_used"]  # the sample (all rows of a smaller workload)
    total = sum(times)
    value = 2.0 * rows * wl["n"] * wl["k"] * args.steps / total / 1e12
    base["value"] = value
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 prep / f64 GEMM (CPU oracle)",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": wl["desc"], "t": wl["t"], "k": wl["k"], "n": wl["n"], "sample_rows_per_step": rows},
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
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="q_proj")
    ap.add_argument("--tokens", type=int, default=None,
                    help="row count of the q_proj / down_proj shapes (down_proj token sweep: 1, 16, 64, 256)")
    ap.add_argument("--extra", choices=["all", "none"], default="all",
                    help="with the default q_proj headline: also measure every other layer shape ('workloads')")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_sharq(args)


if __name__ == "__main__":
    main()
