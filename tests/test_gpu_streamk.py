"""Stream-K form of the CTA-pair GEMM (sharq_linear_ws): K loops of all tiles
split evenly over the SM pairs, partial sums added by the pair that holds each
tile's first K tile.  Results match the oracle like the whole-tile form, agree
with it up to the order of the fp32 partial sums, and leave the workspace
counters as they found them."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparsity_fp4_b200 import sharq, workloads
from gpu_common import assert_close_gemm, gpu_prepare, to_dev

pytestmark = pytest.mark.gpu


def _w(seed, n, k, scale=0.02):
    rng = np.random.default_rng(seed)
    return workloads.to_bf16_values((rng.standard_normal((n, k)) * scale).astype(np.float32))


def _x(seed, t, k):
    rng = np.random.default_rng(seed)
    x = (0.5 * rng.standard_t(3, size=(t, k))).astype(np.float32)
    x[:, rng.permutation(k)[:6]] *= 60.0
    return workloads.to_bf16_values(x)


def _counters(ws: torch.Tensor) -> tuple[np.ndarray, np.ndarray]:
    """The workspace's fixed counter region: stream-K counters (16 per SM pair)
    at the start, then one split-K counter per SM."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    words = ws[: (sms // 2) * 64 + sms * 4].cpu().numpy().view(np.uint32)
    return words[: (sms // 2) * 16], words[(sms // 2) * 16:]


def _flags(ws: torch.Tensor) -> np.ndarray:
    return _counters(ws)[0]


# (t, n, k): few tiles with long K loops, where the split applies: 16 tiles of
# 64 K tiles (each spread over ~5 pairs), and 500 ragged rows in 16 tiles
SHAPES = [(256, 4096, 16384), (500, 2048, 16384)]


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
@pytest.mark.parametrize("shape", SHAPES)
def test_stream_k_matches_oracle_and_whole_tiles(cuda_ok, fmt, shape):
    """fp32 output against fp64 and against the whole-tile form; bf16 output
    equal to the fp32 output rounded to bf16 (same split, same sums)."""
    t, n, k = shape
    x, w = _x(31, t, k), _w(32, n, k)
    p = gpu_prepare(x, "bf16", fmt, "4:8pair")
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), fmt)
    ws = sharq.linear_workspace()
    y_sk = sharq.linear(p, wq, out_dtype=torch.float32, workspace=ws)
    y_bf = sharq.linear(p, wq, out_dtype=torch.bfloat16, workspace=ws)
    y_wt = sharq.linear(p, wq, out_dtype=torch.float32)
    sharq.sharq_sync_status()
    prep = oracle.prepare(x, fmt, "4:8pair", threads=4)
    ref = oracle.linear_ref(prep, oracle.quantize_weight(w, fmt))
    assert_close_gemm(y_sk.cpu().numpy(), ref, f"stream-K {fmt} {shape}")
    assert_close_gemm(y_sk.cpu().numpy(), y_wt.double().cpu().numpy(), "stream-K vs whole tiles")
    assert torch.equal(y_bf, y_sk.to(torch.bfloat16)), "bf16 output != fp32 output rounded to bf16"
    assert (_flags(ws) % 2 == 0).all(), "a partial-sum counter was left odd"


def test_stream_k_repeated_calls_are_deterministic(cuda_ok):
    """The same workspace serves call after call (counters return to even); the
    fixed split gives the same bits every time."""
    t, n, k = SHAPES[0]
    x, w = _x(33, t, k), _w(34, n, k)
    p = gpu_prepare(x, "bf16", "nvfp4", "4:8pair")
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), "nvfp4")
    ws = sharq.linear_workspace()
    ys = [sharq.linear(p, wq, workspace=ws).clone() for _ in range(4)]
    sharq.sharq_sync_status()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    f = _flags(ws)
    assert (f % 2 == 0).all() and f.max() > 0  # used, and every partial consumed


def test_stream_k_not_used_on_the_q_proj_shape(cuda_ok):
    """128 tiles of 16 K tiles (the bench's q_proj launch) keep whole tiles: the
    workspace changes nothing and stays untouched."""
    cfg = workloads.q_proj()
    p = gpu_prepare(cfg["x"], "bf16", "nvfp4", "4:8pair", gamma=cfg["gamma"])
    wq = sharq.FP4Weight.quantize(to_dev(cfg["w"], "bf16"), "nvfp4")
    ws = sharq.linear_workspace()
    a, b = sharq.linear(p, wq, workspace=ws), sharq.linear(p, wq)
    sharq.sharq_sync_status()
    assert torch.equal(a, b)
    assert (_flags(ws) == 0).all()


def test_stream_k_falls_back_where_it_does_not_apply(cuda_ok):
    """Grouped, single-CTA kinds and whole waves ignore the workspace (same bits as sharq_linear)."""
    x, w = _x(35, 300, 1024), _w(36, 512, 1024)  # 384 padded rows: single-CTA kernel
    p = gpu_prepare(x, "bf16", "mxfp4", "2:4")
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), "mxfp4")
    ws = sharq.linear_workspace()
    a, b = sharq.linear(p, wq, workspace=ws), sharq.linear(p, wq)
    sharq.sharq_sync_status()
    assert torch.equal(a, b)
    assert (_flags(ws) == 0).all()


# few tiles with long K (decode-size row counts), K split into slices over the
# SMs and the slices summed in a fixed order: 65..256 rows on the single-CTA
# kernel (workspace slots, the last slice adds them), 2..64 rows on the few-row
# kernel (a cluster per weight tile), 1 row on the CUDA cores
SPLIT_CASES = [("mxfp4", "2:4", 1, 4096, 14336), ("mxfp4", "2:4", 16, 4096, 14336),
               ("mxfp4", "2:4", 64, 4096, 14336), ("mxfp4", "2:4", 128, 4096, 14336),
               ("mxfp4", "2:4", 256, 4096, 14336),
               ("nvfp4", "4:8pair", 16, 4096, 8192), ("nvfp4", "8:16", 100, 1024, 8192),
               ("mxfp4", "4:8pair", 40, 2048, 8192)]


@pytest.mark.parametrize("fmt,pat,t,n,k", SPLIT_CASES)
def test_split_k_single_cta_matches_oracle(cuda_ok, fmt, pat, t, n, k):
    """fp32 output against fp64 and the unsplit kernel; bf16 output equal to the
    fp32 output rounded to bf16; a second call gives the same bits (the slice
    sums are added in a fixed order and every counter is reset)."""
    x, w = _x(40 + t, t, k), _w(41, n, k)
    p = gpu_prepare(x, "bf16", fmt, pat)
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), fmt)
    ws = sharq.linear_workspace()
    y1 = sharq.linear(p, wq, out_dtype=torch.float32, workspace=ws).clone()
    y2 = sharq.linear(p, wq, out_dtype=torch.float32, workspace=ws).clone()
    yb = sharq.linear(p, wq, out_dtype=torch.bfloat16, workspace=ws)
    y0 = sharq.linear(p, wq, out_dtype=torch.float32)
    sharq.sharq_sync_status()
    prep = oracle.prepare(x, fmt, pat, threads=4)
    ref = oracle.linear_ref(prep, oracle.quantize_weight(w, fmt))
    assert_close_gemm(y1.cpu().numpy(), ref, f"split-K {fmt} {pat} t={t}")
    assert_close_gemm(y1.cpu().numpy(), y0.double().cpu().numpy(), "split-K vs unsplit")
    assert torch.equal(y1, y2), "split-K is not reproducible"
    assert torch.equal(yb, y1.to(torch.bfloat16)), "bf16 output != fp32 output rounded to bf16"


def test_one_workspace_serves_every_shape_in_turn(cuda_ok):
    """One workspace kept per device for prefill and decode sizes: split-K at 256
    rows, then 16 rows, then 256 rows again (MXFP4 2:4, k = 14336), then a
    stream-K shape and split-K once more.  The partial sums of one call never
    land on the counters of another (they sit in a fixed region before every
    data slot), so every output matches the unsplit kernel, a repeated shape
    gives the same bits, and every counter is back at zero."""
    n, k = 4096, 14336
    w = _w(50, n, k)
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), "mxfp4")
    preps = {t: gpu_prepare(_x(51 + t, t, k), "bf16", "mxfp4", "2:4") for t in (256, 16)}
    xs, ws_ = _x(53, 256, 16384), _w(54, 4096, 16384)
    psk = gpu_prepare(xs, "bf16", "nvfp4", "4:8pair")
    wsk = sharq.FP4Weight.quantize(to_dev(ws_, "bf16"), "nvfp4")
    ws = sharq.linear_workspace()
    outs = []
    for t in (256, 16, 256):
        outs.append((t, sharq.linear(preps[t], wq, out_dtype=torch.float32, workspace=ws).clone()))
    y_sk = sharq.linear(psk, wsk, out_dtype=torch.float32, workspace=ws).clone()
    outs.append((16, sharq.linear(preps[16], wq, out_dtype=torch.float32, workspace=ws).clone()))
    sharq.sharq_sync_status()
    for t, y in outs:
        y0 = sharq.linear(preps[t], wq, out_dtype=torch.float32)
        sharq.sharq_sync_status()
        assert_close_gemm(y.cpu().numpy(), y0.double().cpu().numpy(), f"reused workspace, t={t}")
    assert torch.equal(outs[0][1], outs[2][1]), "t=256 after t=16 changed bits"
    assert torch.equal(outs[1][1], outs[3][1]), "t=16 after the stream-K call changed bits"
    y0 = sharq.linear(psk, wsk, out_dtype=torch.float32)
    sharq.sharq_sync_status()
    assert_close_gemm(y_sk.cpu().numpy(), y0.double().cpu().numpy(), "stream-K on a reused workspace")
    flags, split_cnt = _counters(ws)
    assert (flags % 2 == 0).all() and flags.max() > 0, "stream-K counters not back to even"
    assert (split_cnt == 0).all(), "a split-K counter was left set"
