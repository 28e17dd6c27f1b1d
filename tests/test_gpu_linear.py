"""Parity of the weight quantizer (bit-exact) and of the fused sparse+dense
FP4 GEMM (rel. Frobenius <= 1e-4 and |d| <= 1e-3 max|Y|) with the oracle's
fp64 product of the dequantized operands."""
import numpy as np
import pytest
import torch

import oracle
from _layout import untile_scales
from activation_sparsity_fp4_b200 import sharq, workloads
from gpu_common import assert_close_gemm, gpu_prepare, readback, assert_prep_equal, to_dev

pytestmark = pytest.mark.gpu

LINEAR_CASES = [("nvfp4", "4:8pair"), ("nvfp4", "8:16"), ("mxfp4", "4:8pair"), ("mxfp4", "8:16"), ("mxfp4", "2:4"),
                ("nvfp4", "8:16pair"), ("mxfp4", "8:16pair")]


def _w(seed, n, k, scale=0.02):
    rng = np.random.default_rng(seed)
    return workloads.to_bf16_values((rng.standard_normal((n, k)) * scale).astype(np.float32))


def _x(seed, t, k):
    rng = np.random.default_rng(seed)
    x = (0.5 * rng.standard_t(3, size=(t, k))).astype(np.float32)
    x[:, rng.permutation(k)[:6]] *= 60.0
    return workloads.to_bf16_values(x)


def gpu_weight(w, w_dtype, fmt):
    wq = sharq.FP4Weight.quantize(to_dev(w, w_dtype), fmt)
    sharq.sharq_sync_status()
    return wq


def weight_readback(wq):
    n, k = wq.n, wq.k
    b = 16 if wq.fmt == sharq.NVFP4 else 32
    codes = wq.codes.cpu().numpy()[: n * k // 2].reshape(n, k // 2)
    dense = untile_scales(wq.scales_dense.cpu().numpy(), n, k // b)
    sparse = untile_scales(wq.scales_sparse.cpu().numpy(), n, k // (2 * b))
    return codes, dense, sparse, wq.tensor.cpu().numpy()


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("wdt", ["f32", "bf16"])
def test_weight_quantization_bit_exact(cuda_ok, fmt, wdt):
    w = _w(1, 512, 1024)
    ref = oracle.quantize_weight(w, fmt)
    codes, dense, sparse, tens = weight_readback(gpu_weight(w, wdt, fmt))
    np.testing.assert_array_equal(codes, ref["codes"])
    np.testing.assert_array_equal(sparse, ref["scales"])
    np.testing.assert_array_equal(dense[:, 0::2], ref["scales"])
    np.testing.assert_array_equal(dense[:, 1::2], ref["scales"])
    np.testing.assert_array_equal(tens, ref["tensor"])


def test_weight_quantization_stacked_experts(cuda_ok):
    w = np.stack([_w(10 + e, 256, 512, scale=0.01 * (e + 1)) for e in range(3)])
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), "nvfp4")
    sharq.sharq_sync_status()
    c, d, s = sharq.sharq_weight_sizes(256, 512, "nvfp4")
    for e in range(3):
        ref = oracle.quantize_weight(w[e], "nvfp4")
        np.testing.assert_array_equal(wq.codes.cpu().numpy()[e * c:(e + 1) * c].reshape(256, 256), ref["codes"])
        np.testing.assert_array_equal(untile_scales(wq.scales_sparse.cpu().numpy()[e * s:(e + 1) * s], 256, 16),
                                      ref["scales"])
        np.testing.assert_array_equal(wq.tensor.cpu().numpy()[3 * e:3 * e + 3], ref["tensor"])


def _run_linear(x, w, fmt, pat, gamma=None, out_dtype=torch.float32, paths=3, x_dtype="bf16", w_dtype="bf16"):
    p = gpu_prepare(x, x_dtype, fmt, pat, gamma=gamma)
    wq = gpu_weight(w, w_dtype, fmt)
    y = sharq.linear(p, wq, out_dtype=out_dtype, paths=paths)
    sharq.sharq_sync_status()
    return p, wq, y.float().cpu().numpy()


def _ref(x, w, fmt, pat, gamma=None, rows=None, act_amax=0.0):
    prep = oracle.prepare(x, fmt, pat, gamma=gamma, act_amax=act_amax, threads=4)
    wq = oracle.quantize_weight(w, fmt)
    return prep, wq


@pytest.mark.parametrize("fmt,pat", LINEAR_CASES)
def test_linear_matches_oracle(cuda_ok, fmt, pat):
    t, k, n = 200, 1024, 512  # 2 row tiles (ragged), 4 K tiles, 2 column tiles
    x, w = _x(2, t, k), _w(3, n, k)
    _, _, y = _run_linear(x, w, fmt, pat)
    prep, wq = _ref(x, w, fmt, pat)
    assert_close_gemm(y, oracle.linear_ref(prep, wq), f"{fmt} {pat}")


@pytest.mark.parametrize("fmt,pat", LINEAR_CASES)
def test_linear_each_path_separately(cuda_ok, fmt, pat):
    """Sparse backbone GEMM alone and dense residual GEMM alone, against the
    oracle's two partial products (this localizes a wrong metadata or scale
    view to one path)."""
    t, k, n = 128, 512, 256
    x, w = _x(4, t, k), _w(5, n, k)
    prep, wq = _ref(x, w, fmt, pat)
    bu, ru = oracle.decode_prepared(prep)
    wu = oracle.decode_weight(wq)
    alpha = float(prep["tensor"][2]) * float(wq["tensor"][2])
    for paths, ref in ((1, alpha * bu @ wu.T), (2, alpha * ru @ wu.T)):
        _, _, y = _run_linear(x, w, fmt, pat, paths=paths)
        assert_close_gemm(y, ref, f"{fmt} {pat} paths={paths}")


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_linear_cta_pairs(cuda_ok, fmt):
    """Row counts whose 128-row padding is a multiple of 256 run on CTA pairs
    (a 256 x 256 tile per pair of SMs): several pair tiles in M and N, ragged
    rows, fewer K tiles than pipeline stages, and each path alone."""
    t, k, n = 700, 768, 768  # padded to 768 rows = 3 pair tiles, 3 column tiles, 3 K tiles
    x, w = _x(8, t, k), _w(9, n, k)
    prep, wq = _ref(x, w, fmt, "4:8pair")
    _, _, y = _run_linear(x, w, fmt, "4:8pair")
    assert_close_gemm(y, oracle.linear_ref(prep, wq), f"{fmt} 4:8pair pairs")
    bu, ru = oracle.decode_prepared(prep)
    wu = oracle.decode_weight(wq)
    alpha = float(prep["tensor"][2]) * float(wq["tensor"][2])
    for paths, ref in ((1, alpha * bu @ wu.T), (2, alpha * ru @ wu.T)):
        _, _, y = _run_linear(x, w, fmt, "4:8pair", paths=paths)
        assert_close_gemm(y, ref, f"{fmt} 4:8pair pairs paths={paths}")


def _bf16_round(a: np.ndarray) -> np.ndarray:
    """fp32 -> the nearest bf16 value (ties to even), as float32."""
    return workloads.to_bf16_values(np.asarray(a, dtype=np.float32))


@pytest.mark.parametrize("fmt,pat", LINEAR_CASES)
@pytest.mark.parametrize("t", [300, 700])
def test_linear_bf16_output_equals_rounded_fp32(cuda_ok, fmt, pat, t):
    """bf16 output (written through shared memory by TMA stores) equals the fp32
    output of the same operands rounded to bf16, element for element, on both
    GEMM kernels (t=300 pads to 384 rows: single-CTA; t=700 pads to 768: CTA
    pairs for 4:8 pair) with several column tiles; rows past t stay untouched."""
    k, n = 512, 768
    x, w = _x(10, t, k), _w(11, n, k)
    p = gpu_prepare(x, "bf16", fmt, pat)
    wq = gpu_weight(w, "bf16", fmt)
    y32 = sharq.linear(p, wq, out_dtype=torch.float32)
    guard = torch.full((t + 64, n), 7.0, dtype=torch.bfloat16, device="cuda")
    sharq.linear(p, wq, out=guard[:t])
    sharq.sharq_sync_status()
    y16 = guard[:t].float().cpu().numpy()
    ref = _bf16_round(y32.cpu().numpy())
    bad = np.argwhere(y16 != ref)
    assert bad.size == 0, f"{fmt} {pat} t={t}: {len(bad)} bf16 outputs differ, first {bad[:3].tolist()}"
    assert bool((guard[t:] == 7.0).all()), "rows past t were written"


def test_linear_grouped_bf16_output_equals_rounded_fp32(cuda_ok):
    """The grouped launch's bf16 output equals its fp32 output rounded to bf16."""
    rng = np.random.default_rng(12)
    experts, k, n = 3, 512, 512
    counts = [128, 256, 128]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    t = int(offsets[-1])
    x = _x(13, t, k)
    w = workloads.to_bf16_values((rng.standard_normal((experts, n, k)) * 0.02).astype(np.float32))
    p = gpu_prepare(x, "bf16", "nvfp4", "4:8pair")
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), "nvfp4")
    off_dev = torch.from_numpy(offsets).cuda()
    y32 = sharq.linear_grouped(p, wq, off_dev, out_dtype=torch.float32)
    y16 = sharq.linear_grouped(p, wq, off_dev, out_dtype=torch.bfloat16)
    sharq.sharq_sync_status()
    ref = _bf16_round(y32.cpu().numpy())
    bad = np.argwhere(y16.float().cpu().numpy() != ref)
    assert bad.size == 0, f"grouped: {len(bad)} bf16 outputs differ, first {bad[:3].tolist()}"


def test_linear_bf16_output_and_single_row(cuda_ok):
    k, n = 512, 256
    w = _w(6, n, k)
    for t in (1, 129):
        x = _x(7, t, k)
        _, _, y = _run_linear(x, w, "nvfp4", "4:8pair", out_dtype=torch.bfloat16)
        prep, wq = _ref(x, w, "nvfp4", "4:8pair")
        ref = oracle.linear_ref(prep, wq)
        # bf16 output: the rounding of the output itself dominates (2^-9 relative)
        err = np.linalg.norm(y - ref) / np.linalg.norm(ref)
        assert err < 4e-3


@pytest.mark.parametrize("pat", ["2:4", "4:8pair"])
def test_linear_tiny_config(cuda_ok, pat):
    """The Tiny case (16 x 256 fp32, channels 3 and 77 x40, MXFP4); 2:4 is the
    configuration as specified, 4:8 pair exercises the other sparse kind."""
    cfg = workloads.tiny()
    _, _, y = _run_linear(cfg["x"], cfg["w"], "mxfp4", pat, x_dtype="f32", w_dtype="f32")
    prep, wq = _ref(cfg["x"], cfg["w"], "mxfp4", pat)
    assert_close_gemm(y, oracle.linear_ref(prep, wq), f"tiny {pat}")


def test_nvfp4_2_4_linear_is_unsupported(cuda_ok):
    p = gpu_prepare(_x(9, 16, 256), "bf16", "nvfp4", "2:4")
    wq = gpu_weight(_w(9, 256, 256), "bf16", "nvfp4")
    with pytest.raises(sharq.SharqError) as ei:
        sharq.linear(p, wq)
    assert ei.value.status == 2


@pytest.mark.parametrize("t", [1, 16, 64, 256])
def test_linear_down_proj_token_sweep(cuda_ok, t):
    """Llama-3.1-8B down_proj (14336 -> 4096), MXFP4 2:4, decode-size token counts."""
    cfg = workloads.down_proj(t=t)
    _, _, y = _run_linear(cfg["x"], cfg["w"], "mxfp4", "2:4")
    prep, wq = _ref(cfg["x"], cfg["w"], "mxfp4", "2:4")
    assert_close_gemm(y, oracle.linear_ref(prep, wq), f"down_proj t={t}")


def test_linear_down_proj_2048_sampled_rows(cuda_ok):
    cfg = workloads.down_proj()
    _, _, y = _run_linear(cfg["x"], cfg["w"], "mxfp4", "2:4", out_dtype=torch.float32)
    rows = np.sort(np.random.default_rng(11).choice(2048, 48, replace=False))
    prep = oracle.prepare(cfg["x"][rows], "mxfp4", "2:4")
    wq = oracle.quantize_weight(cfg["w"], "mxfp4")
    assert_close_gemm(y[rows], oracle.linear_ref(prep, wq), "down_proj sampled rows")


@pytest.mark.parametrize("pat", ["4:8pair", "8:16", "8:16pair"])
def test_linear_wan_full_size_sampled_rows(cuda_ok, pat):
    """Wan2.2 DiT linear (32768 x 5120 -> 5120), NVFP4 with RMSNorm, 4:8 pair, 8:16
    and 8:16 re-packed into the 4:8 pair layout."""
    cfg = workloads.wan(pat=pat)
    p, _, y = _run_linear(cfg["x"], cfg["w"], "nvfp4", pat, gamma=cfg["gamma"], out_dtype=torch.float32)
    rows = np.sort(np.random.default_rng(12).choice(32768, 24, replace=False))
    amax = float(p.tensor[0].item())
    assert np.float32(amax) == np.float32(oracle.rows_amax(cfg["x"], cfg["gamma"])), "device amax differs"
    prep = oracle.prepare(cfg["x"][rows], "nvfp4", pat, gamma=cfg["gamma"], act_amax=amax)
    wq = oracle.quantize_weight(cfg["w"], "nvfp4")
    assert_close_gemm(y[rows], oracle.linear_ref(prep, wq), f"wan {pat} sampled rows")


@pytest.mark.parametrize("which", ["gate_up", "down"])
def test_linear_grouped_qwen_moe(cuda_ok, which):
    """Qwen3-30B-A3B experts: 128 stacked NVFP4 weights, routed rows grouped by
    expert (segments padded to 128 rows), one grouped launch; rows sampled from
    several experts against the oracle with each row's own expert weight."""
    cfg = workloads.qwen_moe()
    x = cfg["x"] if which == "gate_up" else cfg["x_down"]
    w = cfg["w_gu"] if which == "gate_up" else cfg["w_d"]
    offsets = cfg["offsets"]
    p = gpu_prepare(x, "bf16", "nvfp4", "4:8pair")
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), "nvfp4")
    off_dev = torch.from_numpy(offsets.astype(np.int32)).cuda()
    y = sharq.linear_grouped(p, wq, off_dev, out_dtype=torch.float32)
    sharq.sharq_sync_status()
    y = y.cpu().numpy()
    amax = float(p.tensor[0].item())
    # the device-computed tensor amax over all routed rows must be the oracle's
    # before it is handed to the oracle for the sampled rows
    assert np.float32(amax) == np.float32(oracle.rows_amax(x)), "MoE device amax differs from the oracle"
    rng = np.random.default_rng(13)
    experts = [0, 5, 64, 127] + list(rng.choice(128, 4, replace=False))
    for e in experts:
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        rows = np.unique(np.concatenate([[lo, hi - 1], rng.integers(lo, hi, 6)]))
        prep = oracle.prepare(x[rows], "nvfp4", "4:8pair", act_amax=amax)
        wqe = oracle.quantize_weight(w[e], "nvfp4")
        assert_close_gemm(y[rows], oracle.linear_ref(prep, wqe), f"moe {which} expert {e}")


def test_linear_q_proj_full_size_sampled_rows(cuda_ok):
    """Llama-3.1-8B q_proj shape (2048 x 4096 -> 4096), NVFP4 4:8 pair with
    RMSNorm, in the bench's launch configuration; 64 sampled rows against fp64."""
    cfg = workloads.q_proj()
    p, wq_gpu, y = _run_linear(cfg["x"], cfg["w"], "nvfp4", "4:8pair", gamma=cfg["gamma"])
    rows = np.sort(np.random.default_rng(8).choice(2048, 64, replace=False))
    amax = float(p.tensor[0].item())
    assert np.float32(amax) == np.float32(oracle.rows_amax(cfg["x"], cfg["gamma"])), "device amax differs"
    prep = oracle.prepare(cfg["x"][rows], "nvfp4", "4:8pair", gamma=cfg["gamma"], act_amax=amax)
    wq = oracle.quantize_weight(cfg["w"], "nvfp4")
    assert_close_gemm(y[rows], oracle.linear_ref(prep, wq), "q_proj sampled rows")


SWAP_CASES = [("nvfp4", "4:8pair"), ("nvfp4", "8:16"), ("nvfp4", "8:16pair"), ("mxfp4", "2:4"),
              ("mxfp4", "4:8pair"), ("mxfp4", "8:16")]


@pytest.mark.parametrize("fmt,pat", SWAP_CASES)
@pytest.mark.parametrize("t", [2, 5, 32, 33, 64, 65])
@pytest.mark.parametrize("k", [512, 2048])
def test_linear_few_rows_weight_as_operand_a(cuda_ok, fmt, pat, t, k):
    """2..64 rows: the weight tile is the 128-row MMA operand and the rows the
    narrow one, padded to 32 (t <= 32) or 64 (backbone expanded on chip); 65
    rows: the activation-as-A kernels next to it.  k = 512: one K slice per
    weight tile; k = 2048: four
    slices, a cluster per tile reduced through distributed shared memory.
    Against fp64; bf16 = rounded fp32; results repeat bit for bit, with or
    without a workspace."""
    n = 1024
    x, w = _x(60 + t, t, k), _w(61, n, k)
    p = gpu_prepare(x, "bf16", fmt, pat)
    wq = gpu_weight(w, "bf16", fmt)
    ws = sharq.linear_workspace()
    y1 = sharq.linear(p, wq, out_dtype=torch.float32).clone()
    y2 = sharq.linear(p, wq, out_dtype=torch.float32, workspace=ws).clone()
    y3 = sharq.linear(p, wq, out_dtype=torch.float32, workspace=ws).clone()
    yb = sharq.linear(p, wq, out_dtype=torch.bfloat16, workspace=ws)
    sharq.sharq_sync_status()
    prep, wqo = _ref(x, w, fmt, pat)
    ref = oracle.linear_ref(prep, wqo)
    assert_close_gemm(y1.cpu().numpy(), ref, f"{fmt} {pat} t={t} k={k}, no workspace")
    assert_close_gemm(y2.cpu().numpy(), ref, f"{fmt} {pat} t={t} k={k}, workspace")
    assert torch.equal(y2, y3), "the K split is not reproducible"
    if t <= 64:
        assert torch.equal(y1, y2), "the few-row kernel must not depend on the workspace"
    assert torch.equal(yb, y2.to(torch.bfloat16)), "bf16 output != fp32 output rounded to bf16"


# cluster sizes of the few-row kernel's K split: slices = min(SMs / weight tiles,
# K tiles / 2, 8), fewer when not every cluster would be resident at once
CLUSTER_CASES = [(1024, 4096, 8), (5120, 2048, 3), (2048, 1024, 2)]


@pytest.mark.parametrize("n,k,slices", CLUSTER_CASES)
def test_few_rows_cluster_sizes(cuda_ok, n, k, slices):
    """16 rows, MXFP4 2:4: the K slices of each weight tile summed in slice order
    inside a cluster of 8, 3 and 2 CTAs (on a 148-SM part), against fp64; two
    calls give the same bits."""
    t = 16
    x, w = _x(70 + slices, t, k), _w(71, n, k)
    p = gpu_prepare(x, "bf16", "mxfp4", "2:4")
    wq = gpu_weight(w, "bf16", "mxfp4")
    y1 = sharq.linear(p, wq, out_dtype=torch.float32).clone()
    y2 = sharq.linear(p, wq, out_dtype=torch.float32).clone()
    sharq.sharq_sync_status()
    prep, wqo = _ref(x, w, "mxfp4", "2:4")
    assert_close_gemm(y1.cpu().numpy(), oracle.linear_ref(prep, wqo), f"n={n} k={k}, {slices} slices")
    assert torch.equal(y1, y2)
