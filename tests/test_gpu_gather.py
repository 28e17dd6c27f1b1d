"""Parity of the prepared-row gather (mixture-of-experts routing): preparing each
token once and laying its prepared row out once per routed copy must give exactly
what preparing the routed rows does, and what the oracle gives for them."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparsity_fp4_b200 import sharq, workloads
from gpu_common import assert_close_gemm, assert_prep_equal, readback, to_dev

pytestmark = pytest.mark.gpu

FMTS = ["mxfp4", "nvfp4"]
PATS = ["2:4", "4:8pair", "8:16"]
BUFS = ("meta", "bb_codes", "bb_scales", "res_codes", "res_scales", "tensor")


def _routing(seed, tokens, n_experts, top_k, align=128):
    rng = np.random.default_rng(seed)
    experts = workloads.route_top_k(rng.standard_normal((tokens, n_experts)), top_k)
    return workloads.expert_rows(experts, n_experts, align)


def _tokens(seed, tokens, k):
    rng = np.random.default_rng(seed)
    x = (0.5 * rng.standard_t(3, size=(tokens, k))).astype(np.float32)
    x[rng.random((tokens, k)) < 0.01] *= 40.0  # outlier channels
    return workloads.to_bf16_values(x)


def _routed(x_tok, gather):
    x = np.zeros((gather.size, x_tok.shape[1]), np.float32)
    ok = gather >= 0
    x[ok] = x_tok[gather[ok]]
    return x


def _assert_same_buffers(a: sharq.Prepared, b: sharq.Prepared):
    for name in BUFS:
        ga, gb = getattr(a, name), getattr(b, name)
        assert ga.shape == gb.shape, name
        bad = torch.nonzero(ga != gb)
        assert bad.numel() == 0, f"{name}: {bad.shape[0]} bytes differ, first at {bad[:3].tolist()}"


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("pat", PATS)
def test_gather_equals_prepare_of_routed_rows(cuda_ok, fmt, pat):
    k = 768
    x_tok = _tokens(11, 300, k)
    _, offsets, gather = _routing(12, 300, 8, 2)
    xr = _routed(x_tok, gather)
    src = sharq.prepare(to_dev(x_tok, "bf16"), fmt, pat)
    got = sharq.gather_prepared(src, torch.from_numpy(gather).cuda())
    want = sharq.prepare(to_dev(xr, "bf16"), fmt, pat)
    sharq.sharq_sync_status()
    _assert_same_buffers(got, want)
    assert_prep_equal(readback(got), oracle.prepare(xr, fmt, pat, threads=4), pat)


@pytest.mark.parametrize("t_dst", [1, 127, 129, 600])
def test_gather_ragged_destinations(cuda_ok, t_dst):
    """Destinations of any length; repeated, reversed and zero rows; indices at or past
    the source's row count read as zero rows."""
    k, t_src = 512, 200
    x_tok = _tokens(21, t_src, k)
    rng = np.random.default_rng(22)
    rows = rng.integers(-1, t_src + 3, size=t_dst).astype(np.int64)
    rows[: min(t_dst, 4)] = [t_src - 1, 0, -1, t_src][: min(t_dst, 4)]
    xr = _routed(x_tok, np.where(rows < t_src, rows, -1))
    src = sharq.prepare(to_dev(x_tok, "bf16"), "nvfp4", "4:8pair")
    # the tensor amax of the routed rows is that of the tokens only when the largest
    # value is routed; prepare the routed rows with the tokens' amax so that both agree
    amax = float(np.max(np.abs(x_tok)))
    got = sharq.gather_prepared(src, torch.from_numpy(rows).cuda())
    want = sharq.prepare(to_dev(xr, "bf16"), "nvfp4", "4:8pair", act_amax=amax)
    src2 = sharq.prepare(to_dev(x_tok, "bf16"), "nvfp4", "4:8pair", act_amax=amax)
    got2 = sharq.gather_prepared(src2, torch.from_numpy(rows).cuda())
    sharq.sharq_sync_status()
    _assert_same_buffers(got2, want)
    for name in BUFS[:-1]:  # the device amax and the given one decode to the same tensor scale
        assert torch.equal(getattr(got, name), getattr(got2, name)), name


def test_gather_full_moe_layer_feeds_grouped_gemm(cuda_ok):
    """The gate/up projection of the mixture-of-experts layer at full size: 4096
    tokens, 128 experts, top 8.  The gathered rows are byte-identical to the routed
    preparation, so the grouped GEMM over them gives identical outputs."""
    cfg = workloads.qwen_moe()
    x_tok, gather = cfg["x_tok"], cfg["gather"]
    src = sharq.prepare(to_dev(x_tok, "bf16"), "nvfp4", "4:8pair")
    got = sharq.gather_prepared(src, torch.from_numpy(gather).cuda())
    want = sharq.prepare(to_dev(cfg["x"], "bf16"), "nvfp4", "4:8pair")
    sharq.sharq_sync_status()
    _assert_same_buffers(got, want)
    amax = oracle.rows_amax(x_tok, None, 1e-6)
    sel = np.sort(np.random.default_rng(8).choice(gather.size, 48, replace=False))
    sel[-1] = gather.size - 1
    g = readback(got, rows=sel)
    assert g["tensor"][0] == np.float32(amax)
    ref = oracle.prepare(cfg["x"][sel], "nvfp4", "4:8pair", act_amax=amax)
    assert_prep_equal(g, ref, "4:8pair")


def _expert_weight(seed, experts, n, k):
    rng = np.random.default_rng(seed)
    return workloads.to_bf16_values((rng.standard_normal((experts, n, k)) * 0.02).astype(np.float32))


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_gemm_gathers_rows_itself(cuda_ok, y_dtype):
    """The grouped GEMM reading routed rows by index from the token-prepared
    buffers equals the materialised gather followed by the grouped GEMM, bit for
    bit: small ragged routing (padding rows in every segment), repeated rows, and
    indices at or past the token count (zero rows)."""
    k, n, t_tok, experts = 768, 512, 300, 8
    x_tok = _tokens(31, t_tok, k)
    _, offsets, gather = _routing(32, t_tok, experts, 2)
    rows = gather.copy()
    rows[5] = t_tok + 7   # past the tokens: a zero row
    rows[9] = rows[10]    # the same token twice
    w = _expert_weight(33, experts, n, k)
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), "nvfp4")
    src = sharq.prepare(to_dev(x_tok, "bf16"), "nvfp4", "4:8pair")
    rows_d = torch.from_numpy(rows.astype(np.int32)).cuda()
    off_d = torch.from_numpy(offsets.astype(np.int32)).cuda()
    y_in = sharq.linear_grouped_gather(src, rows_d, wq, off_d, out_dtype=y_dtype)
    routed = sharq.gather_prepared(src, rows_d)
    y_mat = sharq.linear_grouped(routed, wq, off_d, out_dtype=y_dtype)
    sharq.sharq_sync_status()
    bad = torch.nonzero(y_in != y_mat)
    assert bad.numel() == 0, f"{bad.shape[0]} outputs differ, first at {bad[:3].tolist()}"
    # and against the oracle on a few real rows of two experts
    amax = float(src.tensor[0].item())
    assert np.float32(amax) == np.float32(oracle.rows_amax(x_tok))
    yn = y_in.float().cpu().numpy()
    for e in (0, experts - 1):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        sel = np.array([r for r in range(lo, hi) if 0 <= rows[r] < t_tok][:6])
        prep = oracle.prepare(x_tok[rows[sel]], "nvfp4", "4:8pair", act_amax=amax)
        ref = oracle.linear_ref(prep, oracle.quantize_weight(w[e], "nvfp4"))
        if y_dtype == torch.float32:
            assert_close_gemm(yn[sel], ref, f"gathered GEMM, expert {e}")
    # padding rows (index < 0) hold the zero row's output
    pad = np.flatnonzero(rows < 0)
    assert pad.size > 0 and float(y_in[torch.from_numpy(pad).cuda()].abs().max()) == 0.0


def test_gemm_gathers_rows_full_moe_layer(cuda_ok):
    """Qwen3-30B-A3B gate/up at full size (4096 tokens, 128 experts, top 8,
    32768 routed rows): the in-GEMM gather equals gather + grouped GEMM bit for bit."""
    cfg = workloads.qwen_moe()
    x_tok, gather, offsets = cfg["x_tok"], cfg["gather"], cfg["offsets"]
    w = cfg["w_gu"]
    e_, n, k = w.shape
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), "nvfp4")
    src = sharq.prepare(to_dev(x_tok, "bf16"), "nvfp4", "4:8pair")
    rows_d = torch.from_numpy(gather.astype(np.int32)).cuda()
    off_d = torch.from_numpy(offsets.astype(np.int32)).cuda()
    y_in = sharq.linear_grouped_gather(src, rows_d, wq, off_d)
    y_mat = sharq.linear_grouped(sharq.gather_prepared(src, rows_d), wq, off_d)
    sharq.sharq_sync_status()
    assert torch.equal(y_in, y_mat)
