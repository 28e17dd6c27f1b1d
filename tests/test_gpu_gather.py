"""Parity of the prepared-row gather (mixture-of-experts routing): preparing each
token once and laying its prepared row out once per routed copy must give exactly
what preparing the routed rows does, and what the oracle gives for them."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparsity_fp4_b200 import sharq, workloads
from gpu_common import assert_prep_equal, readback, to_dev

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
