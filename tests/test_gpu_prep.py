"""Bit-exact parity of the CUDA prep kernel with the CPU oracle.

Small cases span several row tiles, ragged tails and every format x pattern x
norm x input dtype; the configuration cases use the pages' layer shapes at
sizes the oracle finishes in seconds; the full-size cases run the bench's
launch configuration and compare sampled rows."""
import numpy as np
import pytest

import oracle
from activation_sparsity_fp4_b200 import sharq, workloads
from gpu_common import assert_prep_equal, gpu_prepare, readback

pytestmark = pytest.mark.gpu

FMTS = ["mxfp4", "nvfp4"]
PATS = ["2:4", "4:8pair", "8:16", "8:16pair"]


def _x(seed, t, k, outliers=True):
    rng = np.random.default_rng(seed)
    x = (0.5 * rng.standard_t(3, size=(t, k))).astype(np.float32)
    if outliers:
        x[:, rng.permutation(k)[:5]] *= 80.0
    x[:, 3] = 0.0
    x[::7, 10:14] = 1.5  # exact ties inside groups
    return workloads.to_bf16_values(x)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("pat", PATS)
@pytest.mark.parametrize("norm", [False, True])
@pytest.mark.parametrize("xdt", ["f32", "bf16"])
def test_prep_matches_oracle_small(cuda_ok, fmt, pat, norm, xdt):
    t, k = 200, 512
    x = _x(1, t, k)
    gamma = workloads.to_bf16_values(np.random.default_rng(2).uniform(0.5, 1.5, k).astype(np.float32)) if norm else None
    ref = oracle.prepare(x, fmt, pat, gamma=gamma, eps=1e-6)
    p = gpu_prepare(x, xdt, fmt, pat, gamma=gamma, eps=1e-6)
    assert_prep_equal(readback(p), ref, pat)


@pytest.mark.parametrize("k", [256, 768, 2048, 5120, 14336, 16384])
def test_prep_row_lengths(cuda_ok, k):
    # every supported row length class, including multi-row blocks (k = 256, 768)
    # and the largest row (16 warps per row)
    t = 33
    x = _x(3, t, k)
    gamma = workloads.to_bf16_values(np.linspace(0.5, 1.5, k).astype(np.float32))
    ref = oracle.prepare(x, "nvfp4", "4:8pair", gamma=gamma)
    assert_prep_equal(readback(gpu_prepare(x, "bf16", "nvfp4", "4:8pair", gamma=gamma)), ref, "4:8pair")
    ref = oracle.prepare(x, "mxfp4", "2:4")
    assert_prep_equal(readback(gpu_prepare(x, "bf16", "mxfp4", "2:4")), ref, "2:4")


def test_prep_single_row_and_zero_input(cuda_ok):
    for t in (1, 127, 128, 129):
        x = _x(4, t, 256)
        ref = oracle.prepare(x, "nvfp4", "4:8pair")
        assert_prep_equal(readback(gpu_prepare(x, "f32", "nvfp4", "4:8pair")), ref, "4:8pair")
    z = np.zeros((5, 512), np.float32)
    for fmt in FMTS:
        ref = oracle.prepare(z, fmt, "2:4", gamma=np.ones(512, np.float32))
        assert_prep_equal(readback(gpu_prepare(z, "f32", fmt, "2:4", gamma=np.ones(512, np.float32))), ref, "2:4")


@pytest.mark.parametrize("fmt", FMTS)
def test_prep_workspace_gives_same_result(cuda_ok, fmt):
    """With RMSNorm and a device amax the amax pass leaves each row's factor in
    the workspace for the quantization pass; without it prep recomputes it."""
    x = _x(8, 300, 2048)
    gamma = workloads.to_bf16_values(np.random.default_rng(9).uniform(0.5, 1.5, 2048).astype(np.float32))
    ref = oracle.prepare(x, fmt, "4:8pair", gamma=gamma)
    from gpu_common import to_dev
    xd, gd = to_dev(x, "bf16"), to_dev(gamma, "bf16")
    a = sharq.prepare(xd, fmt, "4:8pair", gd, 1e-6, use_workspace=True)
    b = sharq.prepare(xd, fmt, "4:8pair", gd, 1e-6, use_workspace=False)
    sharq.sharq_sync_status()
    assert_prep_equal(readback(a), ref, "4:8pair")
    assert_prep_equal(readback(b), ref, "4:8pair")


def test_prep_caller_amax(cuda_ok):
    x = _x(5, 130, 1024)
    amax = float(np.max(np.abs(x))) * 1.5
    ref = oracle.prepare(x, "nvfp4", "4:8pair", act_amax=amax)
    assert_prep_equal(readback(gpu_prepare(x, "bf16", "nvfp4", "4:8pair", act_amax=amax)), ref, "4:8pair")


def test_prep_padding_rows_are_zero_input(cuda_ok):
    x = _x(6, 3, 256)
    p = gpu_prepare(x, "f32", "mxfp4", "4:8pair")
    g = readback(p, rows=np.arange(3, 128))
    assert np.all(g["bb_codes"] == 0) and np.all(g["res_codes"] == 0)
    assert np.all(g["bb_scales"] == 0) and np.all(g["res_scales"] == 0)
    assert np.all(g["meta"] == 0x44)  # pairs 0 and 1 of every group (ties to the lower index)


# ------------------------------------------------------------ layer configs
def _cfg_case(cfg, t=None):
    x = cfg["x"] if t is None else cfg["x"][:t]
    return x


@pytest.mark.parametrize("name,t", [("tiny", None), ("q_proj", 256), ("down_proj", 64), ("wan", 128),
                                    ("wan_8_16", 128)])
def test_prep_configs(cuda_ok, name, t):
    if name == "tiny":
        cfg = workloads.tiny()
    elif name == "q_proj":
        cfg = workloads.q_proj(t=t)
    elif name == "down_proj":
        cfg = workloads.down_proj(t=t)
    elif name == "wan":
        cfg = workloads.wan(t=t)
    else:
        cfg = workloads.wan(t=t, pat="8:16")
    ref = oracle.prepare(cfg["x"], cfg["fmt"], cfg["pat"], gamma=cfg["gamma"], eps=cfg["eps"], threads=4)
    p = gpu_prepare(cfg["x"], cfg["x_dtype"], cfg["fmt"], cfg["pat"], gamma=cfg["gamma"], eps=cfg["eps"])
    assert_prep_equal(readback(p), ref, cfg["pat"])


def test_prep_down_proj_decode_token_counts(cuda_ok):
    cfg = workloads.down_proj(t=16)
    for t in (1, 16):
        x = cfg["x"][:t]
        ref = oracle.prepare(x, "mxfp4", "2:4")
        assert_prep_equal(readback(gpu_prepare(x, "bf16", "mxfp4", "2:4")), ref, "2:4")


def test_prep_qwen_moe_rows(cuda_ok):
    cfg = workloads.qwen_moe()
    for x in (cfg["x"][:384], cfg["x_down"][:384]):
        ref = oracle.prepare(x, "nvfp4", "4:8pair", threads=4)
        assert_prep_equal(readback(gpu_prepare(x, "bf16", "nvfp4", "4:8pair")), ref, "4:8pair")


@pytest.mark.parametrize("name", ["q_proj", "wan"])
def test_prep_full_size_sampled_rows(cuda_ok, name):
    """The full workload in the launch configuration the bench times; the
    tensor amax must equal the oracle's over all rows, and sampled rows must
    match bit for bit given that amax."""
    cfg = workloads.q_proj() if name == "q_proj" else workloads.wan()
    x, gamma = cfg["x"], cfg["gamma"]
    p = gpu_prepare(x, cfg["x_dtype"], cfg["fmt"], cfg["pat"], gamma=gamma, eps=cfg["eps"])
    amax = oracle.rows_amax(x, gamma, cfg["eps"])
    rows = np.sort(np.random.default_rng(7).choice(x.shape[0], 48, replace=False))
    rows[-1] = x.shape[0] - 1
    g = readback(p, rows=rows)
    assert g["tensor"][0] == np.float32(amax)
    ref = oracle.prepare(x[rows], cfg["fmt"], cfg["pat"], gamma=gamma, eps=cfg["eps"], act_amax=amax)
    assert_prep_equal(g, ref, cfg["pat"])
