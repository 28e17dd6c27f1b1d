"""GPU parity of the SwiGLU form of the preprocessing (sharq_prepare_swiglu:
h = SiLU(gate) * up formed inside the kernel) against the oracle, bit for bit,
and of the layer on its output."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparsity_fp4_b200 import sharq, workloads
from gpu_common import assert_close_gemm, assert_prep_equal, readback, to_dev

pytestmark = pytest.mark.gpu


def _inputs(seed, t, k):
    rng = np.random.default_rng(seed)
    gate = workloads.to_bf16_values(rng.standard_normal((t, k)).astype(np.float32) * 2)
    up = workloads.to_bf16_values(rng.standard_normal((t, k)).astype(np.float32))
    up[:, rng.permutation(k)[:6]] *= 40.0
    up = workloads.to_bf16_values(up)
    gate[0, :8] = [0.0, -0.0, 30.0, -30.0, -120.0, 95.0, 1e-30, -1e-30]  # exp range edges
    return workloads.to_bf16_values(gate), up


@pytest.mark.parametrize("fmt,pat", [("nvfp4", "4:8pair"), ("mxfp4", "2:4"), ("mxfp4", "4:8pair"),
                                     ("nvfp4", "8:16"), ("mxfp4", "8:16")])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_prepare_swiglu_bit_exact(cuda_ok, fmt, pat, dt):
    gate, up = _inputs(21, 200, 1024)
    p = sharq.prepare_swiglu(to_dev(gate, dt), to_dev(up, dt), fmt, pat)
    sharq.sharq_sync_status()
    assert_prep_equal(readback(p), oracle.prepare_swiglu(gate, up, fmt, pat, threads=4), pat)


def test_prepare_swiglu_caller_amax_and_long_rows(cuda_ok):
    gate, up = _inputs(22, 40, 14336)  # down_proj row length
    ref = oracle.prepare_swiglu(gate, up, "nvfp4", "4:8pair", threads=4)
    amax = float(ref["tensor"][0])
    p = sharq.prepare_swiglu(to_dev(gate, "bf16"), to_dev(up, "bf16"), "nvfp4", "4:8pair", act_amax=amax)
    sharq.sharq_sync_status()
    assert_prep_equal(readback(p), ref, "4:8pair")
    p = sharq.prepare_swiglu(to_dev(gate, "bf16"), to_dev(up, "bf16"), "mxfp4", "2:4")
    sharq.sharq_sync_status()
    assert_prep_equal(readback(p), oracle.prepare_swiglu(gate, up, "mxfp4", "2:4", threads=4), "2:4")


def test_down_proj_swiglu_layer_sampled_rows(cuda_ok):
    """The down_proj shape from its gate and up inputs (t=256, MXFP4 2:4): prepared
    rows bit-exact and the GEMM within the layer tolerance on sampled rows."""
    cfg = workloads.down_proj(t=256)
    gate, up, w = cfg["gate"], cfg["up"], cfg["w"]
    p = sharq.prepare_swiglu(to_dev(gate, "bf16"), to_dev(up, "bf16"), "mxfp4", "2:4")
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), "mxfp4")
    y = sharq.linear(p, wq, out_dtype=torch.float32)
    sharq.sharq_sync_status()
    rows = np.array([0, 1, 77, 128, 200, 255])
    ref = oracle.prepare_swiglu(gate[rows], up[rows], "mxfp4", "2:4", threads=4)
    assert_prep_equal(readback(p, rows=rows), ref, "2:4")
    assert_close_gemm(y.cpu().numpy()[rows], oracle.linear_ref(ref, oracle.quantize_weight(w, "mxfp4")),
                      "down_proj swiglu")
