"""The 1-4 row form of the layer's two products (CUDA cores, weight stream):
within the GEMM tolerance of the fp64 oracle for every supported format and
pattern, each path alone, and bf16 output equal to the fp32 output rounded."""
import numpy as np
import pytest
import torch

import oracle
from activation_sparsity_fp4_b200 import sharq, workloads
from gpu_common import assert_close_gemm, gpu_prepare, to_dev

pytestmark = pytest.mark.gpu

CASES = [("nvfp4", "4:8pair"), ("nvfp4", "8:16"), ("mxfp4", "4:8pair"), ("mxfp4", "8:16"), ("mxfp4", "2:4")]


def _w(seed, n, k, scale=0.02):
    rng = np.random.default_rng(seed)
    return workloads.to_bf16_values((rng.standard_normal((n, k)) * scale).astype(np.float32))


def _x(seed, t, k):
    rng = np.random.default_rng(seed)
    x = (0.5 * rng.standard_t(3, size=(t, k))).astype(np.float32)
    x[:, rng.permutation(k)[:6]] *= 60.0
    return workloads.to_bf16_values(x)


@pytest.mark.parametrize("fmt,pat", CASES)
@pytest.mark.parametrize("t", [1, 2, 3, 4])
def test_gemv_matches_oracle(cuda_ok, fmt, pat, t):
    k, n = 2304, 512  # K chunks of 2048 (1-2 rows) or 1024 (3-4 rows) and a partial one; 32 blocks of 8 warps x 2 rows
    x, w = _x(50 + t, t, k), _w(51, n, k)
    p = gpu_prepare(x, "bf16", fmt, pat)
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), fmt)
    y = sharq.linear(p, wq, out_dtype=torch.float32)
    yb = sharq.linear(p, wq, out_dtype=torch.bfloat16)
    sharq.sharq_sync_status()
    prep = oracle.prepare(x, fmt, pat)
    wqo = oracle.quantize_weight(w, fmt)
    assert_close_gemm(y.cpu().numpy(), oracle.linear_ref(prep, wqo), f"gemv {fmt} {pat} t={t}")
    assert torch.equal(yb, y.to(torch.bfloat16))
    bu, ru = oracle.decode_prepared(prep)
    wu = oracle.decode_weight(wqo)
    alpha = float(prep["tensor"][2]) * float(wqo["tensor"][2])
    for paths, ref in ((1, alpha * bu @ wu.T), (2, alpha * ru @ wu.T)):
        yp = sharq.linear(p, wq, out_dtype=torch.float32, paths=paths)
        sharq.sharq_sync_status()
        assert_close_gemm(yp.cpu().numpy(), ref, f"gemv {fmt} {pat} t={t} paths={paths}")


@pytest.mark.parametrize("t", [1, 4])
def test_gemv_down_proj_decode(cuda_ok, t):
    """The down_proj decode shapes (K = 14336, N = 4096, MXFP4 2:4) in full."""
    cfg = workloads.down_proj(t=t)
    p = gpu_prepare(cfg["x"], "bf16", "mxfp4", "2:4")
    wq = sharq.FP4Weight.quantize(to_dev(cfg["w"], "bf16"), "mxfp4")
    y = sharq.linear(p, wq, out_dtype=torch.float32)
    sharq.sharq_sync_status()
    ref = oracle.linear_ref(oracle.prepare(cfg["x"], "mxfp4", "2:4"), oracle.quantize_weight(cfg["w"], "mxfp4"))
    assert_close_gemm(y.cpu().numpy(), ref, f"down_proj t={t}")


@pytest.mark.parametrize("fmt,pat", [("nvfp4", "4:8pair"), ("mxfp4", "2:4"), ("nvfp4", "8:16")])
@pytest.mark.parametrize("k,n", [(256, 256), (768, 512)])
@pytest.mark.parametrize("t", [1, 3])
def test_gemv_short_rows(cuda_ok, fmt, pat, k, n, t):
    """Rows shorter than one K chunk: a single partial chunk, most lanes without a unit."""
    x, w = _x(60 + t, t, k), _w(61, n, k)
    p = gpu_prepare(x, "bf16", fmt, pat)
    wq = sharq.FP4Weight.quantize(to_dev(w, "bf16"), fmt)
    y = sharq.linear(p, wq, out_dtype=torch.float32)
    sharq.sharq_sync_status()
    ref = oracle.linear_ref(oracle.prepare(x, fmt, pat), oracle.quantize_weight(w, fmt))
    assert_close_gemm(y.cpu().numpy(), ref, f"gemv short {fmt} {pat} k={k} t={t}")
