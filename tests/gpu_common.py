"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and read its outputs back in the documented layouts."""
import numpy as np
import torch

import oracle
from _layout import untile_scales
from activation_sparsity_fp4_b200 import sharq

REL_FRO = 1e-4      # GEMM tolerance: relative Frobenius error
MAX_REL = 1e-3      # and per-element |delta| <= 1e-3 * max|Y|


def to_dev(a: np.ndarray, dtype: str):
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dt).cuda()


def gpu_prepare(x, x_dtype, fmt, pat, gamma=None, eps=1e-6, act_amax=0.0):
    xd = to_dev(x, x_dtype)
    gd = to_dev(gamma, x_dtype) if gamma is not None else None
    p = sharq.prepare(xd, fmt, pat, gd, eps, act_amax)
    sharq.sharq_sync_status()
    return p


def readback(p: sharq.Prepared, rows=None) -> dict:
    """Canonical row-major arrays of a GPU Prepared (first t rows or the given rows)."""
    t, k = p.t, p.k
    tp = (t + 127) // 128 * 128
    nv = p.fmt == sharq.NVFP4
    b = 16 if nv else 32
    sel = np.arange(t) if rows is None else np.asarray(rows)
    out = {}
    out["meta"] = p.meta.cpu().numpy()[: tp * (k // 16 if p.pat in (sharq.NM_4_8_PAIR, sharq.NM_8_16_PAIR) else k // 8)].reshape(tp, -1)[sel]
    bbw = k // 2 if p.pat == sharq.NM_8_16 else k // 4
    out["bb_codes"] = p.bb_codes.cpu().numpy()[: tp * bbw].reshape(tp, bbw)[sel]
    sb = k // b if p.pat == sharq.NM_8_16 else k // (2 * b)
    out["bb_scales"] = untile_scales(p.bb_scales.cpu().numpy(), tp, sb)[sel]
    out["res_codes"] = p.res_codes.cpu().numpy()[: tp * k // 2].reshape(tp, k // 2)[sel]
    out["res_scales"] = untile_scales(p.res_scales.cpu().numpy(), tp, k // b)[sel]
    out["tensor"] = p.tensor.cpu().numpy()
    return out


def assert_prep_equal(gpu: dict, ref: dict, pat: str):
    """Bit-exact comparison of prepared outputs (8:16 backbone scales are stored
    twice on the GPU, the dense view)."""
    for name in ("meta", "bb_codes", "res_codes", "res_scales"):
        g, r = gpu[name], ref[name]
        bad = np.argwhere(g != r)
        assert bad.size == 0, f"{name}: {len(bad)} mismatches, first at {bad[:3].tolist()}: gpu {g[tuple(bad[0])]} ref {r[tuple(bad[0])]}"
    g = gpu["bb_scales"]
    if pat == "8:16":
        assert np.array_equal(g[:, 0::2], g[:, 1::2]), "8:16 dense view must repeat each scale"
        g = g[:, 0::2]
    bad = np.argwhere(g != ref["bb_scales"])
    assert bad.size == 0, f"bb_scales: {len(bad)} mismatches, first at {bad[:3].tolist()}"
    np.testing.assert_array_equal(gpu["tensor"], ref["tensor"])


def assert_close_gemm(y: np.ndarray, ref: np.ndarray, what: str = ""):
    y = y.astype(np.float64)
    err = np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-30)
    mx = np.max(np.abs(y - ref))
    lim = MAX_REL * np.max(np.abs(ref))
    assert err <= REL_FRO and mx <= lim, f"{what}: rel_fro={err:.3e} (<= {REL_FRO}), max|d|={mx:.3e} (<= {lim:.3e})"
    return err, mx
