"""Accuracy cost of one shared set of weight codes (oracle only, no GPU).

The sparse tensor-core MMA applies one weight scale per 2b logical K, so one
set of FP4 weight codes can serve both GEMMs of the layer (the SharQ abstract's
shared weight load) only if the weight is quantized in blocks of 2b: 32 for
NVFP4 (format block 16) and 64 for MXFP4 (format block 32).  The alternative
keeps a second code set in the format's own block for the dense residual GEMM
(twice the weight bytes, two weight loads).  This experiment measures the layer
error of both against the unquantized product h . W^T on the pages' layer
shapes (seeded synthetic rows and weights), next to plain dense FP4 for scale.

The orderings asserted are the ones the numbers show with a wide margin; the
numbers themselves are printed (run with -s) and recorded beside the reading.
"""
import numpy as np
import pytest

import oracle
from activation_sparsity_fp4_b200 import workloads


def _rel(y, ref):
    return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))


def _errors(x, w, fmt, pat, gamma=None):
    b = oracle.block_size(fmt)
    prep = oracle.prepare(x, fmt, pat, gamma=gamma, want_float=True)
    h = prep["h"].astype(np.float64)
    y = h @ w.astype(np.float64).T
    gx = float(prep["tensor"][2])
    bu, ru = oracle.decode_prepared(prep)
    bu, ru = bu * gx, ru * gx
    wq = oracle.quantize_weight(w, fmt)
    gw_enc, gw_dec = float(wq["tensor"][1]), float(wq["tensor"][2])
    w_shared = oracle.decode_weight(wq) * gw_dec                     # blocks of 2b, the shared codes
    s16, c16 = oracle.quant_blocks(w, b, fmt, gw_enc)                 # blocks of b, a second code set
    w_own = oracle.dequant_blocks(s16, c16, fmt, gw_dec)
    sx, cx = oracle.quant_blocks(prep["h"], b, fmt, float(prep["tensor"][1]))
    x_dense = oracle.dequant_blocks(sx, cx, fmt, gx)                  # dense FP4 activations, block b
    return {
        "sharq, shared 2b-block weight": _rel((bu + ru) @ w_shared.T, y),
        "sharq, residual GEMM on a b-block weight": _rel(bu @ w_shared.T + ru @ w_own.T, y),
        "sharq, both GEMMs on a b-block weight (not executable)": _rel((bu + ru) @ w_own.T, y),
        "dense FP4, b-block weight": _rel(x_dense @ w_own.T, y),
        "weight alone, 2b blocks": _rel(h @ w_shared.T, y),
        "weight alone, b blocks": _rel(h @ w_own.T, y),
    }


CASES = {
    # Llama-3.1-8B q_proj rows (0.5 t(3), outlier channels, RMSNorm), NVFP4 4:8 pair
    "q_proj nvfp4 4:8pair": ("q_proj", "nvfp4", "4:8pair"),
    # Llama-3.1-8B down_proj rows (SiLU(a) * b), MXFP4 2:4
    "down_proj mxfp4 2:4": ("down_proj", "mxfp4", "2:4"),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_shared_weight_block_cost(case):
    name, fmt, pat = CASES[case]
    cfg = getattr(workloads, name)()
    rows = np.random.default_rng(3).choice(cfg["x"].shape[0], 48, replace=False)
    cols = np.random.default_rng(4).choice(cfg["w"].shape[0], 384, replace=False)
    x, w = cfg["x"][np.sort(rows)], cfg["w"][np.sort(cols)]
    e = _errors(x, w, fmt, pat, cfg.get("gamma"))
    print(f"\n{case}: layer error |Y - h W^T| / |h W^T|")
    for k_, v in e.items():
        print(f"  {k_:<58s} {v:.5f}")
    # the weight's own quantization error grows with the coarser block ...
    assert e["weight alone, 2b blocks"] > e["weight alone, b blocks"]
    # ... and the decomposition still beats dense FP4 with the finer weight
    assert e["sharq, shared 2b-block weight"] < e["dense FP4, b-block weight"]
