"""Accuracy of the three backbones an 8:16 layer can run with (oracle only).

* "8:16": the top 8 of every 16 form the backbone, stored dense and multiplied
  by a dense FP4 GEMM next to the residual one (4*T*N*K on the tensor cores);
* "8:16pair": the same selection re-packed into the 4:8 pair layout of the
  sparse tensor cores (two whole pairs of every 8 ranked by how many of the
  top 8 they hold); what does not fit goes to the residual (3*T*N*K);
* "4:8pair": the NVFP4 4:8 pair pattern itself (SharQ Section 2.2).
The decomposition error |h - deq(B) - deq(R)| and the layer error against the
unquantized product are printed (run with -s) on the Wan2.2 rows (outlier
channels) and the q_proj rows; the orderings asserted hold with a wide margin.
"""
import numpy as np
import pytest

import oracle
from activation_sparsity_fp4_b200 import workloads


def _errors(x, w, gamma, pat):
    prep = oracle.prepare(x, "nvfp4", pat, gamma=gamma, want_float=True)
    h = prep["h"].astype(np.float64)
    dec = np.linalg.norm(h - prep["bdeq"] - prep["rdeq"]) / np.linalg.norm(h)
    kept = np.linalg.norm(prep["bdeq"]) / np.linalg.norm(h)  # share of h carried by the backbone
    y = h @ w.astype(np.float64).T
    yq = oracle.linear_ref(prep, oracle.quantize_weight(w, "nvfp4"))
    return dec, float(np.linalg.norm(yq - y) / np.linalg.norm(y)), kept


@pytest.mark.parametrize("layer", ["wan", "q_proj"])
def test_repacked_8_16_accuracy(layer):
    cfg = getattr(workloads, layer)()
    rows = np.sort(np.random.default_rng(5).choice(cfg["x"].shape[0], 48, replace=False))
    cols = np.sort(np.random.default_rng(6).choice(cfg["w"].shape[0], 256, replace=False))
    x, w = cfg["x"][rows], cfg["w"][cols]
    e = {pat: _errors(x, w, cfg["gamma"], pat) for pat in ("8:16", "8:16pair", "4:8pair")}
    print(f"\n{layer}: decomposition error |h-B-R|/|h|, layer error |Y-hW|/|hW|, backbone share |B|/|h|")
    for pat, (dec, lay, kept) in e.items():
        print(f"  {pat:9s} {dec:.6f}  {lay:.6f}  {kept:.4f}")
    # every form decomposes h to well within the FP4 residual error
    assert all(v[0] < 0.05 for v in e.values())
    # the 8:16 selection keeps at least as much of h in the backbone as either 4:8-pair form
    assert e["8:16"][2] >= e["8:16pair"][2] - 1e-9 and e["8:16"][2] >= e["4:8pair"][2] - 1e-9
