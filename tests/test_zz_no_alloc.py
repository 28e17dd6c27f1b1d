"""GPU tests of sharq_prepare_noalloc, the prepare call whose per-row scratch is
a static device array of the library instead of a caller workspace.

Its outputs must equal those of sharq_prepare (bit for bit, the tolerance of
every prepare test) on two calls in a row with different inputs and row
counts, at the row limit too; t above the limit is refused before any launch.
The file is named to be collected last, so it runs both after the other GPU
tests and alone in a fresh process."""
import numpy as np
import pytest
import torch

from gpu_common import readback, to_dev
from activation_sparsity_fp4_b200 import sharq, workloads

pytestmark = pytest.mark.gpu

FIELDS = ("meta", "bb_codes", "bb_scales", "res_codes", "res_scales", "tensor")


def _inputs(seed: int, t: int, k: int):
    rng = np.random.default_rng(seed)
    x = (0.5 * rng.standard_t(3, size=(t, k))).astype(np.float32)
    x[:, rng.permutation(k)[:6]] *= 60.0
    x = workloads.to_bf16_values(x)
    gamma = workloads.to_bf16_values(rng.uniform(0.5, 1.5, k).astype(np.float32))
    return x, gamma


def _noalloc(xd, gd, fmt, pat, act_amax=0.0) -> sharq.Prepared:
    t, k = xd.shape
    out = sharq.Prepared(t, k, fmt, pat, xd.device)
    sharq.sharq_prepare_noalloc(xd.data_ptr(), xd.dtype, gd.data_ptr() if gd is not None else None, 1e-6, act_amax,
                                out.struct)
    return out


def _assert_same(a: sharq.Prepared, b: sharq.Prepared, what: str):
    ga, gb = readback(a), readback(b)
    for f in FIELDS:
        bad = np.argwhere(ga[f] != gb[f])
        assert bad.size == 0, f"{what}: {f} differs at {len(bad)} places, first {bad[:3].tolist()}"


# (format, pattern, with RMSNorm): NVFP4 + RMSNorm + device amax is the case
# that uses the scratch; the others must simply equal sharq_prepare.
CASES = [("nvfp4", "4:8pair", True), ("nvfp4", "8:16", True), ("mxfp4", "2:4", True), ("nvfp4", "4:8pair", False)]


@pytest.mark.parametrize("fmt,pat,norm", CASES)
def test_noalloc_equals_prepare_on_two_calls_in_a_row(fmt, pat, norm):
    k = 1024
    for seed, t in ((21, 1000), (22, 300)):  # second call: new data, fewer rows than the first
        x, gamma = _inputs(seed, t, k)
        xd = to_dev(x, "bf16")
        gd = to_dev(gamma, "bf16") if norm else None
        ref = sharq.prepare(xd, fmt, pat, gd, 1e-6)  # the existing entry point, caller workspace
        got = _noalloc(xd, gd, fmt, pat)
        sharq.sharq_sync_status()
        _assert_same(got, ref, f"{fmt} {pat} norm={norm} t={t}")


def test_noalloc_at_the_row_limit():
    t, k = sharq.NOALLOC_MAX_ROWS, 256
    x, gamma = _inputs(23, t, k)
    xd, gd = to_dev(x, "bf16"), to_dev(gamma, "bf16")
    for _ in range(2):
        ref = sharq.prepare(xd, "nvfp4", "4:8pair", gd, 1e-6)
        got = _noalloc(xd, gd, "nvfp4", "4:8pair")
        sharq.sharq_sync_status()
        _assert_same(got, ref, "t at the static limit")


def test_noalloc_refuses_rows_beyond_the_limit():
    t, k = sharq.NOALLOC_MAX_ROWS + 1, 256
    xd = torch.zeros((t, k), dtype=torch.bfloat16, device="cuda")
    gd = torch.ones(k, dtype=torch.bfloat16, device="cuda")
    before = sharq.sharq_launch_count()
    with pytest.raises(sharq.SharqError) as ei:
        _noalloc(xd, gd, "nvfp4", "4:8pair")
    assert ei.value.status == 5 and "static scratch" in str(ei.value)
    assert sharq.sharq_launch_count() == before
    sharq.sharq_sync_status()
