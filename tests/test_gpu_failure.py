"""Failure path without a GPU fault: a device wait on a flag that nothing sets
gives up after its time limit, reports SHARQ_ERR_TIMEOUT through the error
word, and the context stays usable."""
import numpy as np
import pytest

from activation_sparsity_fp4_b200 import sharq
from gpu_common import gpu_prepare

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_ok):
    sharq.sharq_sync_status()  # clean start
    sharq.sharq_selftest_wait_timeout(2_000_000)  # 2 ms
    with pytest.raises(sharq.SharqError) as ei:
        sharq.sharq_sync_status()
    assert ei.value.status == 4
    sharq.sharq_sync_status()  # the word was cleared
    x = np.random.default_rng(0).standard_normal((4, 256)).astype(np.float32)
    p = gpu_prepare(x, "f32", "mxfp4", "2:4")
    assert p.tensor.cpu().numpy()[2] == 1.0
