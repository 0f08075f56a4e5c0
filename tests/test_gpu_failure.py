"""Failure detection on the device without faulting it: a bounded wait that
runs out.

Test flag bit 2 makes one wait of the call impossible to satisfy: for a small
tensor (small_kernel), block 0's wait for every block's arrival also waits
for one block past the grid; for a larger single tensor (flat_select_kernel),
the grid-wide exchange waits for one block more than the grid holds.  No
block ever supplies it.  The wait must give up by itself (about a second),
record TOPK_EF_ERR_DEVICE_TIMEOUT in the workspace and let the kernel end,
so that the context stays usable: the next calls on the same workspace are
bit-exact against the oracle again."""
import numpy as np
import pytest
import torch

import datagen
import error_feedback_b200 as ef
from gpu_util import run_compress_steps

pytestmark = pytest.mark.gpu

LR = np.float32(0.1)


@pytest.mark.parametrize("n,k", [(1 << 20, 1048), (3_000_017, 3000)])
def test_bounded_wait_runs_out_then_next_call_is_exact(n, k):
    ws = torch.empty(ef.topk_ef_workspace_bytes(n, k), dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(n)
    g = torch.from_numpy(rng.standard_normal(n).astype(np.float32)).cuda()
    res = torch.zeros(n, dtype=torch.float32, device="cuda")
    old = ef.topk_ef_set_test_flags(4)
    try:
        ef.topk_ef_compress(g, res, LR, k, ws=ws)
        assert ef.topk_ef_last_device_status(ws) == ef.ERR_DEVICE_TIMEOUT
    finally:
        ef.topk_ef_set_test_flags(old)
    # the workspace and the context are usable again, on every path the
    # tensor can take (the residual zeroed between steps keeps the previous
    # call's threshold usable, so the later steps take it)
    grads = [rng.standard_normal(n).astype(np.float32) for _ in range(3)]
    paths = []
    run_compress_steps(grads, LR, k, ws=ws, paths=paths, zero_between=True)
    assert paths[-1]["fallback"] == 0, paths
