"""Failure detection on the device without faulting it: a bounded wait that
runs out.

Test flag bit 2 makes the grid-wide exchange of the single-tensor select wait
for one block more than the grid holds, a count that no block ever supplies.
The wait must give up by itself (about a second), record
TOPK_EF_ERR_DEVICE_TIMEOUT in the workspace and let the kernel end, so that
the context stays usable: the next calls on the same workspace are
bit-exact against the oracle again."""
import numpy as np
import pytest
import torch

import datagen
import error_feedback_b200 as ef
from gpu_util import run_compress_steps

pytestmark = pytest.mark.gpu

LR = np.float32(0.1)


def test_bounded_wait_runs_out_then_next_call_is_exact():
    n, k = 1 << 20, 1048
    ws = torch.empty(ef.topk_ef_workspace_bytes(n, k), dtype=torch.uint8, device="cuda")
    g = torch.from_numpy(datagen.flat_normal(0)).cuda()
    res = torch.zeros(n, dtype=torch.float32, device="cuda")
    old = ef.topk_ef_set_test_flags(4)
    try:
        ef.topk_ef_compress(g, res, LR, k, ws=ws)
        assert ef.topk_ef_last_device_status(ws) == ef.ERR_DEVICE_TIMEOUT
    finally:
        ef.topk_ef_set_test_flags(old)
    # the workspace and the context are usable again
    run_compress_steps([datagen.flat_normal(s) for s in (1, 2)], LR, k, ws=ws)
    assert ef.topk_ef_path_info(ws)["fallback"] == 0
