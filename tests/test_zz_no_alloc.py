"""topk_ef_compress_static against topk_ef_compress.

topk_ef_compress_static is the compress step for callers that cannot
allocate device memory (and so cannot hand the library a workspace): it runs
in a fixed scratch array inside the library.  Called through the C ABI, it
must give exactly the results of topk_ef_compress (indices, values and the
updated residual, bit for bit with NaNs compared as NaNs) on two calls in a
row, so the second call also shows that what the first left in the shared
scratch does not leak into its result.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import datagen
import error_feedback_b200 as ef
from gpu_util import same_bits

pytestmark = pytest.mark.gpu

LR = np.float32(0.1)


def _static_call(g, r, k, oi, ov):
    L = ef.lib()
    return L.topk_ef_compress_static(g.data_ptr(), r.data_ptr(), g.numel(), ctypes.c_float(LR),
                                     k, oi.data_ptr(), ov.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("n,k", [(1 << 20, 1048), (datagen.RESNET50_N, 25_557),
                                 (3_000_017, 30_000)])
def test_static_scratch_matches_workspace_call(n, k):
    if n == datagen.RESNET50_N:
        grads = [datagen.resnet50_mix(s) for s in range(2)]
    else:
        rng = np.random.default_rng(n)
        grads = [rng.laplace(0, 1e-3, n).astype(np.float32) for _ in range(2)]
    res_ws = torch.zeros(n, dtype=torch.float32, device="cuda")
    res_st = torch.zeros(n, dtype=torch.float32, device="cuda")
    ws = torch.empty(ef.topk_ef_workspace_bytes(n, k), dtype=torch.uint8, device="cuda")
    for step, g in enumerate(grads):
        dg = torch.from_numpy(g).cuda()
        ia, va = ef.topk_ef_compress(dg, res_ws, LR, k, ws=ws)
        ib = torch.empty(k, dtype=torch.int32, device="cuda")
        vb = torch.empty(k, dtype=torch.float32, device="cuda")
        rc = _static_call(dg, res_st, k, ib, vb)
        assert rc == 0, ef.status_string(rc)
        st = ef.lib().topk_ef_static_last_device_status(torch.cuda.current_stream().cuda_stream)
        assert st == 0, ef.status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(ia, ib), f"step {step}: indices differ"
        assert same_bits(va.cpu().numpy(), vb.cpu().numpy()).all(), f"step {step}: values differ"
        assert same_bits(res_ws.cpu().numpy(), res_st.cpu().numpy()).all(), \
            f"step {step}: residuals differ"


def test_static_scratch_rejects_oversized_problem():
    n, k = 2_000_000_000, 1_000_000   # workspace far above the 32 MiB array
    assert ef.topk_ef_workspace_bytes(n, k) > (32 << 20)
    L = ef.lib()
    rc = L.topk_ef_compress_static(16, 16, n, ctypes.c_float(LR), k, 16, 16, None)
    assert rc == ef.ERR_WORKSPACE
