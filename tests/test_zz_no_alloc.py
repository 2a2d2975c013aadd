"""The allocation-free GEMV entry point (qhl_qgemv_noalloc).

It serves callers that cannot allocate device memory when they call the GEMV
(a memory pool that already owns the GPU, or a loop that must not pay for
cudaMalloc's device synchronisation): its scratch is one static device array.
These tests check, through the C ABI, that it returns what the regular entry
point returns, on two calls in a row (the array keeps the previous call's
contents, so the second call shows that stale scratch does not leak into the
result), and that problems larger than the array are refused up front.  The
file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

import synth
from synth import Q4_0, Q8_0
from stage_helpers import TOL, rel_err_rows


def test_noalloc_rejects_problems_beyond_its_static_scratch():
    import quantized_hybrid_layer_b200 as q
    from quantized_hybrid_layer_b200 import build as b
    b.build()
    lib = q.lib()
    # 16 tokens x 18688 columns need 73 chunks x 2048 bytes x 16 = 2.28 MiB of input
    # scratch, one chunk past the 2.25 MiB region: refused before any device work
    assert lib.qhl_qgemv_noalloc(2, 64, 18688, 16, 16, 16, 16, None) == -1
    assert b"exceeds" in lib.qhl_last_error()
    assert lib.qhl_qgemv_noalloc(2, 64, 256, None, None, 1, None, None) == -1


@pytest.mark.gpu
def test_noalloc_gemv_matches_the_regular_entry_point_on_two_calls():
    import torch
    import quantized_hybrid_layer_b200 as q
    assert torch.cuda.is_available(), "GPU test needs CUDA"

    def packed(qtype, W):
        rows, nb, _ = W.shape
        g = torch.from_numpy(np.ascontiguousarray(W).reshape(-1)).cuda()
        P = torch.empty(q.qhl_packed_bytes(qtype, rows, nb * 32), dtype=torch.uint8, device="cuda")
        q.qhl_repack(qtype, rows, nb * 32, g, P)
        return P

    # the last case fills the input region exactly: 16 tokens x 72 chunks x 2048
    # bytes = 2.25 MiB, the largest problem the static array accepts
    for seed, qtype, rows, cols, n in ((61, Q4_0, 1000, 5120, 1), (62, Q8_0, 700, 17408, 16),
                                       (63, Q4_0, 130, 18432, 16)):
        W, x = synth.gemv_problem(seed, rows, cols, n, qtype)
        P = packed(qtype, W)
        xt = torch.from_numpy(x).cuda()
        y_ref = torch.empty((n, rows), dtype=torch.float32, device="cuda")
        y_na = torch.full((n, rows), float("nan"), dtype=torch.float32, device="cuda")
        q.qhl_qgemv(qtype, rows, cols, P, xt, y_ref)
        q.qhl_qgemv_noalloc(qtype, rows, cols, P, xt, y_na)
        torch.cuda.synchronize()
        got, ref = y_na.cpu().numpy(), y_ref.cpu().numpy()
        assert max(rel_err_rows(got, ref)) <= TOL
        assert np.array_equal(got, ref)          # same kernels: identical in fact
