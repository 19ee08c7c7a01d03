"""Failure detection without a GPU fault.

Every pipeline wait in the kernels is bounded.  A diagnostic entry point runs
that same bounded wait, with a limit of a few milliseconds, on a barrier no
one arrives on: the wait must give up, the status word must report a
timeout, and the context must stay usable for a normal forward afterwards.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu

MOBA_ERR_TIMEOUT = 5


def test_stuck_wait_reports_timeout_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_long_07_b200 import build
    build.build()
    import block_sparse_long_07_b200 as moba
    lib = moba.load_library()
    ws = moba.alloc_workspace(4096)
    ws.zero_()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.moba_selftest_wait_timeout(ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                        20_000_000, stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert moba.last_device_status(ws) == MOBA_ERR_TIMEOUT
    assert moba.last_device_status(ws) == 0  # reading clears the latch
    # the context still runs the real pipeline
    w = S.Workload("after_timeout", [1024], 4, 2, 128, 256, 3, seed=3)
    q, k, v = S.make_qkv(w, "cuda")
    q4, k4, v4 = (x.view(1, 1024, x.shape[1], 128) for x in (q, k, v))
    o, lse = moba.forward(q4, k4, v4, 256, 3)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
